"""Thin ctypes binding of libkvattn.so with the C entry points' names.

Argument marshalling only: tensors are checked for device, dtype, shape and layout,
their data pointers and the current CUDA stream are passed to the C ABI
(include/kvattn.h), and a non-zero status is raised as KvattnError.  Every step of the
computation runs in the library's CUDA kernels; there is no fallback of any kind.  If
libkvattn.so is missing the first call raises (build it with
``python -m mla_kv_cache_b200.build``).
"""
import ctypes
import os
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libkvattn.so")

KVATTN_OK = 0
KVATTN_ERR_INVALID_ARG = 1
KVATTN_ERR_UNSUPPORTED = 2
KVATTN_ERR_MISALIGNED = 3
KVATTN_ERR_CUDA = 4
KVATTN_ERR_NO_MEMORY = 5

# Every function the header declares, with its ctypes signature.
_c_u16p = ctypes.c_void_p
_SIGNATURES = {
    "kvattn_gqa_decode": (ctypes.c_int, [_c_u16p, _c_u16p, _c_u16p, ctypes.c_void_p, ctypes.c_int,
                                         ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p,
                                         ctypes.c_void_p]),
    "kvattn_mla_decode": (ctypes.c_int, [_c_u16p, _c_u16p, _c_u16p, _c_u16p, ctypes.c_void_p,
                                         ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_int, ctypes.c_float, ctypes.c_void_p,
                                         ctypes.c_void_p, ctypes.c_void_p]),
    "kvattn_gqa_decode_noalloc": (ctypes.c_int, [_c_u16p, _c_u16p, _c_u16p, ctypes.c_void_p,
                                                 ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                 ctypes.c_int, ctypes.c_int, ctypes.c_float,
                                                 ctypes.c_void_p, ctypes.c_void_p,
                                                 ctypes.c_void_p]),
    "kvattn_gqa_decode_multi": (ctypes.c_int, [_c_u16p, _c_u16p, _c_u16p, ctypes.c_void_p, ctypes.c_int,
                                               ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                               ctypes.c_int, ctypes.c_float, ctypes.c_int, ctypes.c_void_p,
                                               ctypes.c_void_p, ctypes.c_void_p]),
    "kvattn_gqa_decode_fp8": (ctypes.c_int, [_c_u16p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                             ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                             ctypes.c_int, ctypes.c_float, ctypes.c_float, ctypes.c_float,
                                             ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]),
    "kvattn_gqa_decode_fp8_paged": (ctypes.c_int, [_c_u16p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                                   ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                   ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                   ctypes.c_float, ctypes.c_float, ctypes.c_float,
                                                   ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]),
    "kvattn_gqa_decode_paged": (ctypes.c_int, [_c_u16p, _c_u16p, _c_u16p, ctypes.c_void_p, ctypes.c_void_p,
                                               ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                               ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float,
                                               ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]),
    "kvattn_mla_decode_paged": (ctypes.c_int, [_c_u16p, _c_u16p, _c_u16p, _c_u16p, ctypes.c_void_p,
                                               ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                               ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                               ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p,
                                               ctypes.c_void_p]),
    "kvattn_rope_append": (ctypes.c_int, [_c_u16p, _c_u16p, _c_u16p, ctypes.c_void_p, _c_u16p, _c_u16p,
                                          ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_int, ctypes.c_float, ctypes.c_int, ctypes.c_void_p]),
    "kvattn_rope_append_fp8": (ctypes.c_int, [_c_u16p, _c_u16p, _c_u16p, ctypes.c_void_p, ctypes.c_void_p,
                                              ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                              ctypes.c_int, ctypes.c_int, ctypes.c_float, ctypes.c_int,
                                              ctypes.c_float, ctypes.c_float, ctypes.c_void_p]),
    "kvattn_mla_rope_append": (ctypes.c_int, [_c_u16p, _c_u16p, _c_u16p, ctypes.c_void_p, _c_u16p,
                                              _c_u16p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                              ctypes.c_int, ctypes.c_int, ctypes.c_float, ctypes.c_int,
                                              ctypes.c_void_p]),
    "kvattn_mla_decode_fp8": (ctypes.c_int, [_c_u16p, _c_u16p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                             ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                             ctypes.c_float, ctypes.c_float, ctypes.c_float, ctypes.c_void_p,
                                             ctypes.c_void_p, ctypes.c_void_p]),
    "kvattn_mla_decode_fp8_paged": (ctypes.c_int, [_c_u16p, _c_u16p, ctypes.c_void_p, ctypes.c_void_p,
                                                   ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                                                   ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                   ctypes.c_int, ctypes.c_float, ctypes.c_float, ctypes.c_float,
                                                   ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]),
    "kvattn_mla_rope_append_fp8": (ctypes.c_int, [_c_u16p, _c_u16p, _c_u16p, ctypes.c_void_p, ctypes.c_void_p,
                                                  ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                  ctypes.c_int, ctypes.c_int, ctypes.c_float, ctypes.c_int,
                                                  ctypes.c_float, ctypes.c_float, ctypes.c_void_p]),
    "kvattn_mla_decode_multi": (ctypes.c_int, [_c_u16p, _c_u16p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                               ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                               ctypes.c_int, ctypes.c_float, ctypes.c_int, ctypes.c_float,
                                               ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]),
    "kvattn_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "kvattn_last_error_detail": (ctypes.c_char_p, []),
    "kvattn_version": (ctypes.c_int, []),
    "kvattn_release_workspace": (None, []),
    "kvattn_read_device_flags": (ctypes.c_int, [ctypes.POINTER(ctypes.c_uint)]),
    "kvattn_clear_device_flags": (ctypes.c_int, []),
    "kvattn_debug_wait_probe": (ctypes.c_int, [ctypes.c_int, ctypes.c_void_p]),
    "kvattn_kernel_launches": (ctypes.c_ulonglong, []),
    "kvattn_debug_set_workers": (None, [ctypes.c_int, ctypes.c_int]),
    "kvattn_debug_set_gqa_kernel": (None, [ctypes.c_int]),
}

_lib = None
_lock = threading.Lock()


class KvattnError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        detail = ""
        if status in (KVATTN_ERR_CUDA, KVATTN_ERR_NO_MEMORY):
            detail = ": " + lib().kvattn_last_error_detail().decode()
        super().__init__(f"{where} -> {lib().kvattn_status_string(status).decode()}{detail}")


def lib():
    """The loaded libkvattn.so (loaded on first use; raises if it is not built)."""
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                if not os.path.exists(LIB_PATH):
                    raise RuntimeError(f"{LIB_PATH} is missing: run python -m mla_kv_cache_b200.build")
                h = ctypes.CDLL(LIB_PATH)
                for name, (res, args) in _SIGNATURES.items():
                    f = getattr(h, name)
                    f.restype = res
                    f.argtypes = args
                _lib = h
    return _lib


def _stream_handle(stream):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(t, name, dtype, shape=None):
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def kvattn_gqa_decode(q, k_cache, v_cache, seq_lens, scale, out=None, lse=None, stream=None):
    """GQA / MQA / MHA decode step (see include/kvattn.h, kvattn_gqa_decode).

    q [B, n_q, d] bf16, k_cache / v_cache [B, n_kv, max_seq_len, d] bf16, seq_lens [B]
    int32 -- all on the current CUDA device.  Returns (out [B, n_q, d] fp32,
    lse [B, n_q] fp32); out / lse may be passed in preallocated.
    """
    import torch
    B, n_q, d = q.shape
    n_kv, T = k_cache.shape[1], k_cache.shape[2]
    _check(q, "q", torch.bfloat16)
    _check(k_cache, "k_cache", torch.bfloat16, (B, n_kv, T, d))
    _check(v_cache, "v_cache", torch.bfloat16, (B, n_kv, T, d))
    _check(seq_lens, "seq_lens", torch.int32, (B,))
    if out is None:
        out = torch.empty((B, n_q, d), dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty((B, n_q), dtype=torch.float32, device=q.device)
    _check(out, "out", torch.float32, (B, n_q, d))
    _check(lse, "lse", torch.float32, (B, n_q))
    st = lib().kvattn_gqa_decode(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
                                 seq_lens.data_ptr(), T, B, n_q, n_kv, d, float(scale),
                                 out.data_ptr(), lse.data_ptr(), _stream_handle(stream))
    if st != KVATTN_OK:
        raise KvattnError(st, "kvattn_gqa_decode")
    return out, lse


def kvattn_mla_decode(q_latent, q_rope, latent_cache, rope_cache, seq_lens, scale, out=None,
                      lse=None, stream=None):
    """Absorbed-MLA decode step (see include/kvattn.h, kvattn_mla_decode).

    q_latent [B, H, 512], q_rope [B, H, 64], latent_cache [B, T, 512],
    rope_cache [B, T, 64] bf16, seq_lens [B] int32.  Returns (out [B, H, 512] fp32,
    lse [B, H] fp32).
    """
    import torch
    B, H, dc = q_latent.shape
    dr = q_rope.shape[2]
    T = latent_cache.shape[1]
    _check(q_latent, "q_latent", torch.bfloat16)
    _check(q_rope, "q_rope", torch.bfloat16, (B, H, dr))
    _check(latent_cache, "latent_cache", torch.bfloat16, (B, T, dc))
    _check(rope_cache, "rope_cache", torch.bfloat16, (B, T, dr))
    _check(seq_lens, "seq_lens", torch.int32, (B,))
    if out is None:
        out = torch.empty((B, H, dc), dtype=torch.float32, device=q_latent.device)
    if lse is None:
        lse = torch.empty((B, H), dtype=torch.float32, device=q_latent.device)
    _check(out, "out", torch.float32, (B, H, dc))
    _check(lse, "lse", torch.float32, (B, H))
    st = lib().kvattn_mla_decode(q_latent.data_ptr(), q_rope.data_ptr(), latent_cache.data_ptr(),
                                 rope_cache.data_ptr(), seq_lens.data_ptr(), T, B, H, dc, dr,
                                 float(scale), out.data_ptr(), lse.data_ptr(),
                                 _stream_handle(stream))
    if st != KVATTN_OK:
        raise KvattnError(st, "kvattn_mla_decode")
    return out, lse


def kvattn_gqa_decode_noalloc(q, k_cache, v_cache, seq_lens, scale, out=None, lse=None,
                              stream=None):
    """kvattn_gqa_decode without any allocation by the library (include/kvattn.h).

    For callers that cannot let the library allocate device memory; the scratch is a
    fixed array inside the library that all calls share, so calls must be ordered on
    one stream.  out / lse are allocated here by torch only when not passed in.
    """
    import torch
    B, n_q, d = q.shape
    n_kv, T = k_cache.shape[1], k_cache.shape[2]
    _check(q, "q", torch.bfloat16)
    _check(k_cache, "k_cache", torch.bfloat16, (B, n_kv, T, d))
    _check(v_cache, "v_cache", torch.bfloat16, (B, n_kv, T, d))
    _check(seq_lens, "seq_lens", torch.int32, (B,))
    if out is None:
        out = torch.empty((B, n_q, d), dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty((B, n_q), dtype=torch.float32, device=q.device)
    _check(out, "out", torch.float32, (B, n_q, d))
    _check(lse, "lse", torch.float32, (B, n_q))
    st = lib().kvattn_gqa_decode_noalloc(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
                                         seq_lens.data_ptr(), T, B, n_q, n_kv, d, float(scale),
                                         out.data_ptr(), lse.data_ptr(), _stream_handle(stream))
    if st != KVATTN_OK:
        raise KvattnError(st, "kvattn_gqa_decode_noalloc")
    return out, lse


def kvattn_status_string(status):
    return lib().kvattn_status_string(int(status)).decode()


def kvattn_last_error_detail():
    return lib().kvattn_last_error_detail().decode()


def kvattn_version():
    return int(lib().kvattn_version())


def kvattn_release_workspace():
    lib().kvattn_release_workspace()


def kvattn_read_device_flags():
    v = ctypes.c_uint(0)
    st = lib().kvattn_read_device_flags(ctypes.byref(v))
    if st != KVATTN_OK:
        raise KvattnError(st, "kvattn_read_device_flags")
    return int(v.value)


def kvattn_clear_device_flags():
    st = lib().kvattn_clear_device_flags()
    if st != KVATTN_OK:
        raise KvattnError(st, "kvattn_clear_device_flags")


def kvattn_kernel_launches():
    """Kernels the library has launched from this thread (include/kvattn.h)."""
    return int(lib().kvattn_kernel_launches())


def kvattn_debug_wait_probe(limit_us, stream=None):
    """Test hook (include/kvattn.h, kvattn_debug_wait_probe): one bounded wait on a barrier
    nothing completes, cut to about limit_us; it runs out and sets bit 0 of the device flags."""
    st = lib().kvattn_debug_wait_probe(int(limit_us), _stream_handle(stream))
    if st != KVATTN_OK:
        raise KvattnError(st, "kvattn_debug_wait_probe")


def kvattn_debug_set_workers(workers, min_tiles=0):
    lib().kvattn_debug_set_workers(int(workers), int(min_tiles))


def kvattn_debug_set_gqa_kernel(which):
    """0: built-in choice, 1: warp-level MMA kernel, 2: tcgen05 kernel."""
    lib().kvattn_debug_set_gqa_kernel(int(which))


def kvattn_rope_append(q, k_new, v_new, positions, k_cache, v_cache, rope_base=10000.0,
                       interleaved=False, stream=None):
    """Rotary embedding of the new token + cache append (include/kvattn.h,
    kvattn_rope_append): q [B, n_q, d] is rotated in place; the rotated k_new
    [B, n_kv, d] and v_new go to the caches [B, n_kv, T, d] at positions [B] (int32)."""
    import torch
    B, n_q, d = q.shape
    n_kv, T = k_cache.shape[1], k_cache.shape[2]
    _check(q, "q", torch.bfloat16)
    _check(k_new, "k_new", torch.bfloat16, (B, n_kv, d))
    _check(v_new, "v_new", torch.bfloat16, (B, n_kv, d))
    _check(positions, "positions", torch.int32, (B,))
    _check(k_cache, "k_cache", torch.bfloat16, (B, n_kv, T, d))
    _check(v_cache, "v_cache", torch.bfloat16, (B, n_kv, T, d))
    st = lib().kvattn_rope_append(q.data_ptr(), k_new.data_ptr(), v_new.data_ptr(), positions.data_ptr(),
                                  k_cache.data_ptr(), v_cache.data_ptr(), T, B, n_q, n_kv, d,
                                  float(rope_base), int(bool(interleaved)), _stream_handle(stream))
    if st != KVATTN_OK:
        raise KvattnError(st, "kvattn_rope_append")


def kvattn_rope_append_fp8(q, k_new, v_new, positions, k_cache, v_cache, k_scale, v_scale, rope_base=10000.0,
                           interleaved=False, stream=None):
    """kvattn_rope_append into an E4M3 cache (include/kvattn.h, kvattn_rope_append_fp8):
    q [B, n_q, d] bf16 rotated in place; the rotated k_new and v_new [B, n_kv, d] bf16 are
    stored as codes of value / scale in the caches [B, n_kv, T, d] (float8_e4m3fn or uint8)
    at positions [B] (int32)."""
    import torch
    B, n_q, d = q.shape
    n_kv, T = k_cache.shape[1], k_cache.shape[2]
    _check(q, "q", torch.bfloat16)
    _check(k_new, "k_new", torch.bfloat16, (B, n_kv, d))
    _check(v_new, "v_new", torch.bfloat16, (B, n_kv, d))
    _check(positions, "positions", torch.int32, (B,))
    _check_e4m3(k_cache, "k_cache", (B, n_kv, T, d))
    _check_e4m3(v_cache, "v_cache", (B, n_kv, T, d))
    st = lib().kvattn_rope_append_fp8(q.data_ptr(), k_new.data_ptr(), v_new.data_ptr(), positions.data_ptr(),
                                      k_cache.data_ptr(), v_cache.data_ptr(), T, B, n_q, n_kv, d, float(rope_base),
                                      int(bool(interleaved)), float(k_scale), float(v_scale), _stream_handle(stream))
    if st != KVATTN_OK:
        raise KvattnError(st, "kvattn_rope_append_fp8")


def kvattn_mla_rope_append(q_rope, latent_new, rope_new, positions, latent_cache, rope_cache,
                           rope_base=10000.0, interleaved=False, stream=None):
    """MLA variant (include/kvattn.h, kvattn_mla_rope_append): q_rope [B, H, r] rotated in
    place; rope_new [B, r] rotated into rope_cache [B, T, r], latent_new [B, c] copied into
    latent_cache [B, T, c], both at positions [B]."""
    import torch
    B, H, r = q_rope.shape
    T, c = latent_cache.shape[1], latent_cache.shape[2]
    _check(q_rope, "q_rope", torch.bfloat16)
    _check(latent_new, "latent_new", torch.bfloat16, (B, c))
    _check(rope_new, "rope_new", torch.bfloat16, (B, r))
    _check(positions, "positions", torch.int32, (B,))
    _check(latent_cache, "latent_cache", torch.bfloat16, (B, T, c))
    _check(rope_cache, "rope_cache", torch.bfloat16, (B, T, r))
    st = lib().kvattn_mla_rope_append(q_rope.data_ptr(), latent_new.data_ptr(), rope_new.data_ptr(),
                                      positions.data_ptr(), latent_cache.data_ptr(), rope_cache.data_ptr(),
                                      T, B, H, c, r, float(rope_base), int(bool(interleaved)),
                                      _stream_handle(stream))
    if st != KVATTN_OK:
        raise KvattnError(st, "kvattn_mla_rope_append")


def kvattn_gqa_decode_paged(q, k_pages, v_pages, block_table, seq_lens, scale, out=None, lse=None,
                            stream=None):
    """GQA decode over a paged cache (include/kvattn.h, kvattn_gqa_decode_paged):
    k_pages / v_pages [num_pages, n_kv, page_size, d] bf16, block_table [B, max_pages]
    int32, seq_lens [B] int32.  Returns (out [B, n_q, d] fp32, lse [B, n_q] fp32)."""
    import torch
    B, n_q, d = q.shape
    P, n_kv, S = k_pages.shape[0], k_pages.shape[1], k_pages.shape[2]
    M = block_table.shape[1]
    _check(q, "q", torch.bfloat16)
    _check(k_pages, "k_pages", torch.bfloat16, (P, n_kv, S, d))
    _check(v_pages, "v_pages", torch.bfloat16, (P, n_kv, S, d))
    _check(block_table, "block_table", torch.int32, (B, M))
    _check(seq_lens, "seq_lens", torch.int32, (B,))
    if out is None:
        out = torch.empty((B, n_q, d), dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty((B, n_q), dtype=torch.float32, device=q.device)
    _check(out, "out", torch.float32, (B, n_q, d))
    _check(lse, "lse", torch.float32, (B, n_q))
    st = lib().kvattn_gqa_decode_paged(q.data_ptr(), k_pages.data_ptr(), v_pages.data_ptr(),
                                       block_table.data_ptr(), seq_lens.data_ptr(), P, S, M, B, n_q, n_kv,
                                       d, float(scale), out.data_ptr(), lse.data_ptr(),
                                       _stream_handle(stream))
    if st != KVATTN_OK:
        raise KvattnError(st, "kvattn_gqa_decode_paged")
    return out, lse


def _check_e4m3(t, name, shape):
    """An E4M3 cache: float8_e4m3fn or uint8 codes."""
    import torch
    if t.dtype not in (torch.float8_e4m3fn, torch.uint8):
        raise ValueError(f"{name} must be float8_e4m3fn (or uint8 codes), got {t.dtype}")
    _check(t, name, t.dtype, shape)


def kvattn_gqa_decode_fp8(q, k_cache, v_cache, seq_lens, scale, k_scale, v_scale, window=0, out=None, lse=None,
                          stream=None):
    """Decode over an E4M3 cache (include/kvattn.h, kvattn_gqa_decode_fp8): q [B, n_q, d]
    (one new token) or [B, L, n_q, d] bf16, caches [B, n_kv, T, d] float8_e4m3fn (or
    uint8 codes), value = code * k_scale / v_scale.  Returns (out, lse) shaped like q
    without / with its L axis, fp32."""
    import torch
    single = q.dim() == 3
    q4 = q.unsqueeze(1) if single else q
    B, L, n_q, d = q4.shape
    n_kv, T = k_cache.shape[1], k_cache.shape[2]
    _check(q4, "q", torch.bfloat16)
    _check_e4m3(k_cache, "k_cache", (B, n_kv, T, d))
    _check_e4m3(v_cache, "v_cache", (B, n_kv, T, d))
    _check(seq_lens, "seq_lens", torch.int32, (B,))
    shape_o, shape_l = ((B, n_q, d), (B, n_q)) if single else ((B, L, n_q, d), (B, L, n_q))
    if out is None:
        out = torch.empty(shape_o, dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty(shape_l, dtype=torch.float32, device=q.device)
    _check(out, "out", torch.float32, shape_o)
    _check(lse, "lse", torch.float32, shape_l)
    st = lib().kvattn_gqa_decode_fp8(q4.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), seq_lens.data_ptr(),
                                     T, B, L, n_q, n_kv, d, float(scale), float(k_scale), float(v_scale),
                                     int(window), out.data_ptr(), lse.data_ptr(), _stream_handle(stream))
    if st != KVATTN_OK:
        raise KvattnError(st, "kvattn_gqa_decode_fp8")
    return out, lse


def kvattn_gqa_decode_fp8_paged(q, k_pages, v_pages, block_table, seq_lens, scale, k_scale, v_scale, out=None,
                                lse=None, stream=None):
    """kvattn_gqa_decode_fp8 over a paged E4M3 cache (include/kvattn.h,
    kvattn_gqa_decode_fp8_paged): k_pages / v_pages [num_pages, n_kv, page_size, d]
    codes, block_table [B, max_pages] int32.  Returns (out [B, n_q, d], lse [B, n_q])."""
    import torch
    B, n_q, d = q.shape
    P, n_kv, S = k_pages.shape[0], k_pages.shape[1], k_pages.shape[2]
    M = block_table.shape[1]
    _check(q, "q", torch.bfloat16)
    _check_e4m3(k_pages, "k_pages", (P, n_kv, S, d))
    _check_e4m3(v_pages, "v_pages", (P, n_kv, S, d))
    _check(block_table, "block_table", torch.int32, (B, M))
    _check(seq_lens, "seq_lens", torch.int32, (B,))
    if out is None:
        out = torch.empty((B, n_q, d), dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty((B, n_q), dtype=torch.float32, device=q.device)
    _check(out, "out", torch.float32, (B, n_q, d))
    _check(lse, "lse", torch.float32, (B, n_q))
    st = lib().kvattn_gqa_decode_fp8_paged(q.data_ptr(), k_pages.data_ptr(), v_pages.data_ptr(),
                                           block_table.data_ptr(), seq_lens.data_ptr(), P, S, M, B, n_q, n_kv, d,
                                           float(scale), float(k_scale), float(v_scale), out.data_ptr(),
                                           lse.data_ptr(), _stream_handle(stream))
    if st != KVATTN_OK:
        raise KvattnError(st, "kvattn_gqa_decode_fp8_paged")
    return out, lse


def kvattn_mla_decode_paged(q_latent, q_rope, latent_pages, rope_pages, block_table, seq_lens, scale,
                            out=None, lse=None, stream=None):
    """MLA decode over a paged cache (include/kvattn.h, kvattn_mla_decode_paged):
    latent_pages [P, page_size, 512], rope_pages [P, page_size, 64] bf16."""
    import torch
    B, H, dc = q_latent.shape
    dr = q_rope.shape[2]
    P, S = latent_pages.shape[0], latent_pages.shape[1]
    M = block_table.shape[1]
    _check(q_latent, "q_latent", torch.bfloat16)
    _check(q_rope, "q_rope", torch.bfloat16, (B, H, dr))
    _check(latent_pages, "latent_pages", torch.bfloat16, (P, S, dc))
    _check(rope_pages, "rope_pages", torch.bfloat16, (P, S, dr))
    _check(block_table, "block_table", torch.int32, (B, M))
    _check(seq_lens, "seq_lens", torch.int32, (B,))
    if out is None:
        out = torch.empty((B, H, dc), dtype=torch.float32, device=q_latent.device)
    if lse is None:
        lse = torch.empty((B, H), dtype=torch.float32, device=q_latent.device)
    _check(out, "out", torch.float32, (B, H, dc))
    _check(lse, "lse", torch.float32, (B, H))
    st = lib().kvattn_mla_decode_paged(q_latent.data_ptr(), q_rope.data_ptr(), latent_pages.data_ptr(),
                                       rope_pages.data_ptr(), block_table.data_ptr(), seq_lens.data_ptr(), P,
                                       S, M, B, H, dc, dr, float(scale), out.data_ptr(), lse.data_ptr(),
                                       _stream_handle(stream))
    if st != KVATTN_OK:
        raise KvattnError(st, "kvattn_mla_decode_paged")
    return out, lse


def kvattn_mla_decode_fp8(q_latent, q_rope, latent_cache, rope_cache, seq_lens, scale, latent_scale, rope_scale,
                          out=None, lse=None, stream=None):
    """Absorbed-MLA decode over an E4M3 cache (include/kvattn.h, kvattn_mla_decode_fp8):
    latent_cache [B, T, 512], rope_cache [B, T, 64] float8_e4m3fn (or uint8 codes), value =
    code * latent_scale / rope_scale.  Returns (out [B, H, 512], lse [B, H]) fp32."""
    import torch
    B, H, dc = q_latent.shape
    dr = q_rope.shape[2]
    T = latent_cache.shape[1]
    _check(q_latent, "q_latent", torch.bfloat16)
    _check(q_rope, "q_rope", torch.bfloat16, (B, H, dr))
    _check_e4m3(latent_cache, "latent_cache", (B, T, dc))
    _check_e4m3(rope_cache, "rope_cache", (B, T, dr))
    _check(seq_lens, "seq_lens", torch.int32, (B,))
    if out is None:
        out = torch.empty((B, H, dc), dtype=torch.float32, device=q_latent.device)
    if lse is None:
        lse = torch.empty((B, H), dtype=torch.float32, device=q_latent.device)
    _check(out, "out", torch.float32, (B, H, dc))
    _check(lse, "lse", torch.float32, (B, H))
    st = lib().kvattn_mla_decode_fp8(q_latent.data_ptr(), q_rope.data_ptr(), latent_cache.data_ptr(),
                                     rope_cache.data_ptr(), seq_lens.data_ptr(), T, B, H, dc, dr, float(scale),
                                     float(latent_scale), float(rope_scale), out.data_ptr(), lse.data_ptr(),
                                     _stream_handle(stream))
    if st != KVATTN_OK:
        raise KvattnError(st, "kvattn_mla_decode_fp8")
    return out, lse


def kvattn_mla_decode_fp8_paged(q_latent, q_rope, latent_pages, rope_pages, block_table, seq_lens, scale,
                                latent_scale, rope_scale, out=None, lse=None, stream=None):
    """kvattn_mla_decode_fp8 over a paged cache (include/kvattn.h): latent_pages [P, page_size,
    512], rope_pages [P, page_size, 64] E4M3 codes, block_table [B, max_pages] int32."""
    import torch
    B, H, dc = q_latent.shape
    dr = q_rope.shape[2]
    P, S = latent_pages.shape[0], latent_pages.shape[1]
    M = block_table.shape[1]
    _check(q_latent, "q_latent", torch.bfloat16)
    _check(q_rope, "q_rope", torch.bfloat16, (B, H, dr))
    _check_e4m3(latent_pages, "latent_pages", (P, S, dc))
    _check_e4m3(rope_pages, "rope_pages", (P, S, dr))
    _check(block_table, "block_table", torch.int32, (B, M))
    _check(seq_lens, "seq_lens", torch.int32, (B,))
    if out is None:
        out = torch.empty((B, H, dc), dtype=torch.float32, device=q_latent.device)
    if lse is None:
        lse = torch.empty((B, H), dtype=torch.float32, device=q_latent.device)
    _check(out, "out", torch.float32, (B, H, dc))
    _check(lse, "lse", torch.float32, (B, H))
    st = lib().kvattn_mla_decode_fp8_paged(q_latent.data_ptr(), q_rope.data_ptr(), latent_pages.data_ptr(),
                                           rope_pages.data_ptr(), block_table.data_ptr(), seq_lens.data_ptr(), P,
                                           S, M, B, H, dc, dr, float(scale), float(latent_scale),
                                           float(rope_scale), out.data_ptr(), lse.data_ptr(), _stream_handle(stream))
    if st != KVATTN_OK:
        raise KvattnError(st, "kvattn_mla_decode_fp8_paged")
    return out, lse


def kvattn_mla_rope_append_fp8(q_rope, latent_new, rope_new, positions, latent_cache, rope_cache, latent_scale,
                               rope_scale, rope_base=10000.0, interleaved=False, stream=None):
    """kvattn_mla_rope_append into an E4M3 cache (include/kvattn.h): latent_cache [B, T, c],
    rope_cache [B, T, r] float8_e4m3fn (or uint8 codes)."""
    import torch
    B, H, r = q_rope.shape
    T, c = latent_cache.shape[1], latent_cache.shape[2]
    _check(q_rope, "q_rope", torch.bfloat16)
    _check(latent_new, "latent_new", torch.bfloat16, (B, c))
    _check(rope_new, "rope_new", torch.bfloat16, (B, r))
    _check(positions, "positions", torch.int32, (B,))
    _check_e4m3(latent_cache, "latent_cache", (B, T, c))
    _check_e4m3(rope_cache, "rope_cache", (B, T, r))
    st = lib().kvattn_mla_rope_append_fp8(q_rope.data_ptr(), latent_new.data_ptr(), rope_new.data_ptr(),
                                          positions.data_ptr(), latent_cache.data_ptr(), rope_cache.data_ptr(),
                                          T, B, H, c, r, float(rope_base), int(bool(interleaved)),
                                          float(latent_scale), float(rope_scale), _stream_handle(stream))
    if st != KVATTN_OK:
        raise KvattnError(st, "kvattn_mla_rope_append_fp8")


def kvattn_mla_decode_multi(q_latent, q_rope, latent_cache, rope_cache, seq_lens, scale, latent_scale=None,
                            rope_scale=None, out=None, lse=None, stream=None):
    """Several new tokens per sequence for MLA (include/kvattn.h, kvattn_mla_decode_multi):
    q_latent [B, L, H, 512], q_rope [B, L, H, 64] bf16; caches [B, T, 512] / [B, T, 64] bf16,
    or float8_e4m3fn codes with latent_scale / rope_scale.  Returns (out [B, L, H, 512],
    lse [B, L, H]) fp32."""
    import torch
    B, L, H, dc = q_latent.shape
    dr = q_rope.shape[3]
    T = latent_cache.shape[1]
    e4m3 = latent_cache.dtype != torch.bfloat16
    _check(q_latent, "q_latent", torch.bfloat16)
    _check(q_rope, "q_rope", torch.bfloat16, (B, L, H, dr))
    if e4m3:
        _check_e4m3(latent_cache, "latent_cache", (B, T, dc))
        _check_e4m3(rope_cache, "rope_cache", (B, T, dr))
    else:
        _check(latent_cache, "latent_cache", torch.bfloat16, (B, T, dc))
        _check(rope_cache, "rope_cache", torch.bfloat16, (B, T, dr))
    _check(seq_lens, "seq_lens", torch.int32, (B,))
    if out is None:
        out = torch.empty((B, L, H, dc), dtype=torch.float32, device=q_latent.device)
    if lse is None:
        lse = torch.empty((B, L, H), dtype=torch.float32, device=q_latent.device)
    _check(out, "out", torch.float32, (B, L, H, dc))
    _check(lse, "lse", torch.float32, (B, L, H))
    st = lib().kvattn_mla_decode_multi(q_latent.data_ptr(), q_rope.data_ptr(), latent_cache.data_ptr(),
                                       rope_cache.data_ptr(), seq_lens.data_ptr(), T, B, L, H, dc, dr, float(scale),
                                       int(e4m3), float(latent_scale or 1.0), float(rope_scale or 1.0),
                                       out.data_ptr(), lse.data_ptr(), _stream_handle(stream))
    if st != KVATTN_OK:
        raise KvattnError(st, "kvattn_mla_decode_multi")
    return out, lse


def kvattn_gqa_decode_multi(q, k_cache, v_cache, seq_lens, scale, window=0, out=None, lse=None, stream=None):
    """Multi-token decode (include/kvattn.h, kvattn_gqa_decode_multi): q [B, L, n_q, d]
    bf16, caches [B, n_kv, T, d] bf16 holding the L new tokens at the end of each
    sequence.  Returns (out [B, L, n_q, d] fp32, lse [B, L, n_q] fp32)."""
    import torch
    B, L, n_q, d = q.shape
    n_kv, T = k_cache.shape[1], k_cache.shape[2]
    _check(q, "q", torch.bfloat16)
    _check(k_cache, "k_cache", torch.bfloat16, (B, n_kv, T, d))
    _check(v_cache, "v_cache", torch.bfloat16, (B, n_kv, T, d))
    _check(seq_lens, "seq_lens", torch.int32, (B,))
    if out is None:
        out = torch.empty((B, L, n_q, d), dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty((B, L, n_q), dtype=torch.float32, device=q.device)
    _check(out, "out", torch.float32, (B, L, n_q, d))
    _check(lse, "lse", torch.float32, (B, L, n_q))
    st = lib().kvattn_gqa_decode_multi(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), seq_lens.data_ptr(),
                                       T, B, L, n_q, n_kv, d, float(scale), int(window), out.data_ptr(),
                                       lse.data_ptr(), _stream_handle(stream))
    if st != KVATTN_OK:
        raise KvattnError(st, "kvattn_gqa_decode_multi")
    return out, lse
