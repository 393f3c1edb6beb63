"""fp64 CPU oracle for decode attention.  TEST INFRASTRUCTURE ONLY.

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never links, loads or calls
it, and it shares no code with the library: the two meet only through the seeded
input generators in ``mla_kv_cache_b200/workloads.py``, which hold none of the
method's arithmetic.

The arithmetic lives in ``kvattn_oracle.c`` (plain fp64 loops, three passes).  This
module builds it with gcc, converts bf16 inputs to fp64 (exact), and calls it one
batch element at a time so that a 2 GiB bf16 cache never has to exist in fp64 all
at once.
"""
import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kvattn_oracle.c")
_LOCK = threading.Lock()
_LIBS = {}


def _lib_path(mutant=0, out_dir=None):
    name = "libkvattn_oracle.so" if mutant == 0 else f"libkvattn_oracle_mutant{mutant}.so"
    return os.path.join(out_dir or _HERE, name)


def build(mutant=0, out_dir=None, force=False):
    """Compile the oracle with gcc (OpenMP); returns the shared-library path."""
    path = _lib_path(mutant, out_dir)
    if (not force and os.path.exists(path)
            and os.path.getmtime(path) >= os.path.getmtime(_SRC)):
        return path
    cmd = ["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11",
           f"-DKVO_MUTANT={int(mutant)}", _SRC, "-o", path + ".tmp", "-lm"]
    subprocess.run(cmd, check=True, capture_output=True)
    os.replace(path + ".tmp", path)
    return path


def load(mutant=0, out_dir=None):
    """Load (building first if needed) the oracle library; cached per variant."""
    key = (mutant, out_dir)
    with _LOCK:
        if key in _LIBS:
            return _LIBS[key]
        lib = ctypes.CDLL(build(mutant, out_dir))
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int32)
        ci, cd = ctypes.c_int, ctypes.c_double
        lib.kvo_gqa_decode.argtypes = [dp, dp, dp, ip, ci, ci, ci, ci, ci, cd, dp, dp]
        lib.kvo_gqa_decode.restype = ci
        lib.kvo_mla_decode.argtypes = [dp, dp, dp, dp, ip, ci, ci, ci, ci, ci, cd, dp, dp]
        lib.kvo_mla_decode.restype = ci
        lib.kvo_gqa_decode_multi.argtypes = [dp, dp, dp, ip, ci, ci, ci, ci, ci, ci, cd, ci, dp, dp]
        lib.kvo_gqa_decode_multi.restype = ci
        lib.kvo_rope.argtypes = [dp, ci, ci, ip, cd, ci, dp]
        lib.kvo_rope.restype = ci
        lib.kvo_num_threads.restype = ci
        u8p = ctypes.POINTER(ctypes.c_uint8)
        lib.kvo_e4m3_value.argtypes = [ctypes.c_uint8]
        lib.kvo_e4m3_value.restype = cd
        lib.kvo_e4m3_dequant.argtypes = [u8p, ctypes.c_longlong, cd, dp]
        lib.kvo_e4m3_dequant.restype = ci
        lib.kvo_e4m3_code.argtypes = [ctypes.c_float]
        lib.kvo_e4m3_code.restype = ctypes.c_uint8
        lib.kvo_e4m3_quant.argtypes = [ctypes.POINTER(ctypes.c_float), ctypes.c_longlong, ctypes.c_float, u8p]
        lib.kvo_e4m3_quant.restype = ci
        lib.kvo_mutant.restype = ci
        _LIBS[key] = lib
        return lib


def num_threads():
    """Threads the oracle's parallel regions use (OpenMP)."""
    return int(load().kvo_num_threads())


def _f64(x):
    """Exact conversion of a torch tensor (any float dtype) or array to contiguous fp64."""
    if hasattr(x, "detach"):
        x = x.detach().to("cpu")
        import torch
        return np.ascontiguousarray(x.to(torch.float64).numpy())
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _lens(seq_lens):
    if hasattr(seq_lens, "detach"):
        seq_lens = seq_lens.detach().to("cpu").numpy()
    return np.ascontiguousarray(np.asarray(seq_lens, dtype=np.int32))


def _rows(length, capacity):
    """Cache rows a sequence of this length attends to: the length clamped to
    [0, capacity], as the fp64 core clamps it.  The per-sequence wrappers below convert
    and pass exactly these rows, so a cache position at or past the length is never read."""
    return int(min(max(int(length), 0), int(capacity)))


def gqa_decode_f64(q, k, v, seq_lens, scale, lib=None):
    """GQA/MQA/MHA decode on fp64 arrays.

    q [B, n_q, d], k and v [B, n_kv, T_max, d], seq_lens [B].
    Returns (out [B, n_q, d], lse [B, n_q]) as fp64 numpy arrays.
    """
    lib = lib or load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    lens = _lens(seq_lens)
    B, n_q, d = q.shape
    n_kv, T_max = k.shape[1], k.shape[2]
    assert k.shape == (B, n_kv, T_max, d) and v.shape == k.shape and lens.shape == (B,)
    out = np.zeros((B, n_q, d))
    lse = np.zeros((B, n_q))
    rc = lib.kvo_gqa_decode(_ptr(q, ctypes.c_double), _ptr(k, ctypes.c_double),
                            _ptr(v, ctypes.c_double), _ptr(lens, ctypes.c_int32),
                            B, n_q, n_kv, d, T_max, float(scale),
                            _ptr(out, ctypes.c_double), _ptr(lse, ctypes.c_double))
    if rc != 0:
        raise RuntimeError(f"oracle kvo_gqa_decode failed ({rc})")
    return out, lse


def mla_decode_f64(q_lat, q_rope, lat, rope, seq_lens, scale, lib=None):
    """Absorbed MLA decode on fp64 arrays.

    q_lat [B, H, d_c], q_rope [B, H, d_r], lat [B, T_max, d_c], rope [B, T_max, d_r]
    (d_r may be 0).  Returns (out [B, H, d_c], lse [B, H]).
    """
    lib = lib or load()
    q_lat, q_rope, lat, rope = _f64(q_lat), _f64(q_rope), _f64(lat), _f64(rope)
    lens = _lens(seq_lens)
    B, H, d_c = q_lat.shape
    d_r = q_rope.shape[2]
    T_max = lat.shape[1]
    assert lat.shape == (B, T_max, d_c) and rope.shape == (B, T_max, d_r)
    if d_r == 0:  # keep valid (never dereferenced) pointers for empty arrays
        q_rope = np.zeros((1,))
        rope = np.zeros((1,))
    out = np.zeros((B, H, d_c))
    lse = np.zeros((B, H))
    rc = lib.kvo_mla_decode(_ptr(q_lat, ctypes.c_double), _ptr(q_rope, ctypes.c_double),
                            _ptr(lat, ctypes.c_double), _ptr(rope, ctypes.c_double),
                            _ptr(lens, ctypes.c_int32), B, H, d_c, d_r, T_max,
                            float(scale), _ptr(out, ctypes.c_double),
                            _ptr(lse, ctypes.c_double))
    if rc != 0:
        raise RuntimeError(f"oracle kvo_mla_decode failed ({rc})")
    return out, lse


def gqa_decode(q, k_cache, v_cache, seq_lens, scale, batch_ids=None, lib=None):
    """Oracle on bf16 (torch) inputs, one batch element at a time.

    Only the first seq_lens[b] cache rows of each sequence are converted and read.
    batch_ids selects a subset of sequences (all by default); results are returned
    in that order as (out [len(ids), n_q, d], lse [len(ids), n_q]) fp64 arrays.
    """
    lens = _lens(seq_lens)
    T_max = k_cache.shape[2]
    ids = range(q.shape[0]) if batch_ids is None else batch_ids
    outs, lses = [], []
    for b in ids:
        T = _rows(lens[b], T_max)
        o, l = gqa_decode_f64(q[b:b + 1], k_cache[b:b + 1, :, :T], v_cache[b:b + 1, :, :T],
                              np.array([T], dtype=np.int32), scale, lib=lib)
        outs.append(o[0])
        lses.append(l[0])
    return np.stack(outs), np.stack(lses)


def mla_decode(q_latent, q_rope, latent_cache, rope_cache, seq_lens, scale, batch_ids=None,
               lib=None):
    """Absorbed-MLA oracle on bf16 (torch) inputs, one batch element at a time."""
    lens = _lens(seq_lens)
    T_max = latent_cache.shape[1]
    ids = range(q_latent.shape[0]) if batch_ids is None else batch_ids
    outs, lses = [], []
    for b in ids:
        T = _rows(lens[b], T_max)
        o, l = mla_decode_f64(q_latent[b:b + 1], q_rope[b:b + 1], latent_cache[b:b + 1, :T],
                              rope_cache[b:b + 1, :T], np.array([T], dtype=np.int32), scale,
                              lib=lib)
        outs.append(o[0])
        lses.append(l[0])
    return np.stack(outs), np.stack(lses)


def _causal_rows(length, q_len, i, capacity):
    """Cache rows query i (0-based, oldest first) of q_len new tokens sees: the tokens at
    positions <= len - q_len + i ("Attention variants: MQA, GQA, and MLA", section
    "Implementation, twice": no query sees a later token)."""
    return max(_rows(length, capacity) - q_len + 1 + i, 0)


def mla_decode_multi(q_latent, q_rope, latent_cache, rope_cache, seq_lens, scale, lib=None):
    """Absorbed MLA with q_len new tokens per sequence under the causal mask.  q_latent
    [B, L, H, d_c], q_rope [B, L, H, d_r] bf16; caches [B, T_max, d_c], [B, T_max, d_r]
    (bf16, or fp64 arrays already dequantised).  Returns (out [B, L, H, d_c], lse [B, L, H]);
    a query that sees no token gets out 0, lse -inf."""
    lens = _lens(seq_lens)
    B, L, H, d_c = q_latent.shape
    T_max = latent_cache.shape[1]
    out = np.zeros((B, L, H, d_c))
    lse = np.zeros((B, L, H))
    for b in range(B):
        for i in range(L):
            n = _causal_rows(lens[b], L, i, T_max)
            o, l = mla_decode_f64(q_latent[b:b + 1, i], q_rope[b:b + 1, i], latent_cache[b:b + 1, :max(n, 1)],
                                  rope_cache[b:b + 1, :max(n, 1)], np.array([n], dtype=np.int32), scale, lib=lib)
            out[b, i], lse[b, i] = o[0], l[0]
    return out, lse


def rope_f64(x, positions, base, interleaved, lib=None):
    """Rotary embedding of the last axis of x (fp64 result, same shape).  positions
    holds one position per vector, broadcast over x's leading axes (e.g. [B] for x of
    shape [B, heads, d]: every head of sequence b at positions[b])."""
    lib = lib or load()
    xx = _f64(x)
    d = xx.shape[-1]
    lead = xx.shape[:-1]
    pos = np.ascontiguousarray(np.broadcast_to(
        np.asarray(positions, dtype=np.int32).reshape(
            np.asarray(positions).shape + (1,) * (len(lead) - np.asarray(positions).ndim)),
        lead).reshape(-1))
    flat = xx.reshape(-1, d)
    out = np.empty_like(flat)
    st = lib.kvo_rope(_ptr(flat, ctypes.c_double), flat.shape[0], d, _ptr(pos, ctypes.c_int32),
                      float(base), int(bool(interleaved)), _ptr(out, ctypes.c_double))
    if st != 0:
        raise ValueError("kvo_rope: bad arguments")
    return out.reshape(xx.shape)


def gqa_decode_multi_f64(q, k, v, seq_lens, scale, window=0, lib=None):
    """Multi-token decode on fp64 arrays: q [B, L, n_q, d], k / v [B, n_kv, T, d];
    returns (out [B, L, n_q, d], lse [B, L, n_q])."""
    lib = lib or load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, L, n_q, d = q.shape
    n_kv, T = k.shape[1], k.shape[2]
    lens = np.ascontiguousarray(np.asarray(seq_lens, dtype=np.int32))
    out = np.zeros((B, L, n_q, d))
    lse = np.zeros((B, L, n_q))
    st = lib.kvo_gqa_decode_multi(_ptr(q, ctypes.c_double), _ptr(k, ctypes.c_double), _ptr(v, ctypes.c_double),
                                  _ptr(lens, ctypes.c_int32), B, L, n_q, n_kv, d, T, float(scale), int(window),
                                  _ptr(out, ctypes.c_double), _ptr(lse, ctypes.c_double))
    if st != 0:
        raise RuntimeError(f"kvo_gqa_decode_multi failed ({st})")
    return out, lse


def gqa_decode_multi(q, k_cache, v_cache, seq_lens, scale, window=0, lib=None):
    """Multi-token decode on the bf16 (or any float) tensors, one sequence at a time so
    only the touched rows are converted to fp64."""
    B = q.shape[0]
    lens = _lens(seq_lens)
    outs, lses = [], []
    for b in range(B):
        T = _rows(lens[b], k_cache.shape[2])
        n = max(T, 1)
        o, l = gqa_decode_multi_f64(q[b:b + 1], k_cache[b:b + 1, :, :n], v_cache[b:b + 1, :, :n],
                                    [T], scale, window, lib=lib)
        outs.append(o[0])
        lses.append(l[0])
    return np.stack(outs), np.stack(lses)


def _codes(x):
    """E4M3 codes as a contiguous uint8 array (torch float8_e4m3fn / uint8 tensor, or array)."""
    if hasattr(x, "detach"):
        import torch
        x = x.detach().to("cpu")
        if x.dtype != torch.uint8:
            x = x.view(torch.uint8)
        x = x.numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.uint8))


def e4m3_value(code, lib=None):
    """Value of one E4M3 code (fp64)."""
    return float((lib or load()).kvo_e4m3_value(int(code) & 0xFF))


def e4m3_dequant(codes, scale, lib=None):
    """Dequantised cache: value(code) * scale, fp64, same shape."""
    lib = lib or load()
    c = _codes(codes)
    out = np.empty(c.shape, dtype=np.float64)
    st = lib.kvo_e4m3_dequant(_ptr(c, ctypes.c_uint8), c.size, float(scale), _ptr(out, ctypes.c_double))
    if st != 0:
        raise ValueError("kvo_e4m3_dequant: bad arguments")
    return out


def e4m3_quant(x, scale, lib=None):
    """E4M3 codes of float32(x) / float32(scale) (ties to even, saturated), uint8."""
    lib = lib or load()
    xf = x.detach().to("cpu").float().numpy() if hasattr(x, "detach") else np.asarray(x, dtype=np.float32)
    xf = np.ascontiguousarray(xf, dtype=np.float32)
    out = np.empty(xf.shape, dtype=np.uint8)
    st = lib.kvo_e4m3_quant(_ptr(xf, ctypes.c_float), xf.size, float(np.float32(scale)), _ptr(out, ctypes.c_uint8))
    if st != 0:
        raise ValueError("kvo_e4m3_quant: bad arguments")
    return out


def mla_decode_fp8(q_latent, q_rope, latent_codes, rope_codes, seq_lens, scale, latent_scale, rope_scale,
                   batch_ids=None, lib=None):
    """Absorbed MLA over an E4M3 latent cache: attention on the dequantised latents
    value(code) * latent_scale (keys' latent part and values alike) and RoPE keys
    value(code) * rope_scale.  q_latent [B, H, d_c], q_rope [B, H, d_r] bf16; caches
    [B, T_max, d_c] and [B, T_max, d_r] of codes; only the first seq_lens[b] rows of each
    sequence are read.  Returns (out [B, H, d_c], lse [B, H])."""
    lib = lib or load()
    lens = _lens(seq_lens)
    lc, rc = _codes(latent_codes), _codes(rope_codes)
    T_max = lc.shape[1]
    ids = range(q_latent.shape[0]) if batch_ids is None else batch_ids
    outs, lses = [], []
    for b in ids:
        T = _rows(lens[b], T_max)
        n = max(T, 1)
        lat = e4m3_dequant(lc[b:b + 1, :n], latent_scale, lib=lib)
        rope = e4m3_dequant(rc[b:b + 1, :n], rope_scale, lib=lib)
        o, l = mla_decode_f64(q_latent[b:b + 1], q_rope[b:b + 1], lat, rope, np.array([T], dtype=np.int32),
                              scale, lib=lib)
        outs.append(o[0])
        lses.append(l[0])
    return np.stack(outs), np.stack(lses)


def gqa_decode_fp8(q, k_codes, v_codes, seq_lens, scale, k_scale, v_scale, window=0, lib=None):
    """Decode over an E4M3 cache: attention on the dequantised keys value(k) * k_scale and
    values value(v) * v_scale.  q [B, n_q, d] (single token: returns out [B, n_q, d],
    lse [B, n_q]) or [B, L, n_q, d] (L new tokens, causal, optional window: returns
    [B, L, n_q, d], [B, L, n_q]).  Caches [B, n_kv, T_max, d] of codes; only the first
    seq_lens[b] rows of each sequence are read."""
    lib = lib or load()
    lens = _lens(seq_lens)
    kc, vc = _codes(k_codes), _codes(v_codes)
    T_max = kc.shape[2]
    multi = len(q.shape) == 4
    outs, lses = [], []
    for b in range(q.shape[0]):
        T = _rows(lens[b], T_max)
        n = max(T, 1)
        kb = e4m3_dequant(kc[b:b + 1, :, :n], k_scale, lib=lib)
        vb = e4m3_dequant(vc[b:b + 1, :, :n], v_scale, lib=lib)
        if multi:
            o, l = gqa_decode_multi_f64(q[b:b + 1], kb, vb, [T], scale, window, lib=lib)
        else:
            o, l = gqa_decode_f64(q[b:b + 1], kb, vb, np.array([T], dtype=np.int32), scale, lib=lib)
        outs.append(o[0])
        lses.append(l[0])
    return np.stack(outs), np.stack(lses)
