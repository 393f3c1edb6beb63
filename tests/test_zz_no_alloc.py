"""kvattn_gqa_decode_noalloc: the decode entry point that allocates nothing.

It is meant for callers that cannot let a library call cudaMalloc: serving engines
that reserve nearly all device memory for their own KV-cache pool, and loops that
cannot afford cudaMalloc's implicit synchronisation.  Its scratch is a fixed array
inside the library shared by every call.

The test calls it through the C ABI (ctypes, no Python wrapper) twice in a row on
different workloads and checks both results against the fp64 oracle and against
kvattn_gqa_decode's at the library's tolerance; the second call runs on a scratch array
that still holds the first call's contents.  It also checks that a plan too large for the array is refused
with a clear error.  This file is collected last on purpose, and it must pass both on
its own in a fresh process (the first call on the device does the one-time set-up) and
after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from mla_kv_cache_b200 import binding as kb
from mla_kv_cache_b200 import workloads as wl
from tests.parity import assert_close

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)


def _c_call(fn_name, d, cfg, out, lse, stream):
    fn = getattr(kb.lib(), fn_name)
    B, n_q, hd = d["q"].shape
    n_kv, T = d["k_cache"].shape[1], d["k_cache"].shape[2]
    return fn(d["q"].data_ptr(), d["k_cache"].data_ptr(), d["v_cache"].data_ptr(),
              d["seq_lens"].data_ptr(), T, B, n_q, n_kv, hd, ctypes.c_float(cfg.scale),
              out.data_ptr(), lse.data_ptr(), ctypes.c_void_p(stream.cuda_stream))


def _inputs(cfg, seed):
    x = wl.make_gqa_inputs(cfg, seed=seed, poison_tail=True)
    d = {k: v.cuda() for k, v in x.items()}
    B, n_q, hd = d["q"].shape
    nan = float("nan")
    bufs = {"out": torch.full((B, n_q, hd), nan, dtype=torch.float32, device="cuda"),
            "lse": torch.full((B, n_q), nan, dtype=torch.float32, device="cuda"),
            "host": x}
    return d, bufs


def test_noalloc_matches_allocating_entry_point_twice():
    kb.kvattn_debug_set_workers(0, 0)
    kb.kvattn_clear_device_flags()
    stream = torch.cuda.current_stream()
    # first call: ragged GQA (group 8) with cut units, so the scratch holds partials
    first = wl.GQAConfig("noalloc_gqa", 4, 64, 8, 128, 3000, 1.0 / np.sqrt(128.0),
                         seq_lens=(3000, 17, 0, 2048))
    # second call: another shape (MQA, head_dim 64) on the scratch the first one left
    second = wl.GQAConfig("noalloc_mqa", 3, 32, 1, 64, 5000, 0.125, seq_lens=(5000, 4999, 64))
    cases = []
    for cfg, seed in ((first, 21), (second, 22)):
        d, ref = _inputs(cfg, seed)
        _, got = _inputs(cfg, seed)
        assert _c_call("kvattn_gqa_decode", d, cfg, ref["out"], ref["lse"], stream) == kb.KVATTN_OK
        cases.append((cfg, d, ref, got))
    torch.cuda.synchronize()
    # the two no-allocation calls, back to back on the same stream
    for cfg, d, _, got in cases:
        assert _c_call("kvattn_gqa_decode_noalloc", d, cfg, got["out"], got["lse"], stream) == kb.KVATTN_OK
    torch.cuda.synchronize()
    for cfg, _, ref, got in cases:
        x = got["host"]
        ro, rl = oracle.gqa_decode(x["q"], x["k_cache"], x["v_cache"], x["seq_lens"], cfg.scale)
        assert_close(got["out"].cpu().numpy(), ro, f"{cfg.name} out vs oracle")
        assert_close(got["lse"].cpu().numpy(), rl, f"{cfg.name} lse vs oracle")
        assert_close(got["out"].cpu().numpy(), ref["out"].cpu().numpy().astype(np.float64),
                     f"{cfg.name} out")
        assert_close(got["lse"].cpu().numpy(), ref["lse"].cpu().numpy().astype(np.float64),
                     f"{cfg.name} lse")
    assert kb.kvattn_read_device_flags() == 0


def test_noalloc_refuses_a_plan_larger_than_its_scratch():
    cfg = wl.GQAConfig("noalloc_big", 2, 32, 1, 128, 4096, 1.0 / np.sqrt(128.0))
    x = wl.make_gqa_inputs(cfg, seed=23)
    d = {k: v.cuda() for k, v in x.items()}
    out = torch.empty((2, 32, 128), dtype=torch.float32, device="cuda")
    lse = torch.empty((2, 32), dtype=torch.float32, device="cuda")
    try:
        # 2000 workers x 2 slots x 32 heads x 129 floats > the 6 MiB array
        kb.kvattn_debug_set_workers(2000, 1)
        st = _c_call("kvattn_gqa_decode_noalloc", d, cfg, out, lse, torch.cuda.current_stream())
    finally:
        kb.kvattn_debug_set_workers(0, 0)
    assert st == kb.KVATTN_ERR_UNSUPPORTED
    assert "static scratch" in kb.kvattn_last_error_detail()
