"""A bounded wait that runs out: the kernels' wait (the same code, its limit cut to ~1 ms)
on a barrier nothing completes gives up, reports through the device flags and returns;
the context stays usable and the next decode still matches the oracle.  No fault, trap
or hang is involved: the wait ends by its own limit."""
import math
import time

import pytest
import torch

import oracle
from mla_kv_cache_b200 import binding as kb
from mla_kv_cache_b200 import workloads as wl
from tests.parity import assert_close

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)


def test_expired_wait_sets_flag_and_context_survives():
    kb.kvattn_clear_device_flags()
    t0 = time.perf_counter()
    kb.kvattn_debug_wait_probe(1000)
    torch.cuda.synchronize()
    assert time.perf_counter() - t0 < 5.0
    assert kb.kvattn_read_device_flags() & 1 == 1, "the expired wait must set bit 0"
    kb.kvattn_clear_device_flags()
    assert kb.kvattn_read_device_flags() == 0
    # the same context runs a decode and gets the oracle's result
    cfg = wl.GQAConfig("after_probe", 2, 8, 2, 128, 300, 1.0 / math.sqrt(128.0), seq_lens=(300, 77))
    x = wl.make_gqa_inputs(cfg, seed=3)
    out, lse = kb.kvattn_gqa_decode(x["q"].cuda(), x["k_cache"].cuda(), x["v_cache"].cuda(),
                                    x["seq_lens"].cuda(), cfg.scale)
    torch.cuda.synchronize()
    ro, rl = oracle.gqa_decode(x["q"], x["k_cache"], x["v_cache"], x["seq_lens"], cfg.scale)
    assert_close(out.cpu().numpy(), ro, "out after probe")
    assert_close(lse.cpu().numpy(), rl, "lse after probe")
    assert kb.kvattn_read_device_flags() == 0


def test_probe_rejects_bad_limits():
    for bad in (0, -5, 2_000_000):
        with pytest.raises(kb.KvattnError):
            kb.kvattn_debug_wait_probe(bad)
