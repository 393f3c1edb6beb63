"""kvattn_kernel_launches: the library's own count of the kernels it enqueues.  A decode
call is one kernel when no unit is cut between workers (one worker per unit on small
problems, the MLA kernel's in-kernel merge), two when a combine kernel merges cut units,
and one more for the virtual batch of a multi-token MLA call.  The bench reports
gpu_launches from this count."""
import math

import pytest
import torch

from mla_kv_cache_b200 import binding as kb
from mla_kv_cache_b200 import workloads as wl

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)


def _count(fn):
    n0 = kb.kvattn_kernel_launches()
    fn()
    torch.cuda.synchronize()
    return kb.kvattn_kernel_launches() - n0


def _gqa(cfg):
    x = wl.make_gqa_inputs(cfg, seed=1)
    d = {k: v.cuda() for k, v in x.items()}
    return lambda: kb.kvattn_gqa_decode(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], cfg.scale)


def test_decode_launch_counts():
    kb.kvattn_debug_set_workers(0, 0)
    small = wl.GQAConfig("lc_small", 1, 8, 2, 64, 512, 0.125)               # one worker per unit
    assert _count(_gqa(small)) == 1
    big = wl.GQAConfig("lc_big", 4, 32, 1, 128, 8192, 1.0 / math.sqrt(128.0))  # units cut: combine
    assert _count(_gqa(big)) == 2
    m = wl.MLAConfig("lc_mla", 2, 128, 512, 64, 600, 1.0 / math.sqrt(192.0), seq_lens=(600, 300))
    x = wl.make_mla_inputs(m, seed=2)
    d = {k: v.cuda() for k, v in x.items()}
    assert _count(lambda: kb.kvattn_mla_decode(d["q_latent"], d["q_rope"], d["latent_cache"], d["rope_cache"],
                                               d["seq_lens"], m.scale)) == 1
    ql = torch.randn((2, 2, 128, 512), device="cuda").to(torch.bfloat16)
    qr = torch.randn((2, 2, 128, 64), device="cuda").to(torch.bfloat16)
    assert _count(lambda: kb.kvattn_mla_decode_multi(ql, qr, d["latent_cache"], d["rope_cache"], d["seq_lens"],
                                                     m.scale)) == 2
