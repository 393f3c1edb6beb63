"""GPU parity of kvattn_rope_append / kvattn_mla_rope_append against the fp64 oracle.

The rotated query and key are compared with the oracle's fp64 rotation rounded once to
bf16: at most one bf16 unit in the last place apart (the kernel turns the pair in fp32,
the oracle in fp64, so a value next to a rounding boundary may round the other way).
Copied values (V, the MLA latent) and every cache row other than the new token's must be
bit-exact.  Then an append followed by a decode is compared with the oracle's decode of
the oracle-appended cache at the library tolerance.
"""
import math

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


@pytest.fixture(autouse=True)
def _flags():
    kb.kvattn_clear_device_flags()
    yield
    assert kb.kvattn_read_device_flags() == 0


def _bf16(x64):
    return torch.from_numpy(np.asarray(x64, dtype=np.float32)).to(torch.bfloat16)


def assert_within_one_ulp(gpu, ref_bf16, what):
    """bf16 tensors equal up to one unit in the last place (same sign)."""
    a = gpu.cpu().view(torch.int16).to(torch.int32)
    b = ref_bf16.view(torch.int16).to(torch.int32)
    diff = (a - b).abs()
    exact = (diff == 0).float().mean().item()
    assert int(diff.max()) <= 1, f"{what}: {int((diff > 1).sum())} values more than 1 ulp apart"
    assert exact > 0.97, f"{what}: only {exact:.3f} of the values bit-exact"


def _rand(shape, g, scale=1.0):
    return (torch.randn(shape, generator=g) * scale).to(torch.bfloat16)


@pytest.mark.parametrize("interleaved", [0, 1], ids=["halves", "interleaved"])
@pytest.mark.parametrize("d,n_q,n_kv", [(128, 32, 8), (64, 8, 2), (128, 4, 4)])
def test_rope_append_gqa(d, n_q, n_kv, interleaved):
    g = torch.Generator().manual_seed(7)
    B, T = 6, 32800
    q = _rand((B, n_q, d), g)
    k_new = _rand((B, n_kv, d), g)
    v_new = _rand((B, n_kv, d), g)
    pos = torch.tensor([0, 1, 4097, 32767, T, -1], dtype=torch.int32)   # the last two: outside the cache
    kc = _rand((B, n_kv, T, d), g)
    vc = _rand((B, n_kv, T, d), g)
    dq, dk, dv, dkc, dvc, dpos = (t.cuda() for t in (q, k_new, v_new, kc, vc, pos))
    kb.kvattn_rope_append(dq, dk, dv, dpos, dkc, dvc, rope_base=10000.0, interleaved=interleaved)
    torch.cuda.synchronize()
    q_ref = _bf16(oracle.rope_f64(q, pos.numpy(), 10000.0, interleaved))
    k_ref = _bf16(oracle.rope_f64(k_new, pos.numpy(), 10000.0, interleaved))
    assert_within_one_ulp(dq, q_ref, "q")
    kc_gpu, vc_gpu = dkc.cpu(), dvc.cpu()
    for b in range(B):
        p = int(pos[b])
        kc_exp, vc_exp = kc[b].clone(), vc[b].clone()
        if 0 <= p < T:
            assert_within_one_ulp(kc_gpu[b, :, p], k_ref[b], f"k row of sequence {b}")
            assert torch.equal(vc_gpu[b, :, p], v_new[b]), f"v row of sequence {b}"
            kc_exp[:, p] = kc_gpu[b, :, p]
            vc_exp[:, p] = v_new[b]
        assert torch.equal(kc_gpu[b], kc_exp), f"other K rows of sequence {b} changed"
        assert torch.equal(vc_gpu[b], vc_exp), f"other V rows of sequence {b} changed"


@pytest.mark.parametrize("interleaved", [0, 1], ids=["halves", "interleaved"])
def test_rope_append_mla(interleaved):
    g = torch.Generator().manual_seed(8)
    B, H, T, dc, dr = 4, 128, 5000, 512, 64
    q_rope = _rand((B, H, dr), g)
    lat_new = _rand((B, dc), g)
    rope_new = _rand((B, dr), g)
    pos = torch.tensor([0, 17, 4999, 5000], dtype=torch.int32)
    lat = _rand((B, T, dc), g)
    rope = _rand((B, T, dr), g)
    dq, dl, dr_, dlat, drope, dpos = (t.cuda() for t in (q_rope, lat_new, rope_new, lat, rope, pos))
    kb.kvattn_mla_rope_append(dq, dl, dr_, dpos, dlat, drope, rope_base=10000.0, interleaved=interleaved)
    torch.cuda.synchronize()
    assert_within_one_ulp(dq, _bf16(oracle.rope_f64(q_rope, pos.numpy(), 10000.0, interleaved)), "q_rope")
    r_ref = _bf16(oracle.rope_f64(rope_new, pos.numpy(), 10000.0, interleaved))
    lat_gpu, rope_gpu = dlat.cpu(), drope.cpu()
    for b in range(B):
        p = int(pos[b])
        lat_exp, rope_exp = lat[b].clone(), rope[b].clone()
        if 0 <= p < T:
            assert_within_one_ulp(rope_gpu[b, p], r_ref[b], f"rope row {b}")
            assert torch.equal(lat_gpu[b, p], lat_new[b]), f"latent row {b}"
            lat_exp[p] = lat_new[b]
            rope_exp[p] = rope_gpu[b, p]
        assert torch.equal(lat_gpu[b], lat_exp) and torch.equal(rope_gpu[b], rope_exp), b


def test_append_then_decode_matches_oracle():
    """One decode step end to end: rotate + append the new token, then attend over the
    cache including it (seq_lens = positions + 1), against the oracle doing the same in
    fp64 (its rotation rounded to bf16 like the stored cache)."""
    cfg = wl.GQAConfig("step", 4, 32, 8, 128, 3000, 1.0 / math.sqrt(128.0), seq_lens=(2999, 1, 1500, 64))
    x = wl.make_gqa_inputs(cfg, seed=21)
    g = torch.Generator().manual_seed(22)
    k_new = _rand((cfg.batch, cfg.n_kv_heads, cfg.head_dim), g)
    v_new = _rand((cfg.batch, cfg.n_kv_heads, cfg.head_dim), g)
    pos = (x["seq_lens"] - 1).to(torch.int32)           # the new token is the last cached one
    d = {k: v.cuda() for k, v in x.items()}
    dq = d["q"].clone()
    kb.kvattn_rope_append(dq, k_new.cuda(), v_new.cuda(), pos.cuda(), d["k_cache"], d["v_cache"])
    out, lse = kb.kvattn_gqa_decode(dq, d["k_cache"], d["v_cache"], d["seq_lens"], cfg.scale)
    torch.cuda.synchronize()
    q_ref = _bf16(oracle.rope_f64(x["q"], pos.numpy(), 10000.0, 0))
    k_ref = _bf16(oracle.rope_f64(k_new, pos.numpy(), 10000.0, 0))
    kc, vc = x["k_cache"].clone(), x["v_cache"].clone()
    for b in range(cfg.batch):
        kc[b, :, int(pos[b])] = k_ref[b]
        vc[b, :, int(pos[b])] = v_new[b]
    ro, rl = oracle.gqa_decode(q_ref, kc, vc, x["seq_lens"], cfg.scale)
    assert_close(out.cpu().numpy(), ro, "step out")
    assert_close(lse.cpu().numpy(), rl, "step lse")
