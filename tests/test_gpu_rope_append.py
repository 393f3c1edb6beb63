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


def _signed_code(c):
    """E4M3 codes as signed integers ordered like their values (sign-magnitude -> +-mag)."""
    c = c.to(torch.int32)
    mag = c & 0x7F
    return torch.where((c & 0x80) != 0, -mag, mag)


@pytest.mark.parametrize("interleaved", [0, 1], ids=["halves", "interleaved"])
def test_rope_append_fp8(interleaved):
    """E4M3 cache: the value's codes are bit-exact against the oracle's encoder (the same
    fp32 quotient, ties to even); the key's are within one code step of the oracle's
    encoding of its fp64 rotation rounded to fp32 (the kernel turns the pair in fp32);
    every other cache row is unchanged."""
    g = torch.Generator().manual_seed(11)
    B, n_q, n_kv, d, T = 5, 32, 8, 128, 3000
    q = _rand((B, n_q, d), g)
    k_new = _rand((B, n_kv, d), g, 3.0)
    v_new = _rand((B, n_kv, d), g, 3.0)
    pos = torch.tensor([0, 2999, 1234, 3000, -5], dtype=torch.int32)
    ks, vs = 0.0125, 0.00875
    kc = torch.randint(0, 256, (B, n_kv, T, d), generator=g, dtype=torch.uint8)
    vc = torch.randint(0, 256, (B, n_kv, T, d), generator=g, dtype=torch.uint8)
    dq, dkc, dvc = q.cuda(), kc.cuda(), vc.cuda()
    kb.kvattn_rope_append_fp8(dq, k_new.cuda(), v_new.cuda(), pos.cuda(), dkc, dvc, ks, vs, rope_base=10000.0,
                              interleaved=interleaved)
    torch.cuda.synchronize()
    assert_within_one_ulp(dq, _bf16(oracle.rope_f64(q, pos.numpy(), 10000.0, interleaved)), "q")
    k_rot = np.asarray(oracle.rope_f64(k_new, pos.numpy(), 10000.0, interleaved), dtype=np.float32)
    k_codes = torch.from_numpy(oracle.e4m3_quant(k_rot, ks))
    v_codes = torch.from_numpy(oracle.e4m3_quant(v_new.float().numpy(), vs))
    kg, vg = dkc.cpu(), dvc.cpu()
    for b in range(B):
        p = int(pos[b])
        ke, ve = kc[b].clone(), vc[b].clone()
        if 0 <= p < T:
            diff = (_signed_code(kg[b, :, p]) - _signed_code(k_codes[b])).abs()
            assert int(diff.max()) <= 1, f"key codes of sequence {b} more than one step apart"
            assert (diff == 0).float().mean().item() > 0.97, f"key codes of sequence {b}"
            assert torch.equal(vg[b, :, p], v_codes[b]), f"value codes of sequence {b}"
            ke[:, p] = kg[b, :, p]
            ve[:, p] = v_codes[b]
        assert torch.equal(kg[b], ke) and torch.equal(vg[b], ve), f"other rows of sequence {b} changed"


def test_append_fp8_then_decode_matches_oracle():
    """One decode step into an E4M3 cache end to end: rotate + quantise-append, then the
    fp8 decode, against the oracle appending its own codes and attending in fp64."""
    cfg = wl.GQAConfig("step8", 4, 32, 8, 128, 3000, 1.0 / math.sqrt(128.0), seq_lens=(2999, 1, 1500, 64))
    x = wl.make_gqa_inputs_fp8(cfg, seed=23)
    g = torch.Generator().manual_seed(24)
    k_new = _rand((cfg.batch, cfg.n_kv_heads, cfg.head_dim), g)
    v_new = _rand((cfg.batch, cfg.n_kv_heads, cfg.head_dim), g)
    pos = (x["seq_lens"] - 1).to(torch.int32)
    dq, dkc, dvc = x["q"].cuda(), x["k_cache"].cuda(), x["v_cache"].cuda()
    kb.kvattn_rope_append_fp8(dq, k_new.cuda(), v_new.cuda(), pos.cuda(), dkc, dvc, x["k_scale"], x["v_scale"])
    out, lse = kb.kvattn_gqa_decode_fp8(dq, dkc, dvc, x["seq_lens"].cuda(), cfg.scale, x["k_scale"], x["v_scale"])
    torch.cuda.synchronize()
    q_ref = _bf16(oracle.rope_f64(x["q"], pos.numpy(), 10000.0, 0))
    k_rot = np.asarray(oracle.rope_f64(k_new, pos.numpy(), 10000.0, 0), dtype=np.float32)
    k_codes = torch.from_numpy(oracle.e4m3_quant(k_rot, x["k_scale"]))
    v_codes = torch.from_numpy(oracle.e4m3_quant(v_new.float().numpy(), x["v_scale"]))
    kc, vc = x["k_cache"].view(torch.uint8).clone(), x["v_cache"].view(torch.uint8).clone()
    for b in range(cfg.batch):
        kc[b, :, int(pos[b])] = k_codes[b]
        vc[b, :, int(pos[b])] = v_codes[b]
    ro, rl = oracle.gqa_decode_fp8(q_ref, kc, vc, x["seq_lens"], cfg.scale, x["k_scale"], x["v_scale"])
    assert_close(out.cpu().numpy(), ro, "fp8 step out")
    assert_close(lse.cpu().numpy(), rl, "fp8 step lse")
