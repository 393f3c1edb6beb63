"""GPU parity of kvattn_mla_decode_fp8 (E4M3 latent + RoPE cache, tcgen05 pair kernel
with kind::f8f6f4 MMAs) against the fp64 oracle on the dequantised cache.

The caches hold E4M3 codes with one scale per tensor (scale = max|x| / 448 of the seeded
bf16 draw); rows past every sequence's length hold the NaN code, so a read of one shows.
The kernel feeds the codes to the tensor cores as they are, and each head's query and the
softmax weights as an E4M3 high part plus remainder, so the library tolerance
|gpu - oracle| <= 2e-3 (1 + |oracle|) applies unchanged.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from mla_kv_cache_b200 import binding as kb
from mla_kv_cache_b200 import workloads as wl
from tests.parity import assert_close
from tests.test_gpu_paged import paginate

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

SCALE = 1.0 / math.sqrt(192.0)


@pytest.fixture(autouse=True)
def _knobs():
    kb.kvattn_debug_set_workers(0, 0)
    kb.kvattn_clear_device_flags()
    yield
    kb.kvattn_debug_set_workers(0, 0)
    assert kb.kvattn_read_device_flags() == 0, "a bounded wait ran out on the device"


def mla8(name, B, H, T, lens):
    return wl.MLAConfig(name, B, H, 512, 64, T, SCALE, seq_lens=tuple(lens))


def run_case(cfg, seed=0, q_gain=1.0, x=None):
    x = wl.make_mla_inputs_fp8(cfg, seed=seed, poison_tail=True) if x is None else x
    if q_gain != 1.0:  # a power of two keeps the bf16 values exact
        x["q_latent"] = (x["q_latent"].float() * q_gain).to(torch.bfloat16)
        x["q_rope"] = (x["q_rope"].float() * q_gain).to(torch.bfloat16)
    out, lse = kb.kvattn_mla_decode_fp8(x["q_latent"].cuda(), x["q_rope"].cuda(), x["latent_cache"].cuda(),
                                        x["rope_cache"].cuda(), x["seq_lens"].cuda(), cfg.scale,
                                        x["latent_scale"], x["rope_scale"])
    torch.cuda.synchronize()
    ro, rl = oracle.mla_decode_fp8(x["q_latent"], x["q_rope"], x["latent_cache"], x["rope_cache"], x["seq_lens"],
                                   cfg.scale, x["latent_scale"], x["rope_scale"])
    assert_close(out.cpu().numpy(), ro, f"{cfg.name} out")
    assert_close(lse.cpu().numpy(), rl, f"{cfg.name} lse")
    return x


@pytest.mark.parametrize("T", [1, 63, 64, 65, 128, 129, 1000])
def test_lengths(T):
    run_case(mla8(f"T{T}", 2, 128, T, [T, max(T // 3, 1)]))


@pytest.mark.parametrize("H", [1, 16, 100, 128])
def test_head_counts(H):
    run_case(mla8(f"H{H}", 3, H, 300, [300, 129, 5]))


def test_ragged_with_empty_sequences():
    run_case(mla8("ragged", 6, 128, 700, [0, 1, 64, 65, 700, 0]))


def test_sharp_softmax_rescales():
    """Queries times 4: the running max moves by more than 2^2 between tiles many times
    (the E4M3 weights' rescale threshold), rescaling the TMEM accumulator."""
    run_case(mla8("sharp", 2, 128, 1500, [1500, 400]), q_gain=4.0)


def test_query_scales_per_head():
    """Heads whose queries differ by powers of two up to 2^12 in magnitude: each head's
    query is scaled into E4M3's range on its own."""
    cfg = mla8("qscale", 2, 128, 600, [600, 333])
    x = wl.make_mla_inputs_fp8(cfg, seed=5, poison_tail=True)
    gain = (2.0 ** (torch.arange(128) % 13 - 6)).reshape(1, 128, 1)
    x["q_latent"] = (x["q_latent"].float() * gain).to(torch.bfloat16)
    x["q_rope"] = (x["q_rope"].float() * gain).to(torch.bfloat16)
    run_case(cfg, x=x)


def test_rope_scale_differs_from_latent_scale():
    """RoPE codes quantised with a scale 64x the latent's: the RoPE part of the query is
    weighted by the ratio of the two scales."""
    cfg = mla8("ratio", 2, 128, 500, [500, 77])
    x = wl.make_mla_inputs_fp8(cfg, seed=6, poison_tail=True)
    x["rope_scale"] = x["rope_scale"] * 64.0
    x["q_rope"] = (x["q_rope"].float() / 64.0).to(torch.bfloat16)
    run_case(cfg, x=x)


@pytest.mark.parametrize("workers,min_tiles", [(1, 1), (2, 1), (3, 1), (7, 1), (40, 1)])
def test_forced_splits(workers, min_tiles):
    kb.kvattn_debug_set_workers(workers, min_tiles)
    run_case(mla8("split", 4, 128, 2000, [2000, 1, 0, 777]))


def test_many_short_ragged_sequences():
    """300 sequences of 0-400 tokens over the E4M3 cache: several pieces per worker (each
    with its own query split) and the merges of the cut sequences."""
    lens = np.random.default_rng(33).integers(0, 401, size=300).tolist()
    run_case(mla8("many8", 300, 128, 400, lens))


def test_workload_full_size():
    """The DeepSeek-shaped workload (batch 32, 128 heads, context 4096) with its cache in
    E4M3, every sequence, in the bench's launch configuration."""
    run_case(wl.CONFIGS["mla_b32_h128_c512_r64_t4096"])


@pytest.mark.parametrize("page_size", [64, 256])
def test_paged(page_size):
    cfg = mla8("paged8", 4, 128, 1024, [1024, 1, 600, 0])
    x = wl.make_mla_inputs_fp8(cfg, seed=9, poison_tail=True)
    lens = x["seq_lens"].tolist()
    lp, table = paginate(x["latent_cache"], lens, page_size, 1, seed=3)
    rp, table2 = paginate(x["rope_cache"], lens, page_size, 1, seed=3)
    assert torch.equal(table, table2)
    out, lse = kb.kvattn_mla_decode_fp8_paged(x["q_latent"].cuda(), x["q_rope"].cuda(), lp.cuda(), rp.cuda(),
                                              table.cuda(), x["seq_lens"].cuda(), cfg.scale, x["latent_scale"],
                                              x["rope_scale"])
    torch.cuda.synchronize()
    ro, rl = oracle.mla_decode_fp8(x["q_latent"], x["q_rope"], x["latent_cache"], x["rope_cache"], x["seq_lens"],
                                   cfg.scale, x["latent_scale"], x["rope_scale"])
    assert_close(out.cpu().numpy(), ro, "mla fp8 paged out")
    assert_close(lse.cpu().numpy(), rl, "mla fp8 paged lse")


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16)


def _signed_code(c):
    """E4M3 codes as signed integers ordered like their values (sign-magnitude -> +-mag)."""
    c = c.to(torch.int32)
    mag = c & 0x7F
    return torch.where((c & 0x80) != 0, -mag, mag)


def test_append_fp8_then_decode_matches_oracle():
    """One MLA step into an E4M3 cache end to end: rotate + quantise-append the new token
    (its latent and RoPE key), then the fp8 decode, against the oracle appending its own
    codes and attending in fp64."""
    cfg = mla8("step8", 4, 128, 1500, [1500, 1, 700, 64])
    x = wl.make_mla_inputs_fp8(cfg, seed=12)
    g = torch.Generator().manual_seed(13)
    lat_new = torch.randn((cfg.batch, 512), generator=g).to(torch.bfloat16)
    rope_new = torch.randn((cfg.batch, 64), generator=g).to(torch.bfloat16)
    pos = (x["seq_lens"] - 1).to(torch.int32)
    dq, dlc, drc = x["q_rope"].cuda(), x["latent_cache"].cuda(), x["rope_cache"].cuda()
    kb.kvattn_mla_rope_append_fp8(dq, lat_new.cuda(), rope_new.cuda(), pos.cuda(), dlc, drc, x["latent_scale"],
                                  x["rope_scale"])
    out, lse = kb.kvattn_mla_decode_fp8(x["q_latent"].cuda(), dq, dlc, drc, x["seq_lens"].cuda(), cfg.scale,
                                        x["latent_scale"], x["rope_scale"])
    torch.cuda.synchronize()
    q_ref = _bf16(oracle.rope_f64(x["q_rope"], pos.numpy(), 10000.0, 0))
    r_rot = np.asarray(oracle.rope_f64(rope_new, pos.numpy(), 10000.0, 0), dtype=np.float32)
    r_codes = torch.from_numpy(oracle.e4m3_quant(r_rot, x["rope_scale"]))
    l_codes = torch.from_numpy(oracle.e4m3_quant(lat_new.float().numpy(), x["latent_scale"]))
    lc, rc = x["latent_cache"].view(torch.uint8).clone(), x["rope_cache"].view(torch.uint8).clone()
    for b in range(cfg.batch):
        p = int(pos[b])
        lc[b, p] = l_codes[b]
        # the kernel rotates in fp32, the oracle in fp64: the key codes may differ by one
        # step, so the oracle attends over the kernel's codes where they are that close
        dk = drc.view(torch.uint8)[b, p].cpu()
        assert int((_signed_code(dk) - _signed_code(r_codes[b])).abs().max()) <= 1
        rc[b, p] = dk
    assert torch.equal(dlc.view(torch.uint8).cpu(), lc), "latent codes"
    ro, rl = oracle.mla_decode_fp8(x["q_latent"], q_ref, lc, rc, x["seq_lens"], cfg.scale, x["latent_scale"],
                                   x["rope_scale"])
    assert_close(out.cpu().numpy(), ro, "mla fp8 step out")
    assert_close(lse.cpu().numpy(), rl, "mla fp8 step lse")


def test_multi_token_fp8():
    """Three new tokens per sequence over the E4M3 cache (causal)."""
    cfg = mla8("multi8", 3, 128, 800, [800, 2, 450])
    x = wl.make_mla_inputs_fp8(cfg, seed=21, poison_tail=True)
    g = torch.Generator().manual_seed(22)
    ql = torch.randn((cfg.batch, 3, 128, 512), generator=g).to(torch.bfloat16)
    qr = torch.randn((cfg.batch, 3, 128, 64), generator=g).to(torch.bfloat16)
    out, lse = kb.kvattn_mla_decode_multi(ql.cuda(), qr.cuda(), x["latent_cache"].cuda(), x["rope_cache"].cuda(),
                                          x["seq_lens"].cuda(), cfg.scale, x["latent_scale"], x["rope_scale"])
    torch.cuda.synchronize()
    lat = oracle.e4m3_dequant(x["latent_cache"], x["latent_scale"])
    rope = oracle.e4m3_dequant(x["rope_cache"], x["rope_scale"])
    ro, rl = oracle.mla_decode_multi(ql, qr, lat, rope, x["seq_lens"], cfg.scale)
    assert_close(out.cpu().numpy(), ro, "mla fp8 multi out")
    assert_close(lse.cpu().numpy(), rl, "mla fp8 multi lse")
