"""GPU parity of kvattn_mla_decode (tcgen05 CTA-pair kernel) against the fp64 oracle.

Cache positions >= seq_len are NaN-filled; the full-size DeepSeek-shaped workload is
compared on every sequence in the bench's launch configuration.
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

SCALE = 1.0 / math.sqrt(192.0)


@pytest.fixture(autouse=True)
def _reset_knob():
    kb.kvattn_debug_set_workers(0, 0)
    kb.kvattn_clear_device_flags()
    yield
    kb.kvattn_debug_set_workers(0, 0)
    assert kb.kvattn_read_device_flags() == 0, "a bounded wait ran out on the device"


def run_case(cfg, seed=0, poison=True, q_gain=1.0, lat_gain=1.0, out_offset=0):
    x = wl.make_mla_inputs(cfg, seed=seed, poison_tail=poison)
    if q_gain != 1.0:  # a power of two keeps the bf16 values exact
        x["q_latent"] = (x["q_latent"].float() * q_gain).to(torch.bfloat16)
        x["q_rope"] = (x["q_rope"].float() * q_gain).to(torch.bfloat16)
    if lat_gain != 1.0:  # latents times a power of two, latent queries divided by it
        x["latent_cache"] = (x["latent_cache"].float() * lat_gain).to(torch.bfloat16)
        x["q_latent"] = (x["q_latent"].float() / lat_gain).to(torch.bfloat16)
    d = {k: v.cuda() for k, v in x.items()}
    out = None
    if out_offset:  # an output buffer that starts out_offset floats into an allocation
        B, H = cfg.batch, cfg.n_heads
        out = torch.full((B * H * 512 + out_offset,), float("nan"), device="cuda")[out_offset:].view(B, H, 512)
    out, lse = kb.kvattn_mla_decode(d["q_latent"], d["q_rope"], d["latent_cache"], d["rope_cache"],
                                    d["seq_lens"], cfg.scale, out=out)
    torch.cuda.synchronize()
    ro, rl = oracle.mla_decode(x["q_latent"], x["q_rope"], x["latent_cache"], x["rope_cache"],
                               x["seq_lens"], cfg.scale)
    # the output scales with the latents; compare it in the base case's units so the
    # tolerance's absolute floor means the same thing
    assert_close(out.cpu().numpy() / lat_gain, ro / lat_gain, f"{cfg.name} out")
    assert_close(lse.cpu().numpy(), rl, f"{cfg.name} lse")
    return out, lse


def mla(name, B, H, T, lens=None):
    return wl.MLAConfig(name, B, H, 512, 64, T, SCALE, seq_lens=tuple(lens) if lens else None)


@pytest.mark.parametrize("T", [1, 2, 3, 63, 64, 65, 128, 200, 1000])
def test_lengths(T):
    run_case(mla(f"T{T}", 2, 128, T, lens=[T, max(T // 3, 1)]))


@pytest.mark.parametrize("H", [1, 16, 64, 100, 128])
def test_head_counts(H):
    run_case(mla(f"H{H}", 3, H, 300, lens=[300, 129, 5]))


def test_ragged_with_empty_sequences():
    run_case(mla("ragged", 6, 128, 700, lens=[0, 1, 64, 65, 700, 0]))


def test_sharp_softmax_rescales():
    """Queries scaled by 4: the running max keeps growing by more than 2^8 between tiles,
    which exercises the rescale of the TMEM accumulator."""
    run_case(mla("sharp", 2, 128, 1500, lens=[1500, 400]), q_gain=4.0)


def test_latents_beyond_fp16_range():
    """Latent values up to ~2^19 (far outside fp16) with the same scores as the base case:
    the values stay bf16 all the way through the value product, and the output (divided
    by the gain, like the oracle's) meets the base case's tolerance."""
    run_case(mla("big", 2, 128, 700, lens=[700, 129]), lat_gain=2.0 ** 17)


def test_output_16_byte_aligned():
    """An output 16 but not 32 bytes aligned (the epilogue's 32-byte stores need 32)."""
    run_case(mla("out16", 3, 128, 500, lens=[500, 77, 260]), out_offset=4)


@pytest.mark.parametrize("workers,min_tiles", [(1, 1), (2, 1), (3, 1), (7, 1), (40, 1)])
def test_forced_splits(workers, min_tiles):
    kb.kvattn_debug_set_workers(workers, min_tiles)
    run_case(mla("split", 4, 128, 2000, lens=[2000, 1, 0, 777]))


def test_many_short_ragged_sequences():
    """300 sequences of 0-400 tokens: every worker runs pieces of several sequences, and
    the sequences cut by worker boundaries are merged by their last worker."""
    lens = np.random.default_rng(31).integers(0, 401, size=300).tolist()
    run_case(mla("many", 300, 128, 400, lens=lens))


def test_largest_batch():
    """1024 sequences (the largest batch) of at most 64 tokens: one tile each, ~14 pieces
    per worker, the merge counters of every sequence in use."""
    lens = np.random.default_rng(32).integers(1, 65, size=1024).tolist()
    run_case(mla("b1024", 1024, 128, 64, lens=lens))


def test_workload_full_size():
    run_case(wl.CONFIGS["mla_b32_h128_c512_r64_t4096"])


@pytest.mark.parametrize("L", [2, 4])
def test_multi_token(L):
    """L new tokens per sequence (causal), including sequences shorter than L (their first
    queries see nothing)."""
    cfg = mla("multi", 4, 128, 900, lens=[900, 1, 3, 500])
    x = wl.make_mla_inputs(cfg, seed=17, poison_tail=True)
    g = torch.Generator().manual_seed(18)
    ql = torch.randn((cfg.batch, L, 128, 512), generator=g).to(torch.bfloat16)
    qr = torch.randn((cfg.batch, L, 128, 64), generator=g).to(torch.bfloat16)
    out, lse = kb.kvattn_mla_decode_multi(ql.cuda(), qr.cuda(), x["latent_cache"].cuda(), x["rope_cache"].cuda(),
                                          x["seq_lens"].cuda(), cfg.scale)
    torch.cuda.synchronize()
    ro, rl = oracle.mla_decode_multi(ql, qr, x["latent_cache"], x["rope_cache"], x["seq_lens"], cfg.scale)
    assert_close(out.cpu().numpy(), ro, f"mla multi L{L} out")
    assert_close(lse.cpu().numpy(), rl, f"mla multi L{L} lse")


def test_lengths_past_the_capacity_are_clamped():
    """seq_lens above max_seq_len attend to the whole cache (clamped), no further."""
    cfg = mla("clamp", 2, 128, 300, lens=[300, 120])
    x = wl.make_mla_inputs(cfg, seed=19)
    d = {k: v.cuda() for k, v in x.items()}
    big = torch.tensor([5000, 120], dtype=torch.int32, device="cuda")
    out, lse = kb.kvattn_mla_decode(d["q_latent"], d["q_rope"], d["latent_cache"], d["rope_cache"], big, cfg.scale)
    torch.cuda.synchronize()
    ro, rl = oracle.mla_decode(x["q_latent"], x["q_rope"], x["latent_cache"], x["rope_cache"], x["seq_lens"],
                               cfg.scale)
    assert_close(out.cpu().numpy(), ro, "clamped out")
    assert_close(lse.cpu().numpy(), rl, "clamped lse")
