"""GPU parity of kvattn_gqa_decode_multi (several new tokens per sequence, causal mask,
optional sliding window) against the fp64 oracle (B200).

The cache positions >= seq_len are NaN, so a read past a sequence shows; with a window
the tiles wholly before the earliest visible position are skipped, so the tests also
poison those rows for the windowed cases that skip whole tiles.
"""
import math

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
def _knobs():
    kb.kvattn_debug_set_workers(0, 0)
    kb.kvattn_debug_set_gqa_kernel(0)
    kb.kvattn_clear_device_flags()
    yield
    kb.kvattn_debug_set_workers(0, 0)
    kb.kvattn_debug_set_gqa_kernel(0)
    assert kb.kvattn_read_device_flags() == 0


def run_multi(B, L, n_q, n_kv, T, lens, window, seed=0, poison_before=False, d=128):
    cfg = wl.GQAConfig("multi", B, n_q, n_kv, d, T, 1.0 / math.sqrt(d), seq_lens=tuple(lens))
    x = wl.make_gqa_inputs(cfg, seed=seed, poison_tail=True)
    g = torch.Generator().manual_seed(seed + 1)
    q = torch.randn((B, L, n_q, d), generator=g).to(torch.bfloat16)
    k, v = x["k_cache"], x["v_cache"]
    if poison_before and window > 0:
        # rows before every query's window, in tiles of 128 that hold no visible row
        for b, n in enumerate(lens):
            first = max(0, n - L + 1 - window)
            cut = (first // 128) * 128
            k[b, :, :cut] = float("nan")
            v[b, :, :cut] = float("nan")
    out, lse = kb.kvattn_gqa_decode_multi(q.cuda(), k.cuda(), v.cuda(), x["seq_lens"].cuda(), cfg.scale,
                                          window=window)
    torch.cuda.synchronize()
    if poison_before and window > 0:
        k, v = torch.nan_to_num(k, nan=0.0), torch.nan_to_num(v, nan=0.0)
    ro, rl = oracle.gqa_decode_multi(q, k, v, x["seq_lens"], cfg.scale, window=window)
    assert_close(out.cpu().numpy(), ro, f"multi L{L} w{window} out")
    assert_close(lse.cpu().numpy(), rl, f"multi L{L} w{window} lse")
    return q, x, out, lse


CASES = [
    # (n_q, n_kv, L, window)
    (32, 8, 4, 0), (32, 8, 8, 0), (8, 8, 8, 0), (64, 16, 16, 0), (32, 4, 8, 100), (32, 8, 2, 1),
    (32, 32, 1, 300), (16, 1, 4, 5000), (32, 8, 3, 129),
]


@pytest.mark.parametrize("n_q,n_kv,L,window", CASES, ids=[f"g{a // b}_L{c}_w{d}" for a, b, c, d in CASES])
def test_multi_token(n_q, n_kv, L, window):
    lens = [1000, 0, 1, 2, 129, 3000, 128, 257]
    run_multi(len(lens), L, n_q, n_kv, 3000, lens, window)


def test_sliding_window_long_skips_tiles():
    """Mistral-style window of 4096 over contexts up to 8192: the tiles before the window
    hold NaN and must not be read."""
    lens = [8192, 5000, 4097, 4096, 300, 8000]
    run_multi(len(lens), 4, 32, 8, 8192, lens, 4096, seed=3, poison_before=True)


@pytest.mark.parametrize("workers", [7, 64, 300])
def test_multi_forced_splits(workers):
    kb.kvattn_debug_set_workers(workers, 1)
    run_multi(4, 4, 32, 8, 2000, [2000, 1500, 3, 777], 0, seed=5)
    run_multi(4, 2, 32, 8, 2000, [2000, 1500, 3, 777], 600, seed=6)


def test_single_token_matches_decode():
    """q_len 1 without a window is the single-token call, bit for bit (same kernel)."""
    lens = [1000, 0, 1, 129]
    cfg = wl.GQAConfig("one", len(lens), 32, 8, 128, 1000, 1.0 / math.sqrt(128.0), seq_lens=tuple(lens))
    x = wl.make_gqa_inputs(cfg, seed=9, poison_tail=True)
    d = {k: v.cuda() for k, v in x.items()}
    kb.kvattn_debug_set_gqa_kernel(2)       # the single-token call on the kernel the multi call runs
    o1, l1 = kb.kvattn_gqa_decode_multi(d["q"][:, None].contiguous(), d["k_cache"], d["v_cache"], d["seq_lens"],
                                        cfg.scale)
    o2, l2 = kb.kvattn_gqa_decode(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], cfg.scale)
    torch.cuda.synchronize()
    assert torch.equal(o1[:, 0], o2) and torch.equal(l1[:, 0], l2)


# Shapes the multi-token kernel does not take (head_dim 64; a group's heads times the new
# tokens above 64 columns): the call runs as a virtual batch of single-token sequences.
VIRTUAL = [
    # (B, L, n_q, n_kv, T, lens, window, d)
    (3, 3, 16, 4, 700, (700, 2, 333), 0, 64),
    (2, 5, 64, 4, 1500, (1500, 3), 0, 128),        # 16 heads x 5 tokens = 80 columns
    (2, 5, 64, 4, 1500, (1500, 777), 200, 128),    # the same with a window
    (2, 4, 32, 1, 3000, (3000, 1), 0, 128),        # MQA, 32 heads x 4 tokens
    (2, 2, 128, 2, 600, (600, 1), 0, 128),         # 64-head groups x 2 tokens
]


@pytest.mark.parametrize("B,L,n_q,n_kv,T,lens,window,d", VIRTUAL,
                         ids=[f"d{c[7]}_g{c[2] // c[3]}_L{c[1]}_w{c[6]}" for c in VIRTUAL])
def test_multi_as_virtual_batch(B, L, n_q, n_kv, T, lens, window, d):
    run_multi(B, L, n_q, n_kv, T, list(lens), window, seed=7, poison_before=window > 0, d=d)
