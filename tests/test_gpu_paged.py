"""GPU parity of the paged-cache decode entry points (B200).

Each case takes a seeded contiguous cache, cuts every sequence into pages of page_size
rows and scatters them over a shuffled pool that also holds never-referenced pages full
of NaN (a read of one would show); block-table entries past a sequence's last page are
out-of-range values that must never be read.  The paged result is compared with the fp64
oracle on the contiguous cache, and with the contiguous entry point's result, which it
must equal bit for bit (same kernel, same work split, same tiles).
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
def _knobs():
    kb.kvattn_debug_set_workers(0, 0)
    kb.kvattn_debug_set_gqa_kernel(0)
    kb.kvattn_clear_device_flags()
    yield
    kb.kvattn_debug_set_workers(0, 0)
    kb.kvattn_debug_set_gqa_kernel(0)
    assert kb.kvattn_read_device_flags() == 0


def paginate(cache, lens, page_size, seq_axis, seed, extra_pages=5):
    """cache [B, ..., T, ...] (T at seq_axis) -> (pool [P, ...page...], block_table [B, T/page_size])."""
    B, T = cache.shape[0], cache.shape[seq_axis]
    M = T // page_size
    need = [max(0, math.ceil(int(l) / page_size)) for l in lens]
    total = sum(need) + extra_pages
    rng = np.random.default_rng(seed)
    phys = rng.permutation(total)
    page_shape = list(cache.shape[1:])
    page_shape[seq_axis - 1] = page_size
    pool = torch.full([total] + page_shape, float("nan"), dtype=cache.dtype)
    table = torch.full((B, M), 1 << 30, dtype=torch.int32)     # never read past a sequence's pages
    nxt = 0
    for b in range(B):
        for lp in range(need[b]):
            p = int(phys[nxt])
            nxt += 1
            table[b, lp] = p
            pool[p] = cache[b].narrow(seq_axis - 1, lp * page_size, page_size)
    return pool, table


GQA_CASES = [
    # (n_q, n_kv, d, page_size, kernel)   kernel: 1 warp-level, 2 tcgen05, 0 built-in choice
    (32, 32, 128, 64, 0), (32, 4, 128, 64, 0), (32, 4, 128, 128, 2), (32, 4, 128, 128, 1),
    (64, 2, 128, 256, 2), (16, 2, 64, 128, 0), (32, 1, 128, 256, 0),
]


@pytest.mark.parametrize("n_q,n_kv,d,page_size,kernel", GQA_CASES,
                         ids=[f"g{a // b}_d{c}_page{e}_k{f}" for a, b, c, e, f in GQA_CASES])
def test_gqa_paged(n_q, n_kv, d, page_size, kernel):
    kb.kvattn_debug_set_gqa_kernel(kernel)
    T = 1024
    lens = (1024, 0, 1, 64, 65, 127, 128, 129, 700, 256)
    cfg = wl.GQAConfig("paged", len(lens), n_q, n_kv, d, T, 1.0 / math.sqrt(d), seq_lens=lens)
    x = wl.make_gqa_inputs(cfg, seed=31, poison_tail=True)
    kp, table = paginate(x["k_cache"], lens, page_size, 2, seed=5)
    vp, _ = paginate(x["v_cache"], lens, page_size, 2, seed=5)
    dq, dlens = x["q"].cuda(), x["seq_lens"].cuda()
    out, lse = kb.kvattn_gqa_decode_paged(dq, kp.cuda(), vp.cuda(), table.cuda(), dlens, cfg.scale)
    # the contiguous call on the kernel the paged call ran (the tcgen05 kernel needs pages
    # of whole 128-token tiles; the built-in choice would otherwise differ)
    used = kernel or (2 if d == 128 and n_q // n_kv >= 4 and page_size % 128 == 0 else 1)
    kb.kvattn_debug_set_gqa_kernel(used)
    oc, lc = kb.kvattn_gqa_decode(dq, x["k_cache"].cuda(), x["v_cache"].cuda(), dlens, cfg.scale)
    torch.cuda.synchronize()
    ro, rl = oracle.gqa_decode(x["q"], x["k_cache"], x["v_cache"], x["seq_lens"], cfg.scale)
    assert_close(out.cpu().numpy(), ro, "paged out")
    assert_close(lse.cpu().numpy(), rl, "paged lse")
    assert torch.equal(out, oc) and torch.equal(lse, lc), "paged and contiguous results differ"


@pytest.mark.parametrize("page_size", [64, 128])
def test_mla_paged(page_size):
    T = 1024
    lens = (1024, 0, 1, 64, 65, 200, 513)
    cfg = wl.MLAConfig("paged", len(lens), 128, 512, 64, T, 1.0 / math.sqrt(192.0), seq_lens=lens)
    x = wl.make_mla_inputs(cfg, seed=32, poison_tail=True)
    lp, table = paginate(x["latent_cache"], lens, page_size, 1, seed=6)
    rp, _ = paginate(x["rope_cache"], lens, page_size, 1, seed=6)
    d = {k: v.cuda() for k, v in x.items()}
    out, lse = kb.kvattn_mla_decode_paged(d["q_latent"], d["q_rope"], lp.cuda(), rp.cuda(), table.cuda(),
                                          d["seq_lens"], cfg.scale)
    oc, lc = kb.kvattn_mla_decode(d["q_latent"], d["q_rope"], d["latent_cache"], d["rope_cache"],
                                  d["seq_lens"], cfg.scale)
    torch.cuda.synchronize()
    ro, rl = oracle.mla_decode(x["q_latent"], x["q_rope"], x["latent_cache"], x["rope_cache"],
                               x["seq_lens"], cfg.scale)
    assert_close(out.cpu().numpy(), ro, "mla paged out")
    assert_close(lse.cpu().numpy(), rl, "mla paged lse")
    assert torch.equal(out, oc) and torch.equal(lse, lc), "paged and contiguous results differ"


def test_paged_forced_splits():
    """Many workers: pieces start and end inside pages and the combine merges them."""
    kb.kvattn_debug_set_workers(37, 1)
    T, lens = 2048, (2048, 1500, 3, 1024)
    cfg = wl.GQAConfig("paged_split", len(lens), 32, 8, 128, T, 1.0 / math.sqrt(128.0), seq_lens=lens)
    x = wl.make_gqa_inputs(cfg, seed=33, poison_tail=True)
    kp, table = paginate(x["k_cache"], lens, 128, 2, seed=7)
    vp, _ = paginate(x["v_cache"], lens, 128, 2, seed=7)
    out, lse = kb.kvattn_gqa_decode_paged(x["q"].cuda(), kp.cuda(), vp.cuda(), table.cuda(),
                                          x["seq_lens"].cuda(), cfg.scale)
    torch.cuda.synchronize()
    ro, rl = oracle.gqa_decode(x["q"], x["k_cache"], x["v_cache"], x["seq_lens"], cfg.scale)
    assert_close(out.cpu().numpy(), ro, "split out")
    assert_close(lse.cpu().numpy(), rl, "split lse")
