"""GPU parity of the E4M3 (fp8) KV-cache decode against the fp64 oracle (B200).

The caches hold E4M3 codes with one scale per tensor (the seeded generator takes the
scale from the tensor's largest magnitude); rows past every sequence's length hold the
NaN code, so a read of one shows.  The oracle attends over the dequantised cache in
fp64; the kernel feeds the codes to the tensor cores as they are and the bf16 query and
the softmax weights as two E4M3 parts each, so the library tolerance
|gpu - oracle| <= 2e-3 (1 + |oracle|) applies unchanged.
"""
import math

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


@pytest.fixture(autouse=True)
def _knobs():
    kb.kvattn_debug_set_workers(0, 0)
    kb.kvattn_clear_device_flags()
    yield
    kb.kvattn_debug_set_workers(0, 0)
    assert kb.kvattn_read_device_flags() == 0


def fp8_inputs(B, n_q, n_kv, T, lens, seed, **cfg_kw):
    cfg = wl.GQAConfig("fp8", B, n_q, n_kv, 128, T, 1.0 / math.sqrt(128.0), seq_lens=tuple(lens), **cfg_kw)
    return cfg, wl.make_gqa_inputs_fp8(cfg, seed=seed, poison_tail=True)


def run_fp8(cfg, x, q=None, window=0):
    q = x["q"] if q is None else q
    out, lse = kb.kvattn_gqa_decode_fp8(q.cuda(), x["k_cache"].cuda(), x["v_cache"].cuda(), x["seq_lens"].cuda(),
                                        cfg.scale, x["k_scale"], x["v_scale"], window=window)
    torch.cuda.synchronize()
    ro, rl = oracle.gqa_decode_fp8(q, x["k_cache"], x["v_cache"], x["seq_lens"], cfg.scale, x["k_scale"],
                                   x["v_scale"], window=window)
    return out, lse, ro, rl


CASES = [(32, 32), (32, 8), (64, 8), (32, 1), (64, 1), (16, 2)]


@pytest.mark.parametrize("n_q,n_kv", CASES, ids=[f"g{a // b}" for a, b in CASES])
def test_fp8_decode(n_q, n_kv):
    lens = [2000, 0, 1, 127, 128, 129, 1500, 64]
    cfg, x = fp8_inputs(len(lens), n_q, n_kv, 2000, lens, seed=61)
    out, lse, ro, rl = run_fp8(cfg, x)
    assert_close(out.cpu().numpy(), ro, "fp8 out")
    assert_close(lse.cpu().numpy(), rl, "fp8 lse")


def test_fp8_spiky_keys():
    """The long-context MQA distribution (1 % of key positions offset by +4 on every
    dimension): a few dominant weights next to a long tail of small ones."""
    lens = [8192, 8192, 5000]
    cfg, x = fp8_inputs(3, 32, 1, 8192, lens, seed=62, spike_fraction=0.01, spike_value=4.0)
    out, lse, ro, rl = run_fp8(cfg, x)
    assert_close(out.cpu().numpy(), ro, "fp8 spiky out")
    assert_close(lse.cpu().numpy(), rl, "fp8 spiky lse")


def test_fp8_sharp_keys_ragged():
    """Keys scaled by 2 (the 70B-shaped workload's sharper softmax), ragged lengths."""
    lens = [1024, 8192, 3333, 4097]
    cfg, x = fp8_inputs(4, 64, 8, 8192, lens, seed=63, key_scale=2.0)
    out, lse, ro, rl = run_fp8(cfg, x)
    assert_close(out.cpu().numpy(), ro, "fp8 sharp out")
    assert_close(lse.cpu().numpy(), rl, "fp8 sharp lse")


@pytest.mark.parametrize("B,n_q,n_kv,T", [(2, 32, 1, 128 * 37), (3, 16, 2, 1000)],
                         ids=["2units_37tiles", "6units_8tiles"])
def test_fp8_equal_units_in_parts(B, n_q, n_kv, T):
    """Every sequence of the same length and no more units than workers: each unit is cut
    into consecutive parts of its own (the last one shorter), which the combine merges."""
    cfg, x = fp8_inputs(B, n_q, n_kv, T, [T] * B, seed=66)
    out, lse, ro, rl = run_fp8(cfg, x)
    assert_close(out.cpu().numpy(), ro, "fp8 parts out")
    assert_close(lse.cpu().numpy(), rl, "fp8 parts lse")
    # several new tokens over equal lengths (the multi-token instantiation)
    g = torch.Generator().manual_seed(67)
    q = torch.randn((B, 2, n_q, 128), generator=g).to(torch.bfloat16)
    out, lse, ro, rl = run_fp8(cfg, x, q=q)
    assert_close(out.cpu().numpy(), ro, "fp8 parts multi out")
    assert_close(lse.cpu().numpy(), rl, "fp8 parts multi lse")


@pytest.mark.parametrize("L,window", [(4, 0), (8, 100), (2, 1), (16, 0)])
def test_fp8_multi_token(L, window):
    lens = [1000, 0, 2, 129, 3000, 257]
    cfg, x = fp8_inputs(len(lens), 32, 8, 3000, lens, seed=64)
    g = torch.Generator().manual_seed(65)
    q = torch.randn((len(lens), L, 32, 128), generator=g).to(torch.bfloat16)
    out, lse, ro, rl = run_fp8(cfg, x, q=q, window=window)
    assert_close(out.cpu().numpy(), ro, f"fp8 multi L{L} w{window} out")
    assert_close(lse.cpu().numpy(), rl, f"fp8 multi L{L} w{window} lse")


def test_fp8_query_scale_extremes():
    """Query blocks far from unit scale (the split rescales each block by a power of two)."""
    lens = [700, 300]
    cfg, x = fp8_inputs(2, 16, 2, 700, lens, seed=66)
    for mult in (1e-3, 40.0):
        q = (x["q"].float() * mult).to(torch.bfloat16)
        out, lse, ro, rl = run_fp8(cfg, x, q=q)
        assert_close(out.cpu().numpy(), ro, f"fp8 q*{mult} out")
        assert_close(lse.cpu().numpy(), rl, f"fp8 q*{mult} lse")


@pytest.mark.parametrize("workers", [5, 97])
def test_fp8_forced_splits(workers):
    kb.kvattn_debug_set_workers(workers, 1)
    lens = [3000, 1500, 3, 777]
    cfg, x = fp8_inputs(4, 32, 8, 3000, lens, seed=67)
    out, lse, ro, rl = run_fp8(cfg, x)
    assert_close(out.cpu().numpy(), ro, "fp8 split out")
    assert_close(lse.cpu().numpy(), rl, "fp8 split lse")


@pytest.mark.parametrize("page_size", [128, 256])
def test_fp8_paged(page_size):
    lens = (1024, 0, 1, 128, 129, 700, 1000)
    cfg, x = fp8_inputs(len(lens), 32, 4, 1024, lens, seed=68)
    # pages of codes: the NaN fill of unreferenced pages is the NaN code
    kp, table = paginate(x["k_cache"].view(torch.uint8).float(), lens, page_size, 2, seed=9)
    vp, _ = paginate(x["v_cache"].view(torch.uint8).float(), lens, page_size, 2, seed=9)
    kp = torch.nan_to_num(kp, nan=127.0).to(torch.uint8)
    vp = torch.nan_to_num(vp, nan=127.0).to(torch.uint8)
    dq, dl = x["q"].cuda(), x["seq_lens"].cuda()
    out, lse = kb.kvattn_gqa_decode_fp8_paged(dq, kp.cuda(), vp.cuda(), table.cuda(), dl, cfg.scale,
                                              x["k_scale"], x["v_scale"])
    oc, lc = kb.kvattn_gqa_decode_fp8(dq, x["k_cache"].cuda(), x["v_cache"].cuda(), dl, cfg.scale, x["k_scale"],
                                      x["v_scale"])
    torch.cuda.synchronize()
    ro, rl = oracle.gqa_decode_fp8(x["q"], x["k_cache"], x["v_cache"], x["seq_lens"], cfg.scale, x["k_scale"],
                                   x["v_scale"])
    assert_close(out.cpu().numpy(), ro, "fp8 paged out")
    assert_close(lse.cpu().numpy(), rl, "fp8 paged lse")
    assert torch.equal(out, oc) and torch.equal(lse, lc), "paged and contiguous results differ"



def test_fp8_multi_token_beyond_64_columns():
    """32-head groups at 3 new tokens (96 columns): a virtual batch of single-token
    sequences through the E4M3 kernel."""
    lens = [1500, 2, 700]
    cfg, x = fp8_inputs(len(lens), 64, 2, 1500, lens, seed=64)
    g = torch.Generator().manual_seed(65)
    q = torch.randn((len(lens), 3, 64, 128), generator=g).to(torch.bfloat16)
    out, lse, ro, rl = run_fp8(cfg, x, q=q)
    assert_close(out.cpu().numpy(), ro, "fp8 multi out")
    assert_close(lse.cpu().numpy(), rl, "fp8 multi lse")
