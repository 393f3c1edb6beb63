"""The oracle, pinned to what the pages and the mathematics fix (CPU only)."""
import json
import os

import numpy as np
import pytest

import oracle
from oracle import cache_bytes as cb
from tests import oracle_pins

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "cache_bytes.json")


@pytest.fixture(scope="module")
def golden():
    with open(GOLDEN) as f:
        return json.load(f)


def test_cache_bytes_golden(golden):
    for case in golden["cases"]:
        fn = getattr(cb, case["fn"])
        assert fn(*case["args"]) == case["expected"], case["cite"]


def test_cache_bytes_bandwidth_table(golden):
    # per step over all 12 layers of the running model (h = 8, d_k = d_v = 64)
    for t, mha, gqa2, mqa in golden["bandwidth_table_mib"]["rows"]:
        assert cb.kv_cache_bytes(12, 8, 64, t) / 2**20 == mha
        assert cb.kv_cache_bytes(12, 2, 64, t) / 2**20 == gqa2
        assert cb.kv_cache_bytes(12, 1, 64, t) / 2**20 == mqa


def test_cache_bytes_calculator_printout(golden):
    for n_kv, line in golden["calculator_printout"]["lines"]:
        gib = cb.kv_cache_bytes(32, n_kv, 128, 4096) / 2**30
        assert f"n_kv_heads={n_kv:2d}: {gib:.3f} GiB" == line


def test_cache_bytes_reduction_and_mla(golden):
    # the reduction factor is n_q / n_kv whatever the other terms are
    for L, d, T in [(12, 64, 4096), (32, 128, 1), (80, 128, 128000)]:
        for n_q, n_kv in [(8, 2), (32, 8), (64, 8), (32, 1)]:
            ratio = cb.kv_cache_bytes(L, n_q, d, T) / cb.kv_cache_bytes(L, n_kv, d, T)
            assert ratio == cb.reduction_factor(n_q, n_kv)
    # notebook checks: g = 4 saves 4x, MQA saves n_head x (16 heads, head_dim 16)
    assert cb.kv_bytes_per_token_layer(16, 16, 16) / cb.kv_bytes_per_token_layer(4, 16, 16) == 4.0
    assert cb.kv_bytes_per_token_layer(16, 16, 16) / cb.kv_bytes_per_token_layer(1, 16, 16) == 16.0
    mla = golden["mla"]
    assert 2 * 128 * 128 == mla["mha_numbers_per_token"]
    assert mla["mha_numbers_per_token"] // mla["latent"] == mla["latent_reduction"]
    assert mla["latent"] + mla["rope"] == mla["per_token_elements"]
    assert cb.mla_cache_bytes(1, 512, 64, 1) == 2 * mla["per_token_elements"]
    assert mla["per_token_elements"] / (2 * 128) == mla["equivalent_gqa_groups"]


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(pin, oracle_lib):
    pin(oracle_lib)


def test_bf16_conversion_is_exact():
    """The wrapper's bf16 -> fp64 conversion keeps every bf16 value exactly."""
    import torch
    bits = torch.arange(0, 1 << 16, dtype=torch.int32).to(torch.int16).view(torch.bfloat16)
    as64 = oracle._f64(bits)
    back = torch.from_numpy(as64).to(torch.bfloat16)
    finite = torch.isfinite(bits.float())
    assert torch.equal(back[finite].view(torch.int16), bits[finite].view(torch.int16))


def test_bf16_wrapper_matches_f64_core(oracle_lib):
    """gqa_decode (bf16 inputs, per-sequence calls, tails never read) equals the fp64
    core on the converted arrays; NaN in the unread tail must not leak in."""
    import torch
    from mla_kv_cache_b200 import workloads as wl
    cfg = wl.GQAConfig("t", 3, 8, 2, 16, 40, 0.25, seq_lens=(40, 7, 0))
    x = wl.make_gqa_inputs(cfg, seed=3, poison_tail=True)
    o, l = oracle.gqa_decode(x["q"], x["k_cache"], x["v_cache"], x["seq_lens"], 0.25)
    k = x["k_cache"].clone(); v = x["v_cache"].clone()
    k[torch.isnan(k)] = 0; v[torch.isnan(v)] = 0
    o2, l2 = oracle.gqa_decode_f64(x["q"], k, v, x["seq_lens"], 0.25)
    assert np.array_equal(o, o2) and np.array_equal(l, l2)
    assert np.isfinite(o).all()
