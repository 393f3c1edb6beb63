"""The oracle's per-sequence wrappers, pinned to its fp64 core (CPU only).

The GPU parity tests call the wrappers (oracle.gqa_decode, oracle.mla_decode,
oracle.gqa_decode_multi, oracle.gqa_decode_fp8, oracle.mla_decode_fp8): they take the bf16 (or E4M3) tensors,
convert only the rows a sequence attends to, and call the fp64 core one sequence at a
time.  The core itself is pinned by tests/oracle_pins.py; here each wrapper must give
exactly (bit for bit) what the core gives on the whole batch at once, on inputs whose
cache positions past each length hold NaN (NaN codes for E4M3).  The whole-batch
reference sees those tails zeroed, so a wrapper that read one row too many would leak
a NaN, and one that read one row too few would drop a token.  Lengths cover 0, 1, a
ragged middle and the full capacity; the multi-token case also has sequences shorter
than the number of new tokens (queries that precede the cache's start).

A planted mistake -- the wrappers' row count one short -- must make every check fail.
"""
import numpy as np
import pytest
import torch

import oracle
from mla_kv_cache_b200 import workloads as wl


def _zero_nan(x):
    x = x.clone()
    x[torch.isnan(x)] = 0
    return x


def check_mla():
    cfg = wl.MLAConfig("wrap_mla", 5, 6, 32, 8, 23, 0.21, seq_lens=(23, 0, 1, 9, 22))
    x = wl.make_mla_inputs(cfg, seed=31, poison_tail=True)
    o, l = oracle.mla_decode(x["q_latent"], x["q_rope"], x["latent_cache"], x["rope_cache"],
                             x["seq_lens"], cfg.scale)
    o2, l2 = oracle.mla_decode_f64(x["q_latent"], x["q_rope"], _zero_nan(x["latent_cache"]),
                                   _zero_nan(x["rope_cache"]), x["seq_lens"], cfg.scale)
    assert np.array_equal(o, o2) and np.array_equal(l, l2), "mla wrapper differs from the core"
    assert np.isfinite(o).all()
    # a subset of sequences, in the order asked for
    o3, l3 = oracle.mla_decode(x["q_latent"], x["q_rope"], x["latent_cache"], x["rope_cache"],
                               x["seq_lens"], cfg.scale, batch_ids=[3, 0])
    assert np.array_equal(o3, o2[[3, 0]]) and np.array_equal(l3, l2[[3, 0]])


def check_gqa():
    cfg = wl.GQAConfig("wrap_gqa", 4, 8, 2, 16, 30, 0.25, seq_lens=(30, 0, 1, 17))
    x = wl.make_gqa_inputs(cfg, seed=32, poison_tail=True)
    o, l = oracle.gqa_decode(x["q"], x["k_cache"], x["v_cache"], x["seq_lens"], cfg.scale)
    o2, l2 = oracle.gqa_decode_f64(x["q"], _zero_nan(x["k_cache"]), _zero_nan(x["v_cache"]),
                                   x["seq_lens"], cfg.scale)
    assert np.array_equal(o, o2) and np.array_equal(l, l2), "gqa wrapper differs from the core"
    assert np.isfinite(o).all()


def check_multi():
    L = 4
    cfg = wl.GQAConfig("wrap_multi", 5, 8, 2, 16, 26, 0.25, seq_lens=(26, 0, 2, 11, 4))
    x = wl.make_gqa_inputs(cfg, seed=33, poison_tail=True)
    q = torch.randn((cfg.batch, L, 8, 16), generator=torch.Generator().manual_seed(34)).to(torch.bfloat16)
    k0, v0 = _zero_nan(x["k_cache"]), _zero_nan(x["v_cache"])
    for window in (0, 3):
        o, l = oracle.gqa_decode_multi(q, x["k_cache"], x["v_cache"], x["seq_lens"], cfg.scale, window)
        o2, l2 = oracle.gqa_decode_multi_f64(q, k0, v0, x["seq_lens"].numpy(), cfg.scale, window)
        assert np.array_equal(o, o2) and np.array_equal(l, l2), f"multi wrapper differs (window {window})"
        assert np.isfinite(o).all()
        # queries before the cache's start see nothing
        assert np.all(np.isneginf(l[1])) and np.all(np.isneginf(l[2, :2]))
        assert np.all(np.isfinite(l[2, 2:]))


def check_fp8():
    cfg = wl.GQAConfig("wrap_fp8", 4, 8, 2, 16, 21, 0.25, seq_lens=(21, 0, 1, 13))
    x = wl.make_gqa_inputs_fp8(cfg, seed=35, poison_tail=True)
    kc = x["k_cache"].view(torch.uint8).clone()
    vc = x["v_cache"].view(torch.uint8).clone()
    lens = x["seq_lens"]
    for b in range(cfg.batch):            # the tails carry the NaN code
        assert torch.all((kc[b, :, int(lens[b]):] & 0x7F) == 0x7F)
    k64 = oracle.e4m3_dequant(kc, x["k_scale"])
    v64 = oracle.e4m3_dequant(vc, x["v_scale"])
    k64[np.isnan(k64)] = 0
    v64[np.isnan(v64)] = 0
    o, l = oracle.gqa_decode_fp8(x["q"], x["k_cache"], x["v_cache"], lens, cfg.scale, x["k_scale"], x["v_scale"])
    o2, l2 = oracle.gqa_decode_f64(x["q"], k64, v64, lens, cfg.scale)
    assert np.array_equal(o, o2) and np.array_equal(l, l2), "fp8 wrapper differs from the core"
    assert np.isfinite(o).all()


def check_mla_fp8():
    cfg = wl.MLAConfig("wrap_mla8", 4, 6, 32, 8, 19, 0.3, seq_lens=(19, 0, 1, 11))
    x = wl.make_mla_inputs_fp8(cfg, seed=36, poison_tail=True)
    lc = x["latent_cache"].view(torch.uint8)
    rc = x["rope_cache"].view(torch.uint8)
    lens = x["seq_lens"]
    for b in range(cfg.batch):            # the tails carry the NaN code
        assert torch.all((lc[b, int(lens[b]):] & 0x7F) == 0x7F)
        assert torch.all((rc[b, int(lens[b]):] & 0x7F) == 0x7F)
    lat = oracle.e4m3_dequant(lc, x["latent_scale"])
    rope = oracle.e4m3_dequant(rc, x["rope_scale"])
    lat[np.isnan(lat)] = 0
    rope[np.isnan(rope)] = 0
    o, l = oracle.mla_decode_fp8(x["q_latent"], x["q_rope"], x["latent_cache"], x["rope_cache"], lens, cfg.scale,
                                 x["latent_scale"], x["rope_scale"])
    o2, l2 = oracle.mla_decode_f64(x["q_latent"], x["q_rope"], lat, rope, lens, cfg.scale)
    assert np.array_equal(o, o2) and np.array_equal(l, l2), "mla fp8 wrapper differs from the core"
    assert np.isfinite(o).all()
    # the two scales are not interchangeable: swapping them changes the result
    o3, _ = oracle.mla_decode_fp8(x["q_latent"], x["q_rope"], x["latent_cache"], x["rope_cache"], lens, cfg.scale,
                                  x["rope_scale"], x["latent_scale"])
    assert not np.allclose(o3, o2)


CHECKS = [check_mla, check_gqa, check_multi, check_fp8, check_mla_fp8]


@pytest.mark.parametrize("check", CHECKS, ids=lambda c: c.__name__)
def test_wrapper_equals_core(check):
    check()


@pytest.mark.parametrize("check", CHECKS, ids=lambda c: c.__name__)
def test_planted_short_slice_is_caught(check, monkeypatch):
    """Plant the off-by-one in the wrappers' row count (one row short) and require the
    check to fail."""
    real = oracle._rows
    monkeypatch.setattr(oracle, "_rows", lambda length, capacity: max(real(length, capacity) - 1, 0))
    with pytest.raises(AssertionError):
        check()
