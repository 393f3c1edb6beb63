"""The oracle's multi-token MLA (oracle.mla_decode_multi), pinned to a different core
(CPU only).

Absorbed MLA scores head h at token t as q_lat . c_t + q_rope . r_t and returns the
weighted sum of the latents c_t; that is GQA with one KV head of width d_c + d_r whose key
is [c_t, r_t] and whose value is [c_t, 0], the query being [q_lat, q_rope].  So with the
causal mask the MLA multi-token result must equal the multi-token GQA core
(oracle.gqa_decode_multi_f64, itself pinned to PyTorch SDPA with an explicit mask) on
those concatenations, the output's first d_c columns.  Lengths cover sequences shorter than
the number of new tokens (queries that see nothing) and the full capacity.  A planted
off-by-one in the causal row count must be caught, and one new token must reduce to the
single-token MLA oracle.
"""
import numpy as np
import pytest
import torch

import oracle


def _case(seed=3, B=4, L=3, H=5, dc=24, dr=8, T=17, lens=(17, 0, 2, 9)):
    g = torch.Generator().manual_seed(seed)
    ql = torch.randn((B, L, H, dc), generator=g).to(torch.bfloat16)
    qr = torch.randn((B, L, H, dr), generator=g).to(torch.bfloat16)
    lat = torch.randn((B, T, dc), generator=g).to(torch.bfloat16)
    rope = torch.randn((B, T, dr), generator=g).to(torch.bfloat16)
    return ql, qr, lat, rope, torch.tensor(lens, dtype=torch.int32), 0.3


def _as_gqa(ql, qr, lat, rope):
    q = torch.cat([ql.double(), qr.double()], dim=-1)                         # [B, L, H, dc + dr]
    k = torch.cat([lat.double(), rope.double()], dim=-1)[:, None]             # [B, 1, T, dc + dr]
    v = torch.cat([lat.double(), torch.zeros_like(rope.double())], dim=-1)[:, None]
    return q.numpy(), k.numpy(), v.numpy()


def check_against_gqa():
    ql, qr, lat, rope, lens, scale = _case()
    o, l = oracle.mla_decode_multi(ql, qr, lat, rope, lens, scale)
    q, k, v = _as_gqa(ql, qr, lat, rope)
    og, lg = oracle.gqa_decode_multi_f64(q, k, v, lens.numpy(), scale)
    dc = ql.shape[-1]
    assert np.allclose(o, og[..., :dc], rtol=1e-12, atol=1e-12), "mla multi differs from the GQA core"
    assert np.array_equal(np.isinf(l), np.isinf(lg)) and np.allclose(l[np.isfinite(l)], lg[np.isfinite(lg)],
                                                                       rtol=1e-12, atol=1e-12)
    # sequence 1 (length 0) sees nothing; sequence 2 (length 2): its first new token nothing
    assert np.all(np.isneginf(l[1])) and np.all(np.isneginf(l[2, 0])) and np.all(np.isfinite(l[2, 1:]))


def test_multi_equals_gqa_core():
    check_against_gqa()


def test_one_token_is_single_token_oracle():
    ql, qr, lat, rope, lens, scale = _case(seed=4, L=1)
    o, l = oracle.mla_decode_multi(ql, qr, lat, rope, lens, scale)
    o1, l1 = oracle.mla_decode(ql[:, 0], qr[:, 0], lat, rope, lens, scale)
    assert np.array_equal(o[:, 0], o1) and np.array_equal(l[:, 0], l1)


def test_planted_causal_off_by_one_is_caught(monkeypatch):
    real = oracle._causal_rows
    monkeypatch.setattr(oracle, "_causal_rows", lambda n, L, i, cap: max(real(n, L, i, cap) - 1, 0))
    with pytest.raises(AssertionError):
        check_against_gqa()
