"""Checks that pin the oracle to facts other than itself.

Each check takes the oracle library handle (so the same check can be run against a
build with a planted mistake) and raises AssertionError on failure.  None of them
retypes the oracle's formula: they use values the pages print, closed forms,
invariants, library routines the pages name (PyTorch's scaled_dot_product_attention
with enable_gqa, as in "Attention variants: MQA, GQA, and MLA", section "Against the
real libraries") and brute force in pure Python on tiny inputs.
"""
import math

import numpy as np
import torch
import torch.nn.functional as F

import oracle


def _rng(seed):
    return np.random.default_rng(seed)


def _gqa_case(seed, B=2, n_q=8, n_kv=2, d=16, T=13, lens=None):
    r = _rng(seed)
    q = r.standard_normal((B, n_q, d))
    k = r.standard_normal((B, n_kv, T, d))
    v = r.standard_normal((B, n_kv, T, d))
    if lens is None:
        lens = r.integers(1, T + 1, size=B)
    return q, k, v, np.asarray(lens, dtype=np.int32)


# --------------------------------------------------------------------------------------
# Group indexing: GQA equals MHA run on repeat_interleave'd K/V ("Attention variants:
# MQA, GQA, and MLA", "Implementation, twice"; "KV cache variants: MHA, GQA, MLA",
# "MHA vs GQA when group_size = 1").  The oracle treats every head independently with
# the same arithmetic, so the two must agree bit for bit.
# --------------------------------------------------------------------------------------
def pin_gqa_equals_mha_on_repeated_kv(lib):
    for seed, (n_q, n_kv) in enumerate([(8, 2), (8, 4), (8, 1), (6, 3), (12, 4)]):
        q, k, v, lens = _gqa_case(100 + seed, n_q=n_q, n_kv=n_kv)
        g = n_q // n_kv
        o1, l1 = oracle.gqa_decode_f64(q, k, v, lens, 0.3, lib=lib)
        o2, l2 = oracle.gqa_decode_f64(q, np.repeat(k, g, axis=1), np.repeat(v, g, axis=1),
                                       lens, 0.3, lib=lib)
        assert np.array_equal(o1, o2) and np.array_equal(l1, l2), (n_q, n_kv)


# --------------------------------------------------------------------------------------
# Library cross-check: PyTorch SDPA with enable_gqa=True in fp64 on the CPU, atol 1e-12,
# the check the pages run ("Against the real libraries").  Decode = one query token,
# no causal mask; positions >= seq_len are masked out.  The log-sum-exp is read off the
# same routine by appending one extra token whose score is exactly 0 and whose value is
# a one-hot in an extra dimension: its output weight is 1 / (1 + exp(lse)).
# --------------------------------------------------------------------------------------
def _sdpa_reference(q, k, v, lens, scale):
    B, n_q, d = q.shape
    n_kv, T = k.shape[1], k.shape[2]
    qt = torch.from_numpy(q).reshape(B, n_q, 1, d)
    kt = torch.from_numpy(k)
    vt = torch.from_numpy(v)
    # extra token: zero key (score exactly 0), value one-hot in an extra dimension
    k_ext = torch.cat([kt, torch.zeros(B, n_kv, 1, d, dtype=torch.float64)], dim=2)
    v_pad = torch.cat([vt, torch.zeros(B, n_kv, T, 1, dtype=torch.float64)], dim=3)
    extra = torch.zeros(B, n_kv, 1, d + 1, dtype=torch.float64)
    extra[..., d] = 1.0
    v_ext = torch.cat([v_pad, extra], dim=2)
    pos = torch.arange(T + 1)
    mask = (pos[None, :] < torch.from_numpy(lens.astype(np.int64))[:, None]) | (pos[None, :] == T)
    mask = mask[:, None, None, :]
    plain = F.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask[..., :T], scale=scale,
                                           enable_gqa=True)
    ext = F.scaled_dot_product_attention(qt, k_ext, v_ext, attn_mask=mask, scale=scale,
                                         enable_gqa=True)
    w0 = ext[..., 0, d]
    lse = torch.log((1.0 - w0) / w0)
    return plain[:, :, 0, :].numpy(), lse.numpy()


def pin_sdpa_enable_gqa(lib):
    for seed, (n_q, n_kv, d, T) in enumerate([(8, 2, 32, 64), (4, 4, 8, 5), (16, 1, 16, 40),
                                              (6, 2, 64, 17)]):
        q, k, v, lens = _gqa_case(200 + seed, B=3, n_q=n_q, n_kv=n_kv, d=d, T=T)
        scale = 1.0 / math.sqrt(d)
        o, l = oracle.gqa_decode_f64(q, k, v, lens, scale, lib=lib)
        o_ref, l_ref = _sdpa_reference(q, k, v, lens, scale)
        assert np.allclose(o, o_ref, rtol=0, atol=1e-12), np.abs(o - o_ref).max()
        assert np.allclose(l, l_ref, rtol=0, atol=1e-10), np.abs(l - l_ref).max()


# --------------------------------------------------------------------------------------
# Closed forms of the softmax-weighted sum.
# --------------------------------------------------------------------------------------
def pin_closed_forms(lib):
    r = _rng(300)
    d = 8
    # T = 1: the only weight is 1, so out = v_0 and lse = s_0 = scale * q . k_0
    q = r.standard_normal((1, 2, d)); k = r.standard_normal((1, 1, 1, d))
    v = r.standard_normal((1, 1, 1, d))
    o, l = oracle.gqa_decode_f64(q, k, v, [1], 0.5, lib=lib)
    assert np.allclose(o[0], v[0, 0, 0][None, :], atol=1e-15)
    assert np.allclose(l[0], 0.5 * (q[0] @ k[0, 0, 0]), atol=1e-14)
    # identical keys: uniform weights, out = mean of the values, lse = s + ln T
    T = 7
    k = np.repeat(r.standard_normal((1, 1, 1, d)), T, axis=2)
    v = r.standard_normal((1, 1, T, d))
    o, l = oracle.gqa_decode_f64(q, k, v, [T], 0.25, lib=lib)
    assert np.allclose(o[0], v[0, 0].mean(axis=0)[None, :], atol=1e-14)
    assert np.allclose(l[0], 0.25 * (q[0] @ k[0, 0, 0]) + math.log(T), atol=1e-13)
    # T = 2: weight of token 0 is the logistic function of s_0 - s_1, lse = logaddexp
    k = r.standard_normal((1, 1, 2, d)); v = r.standard_normal((1, 1, 2, d))
    o, l = oracle.gqa_decode_f64(q, k, v, [2], 0.7, lib=lib)
    for h in range(2):
        s0, s1 = 0.7 * q[0, h] @ k[0, 0, 0], 0.7 * q[0, h] @ k[0, 0, 1]
        w0 = 1.0 / (1.0 + math.exp(s1 - s0))
        assert np.allclose(o[0, h], w0 * v[0, 0, 0] + (1 - w0) * v[0, 0, 1], atol=1e-14)
        assert abs(l[0, h] - np.logaddexp(s0, s1)) < 1e-13


def pin_empty_sequence(lib):
    q, k, v, _ = _gqa_case(310, B=2, T=4)
    o, l = oracle.gqa_decode_f64(q, k, v, [0, 3], 1.0, lib=lib)
    assert np.all(o[0] == 0.0) and np.all(np.isneginf(l[0]))
    assert np.all(np.isfinite(l[1]))


# --------------------------------------------------------------------------------------
# Brute force in pure Python on tiny inputs (B=1, n_q=2, n_kv=1, d=2, T<=3 and a few
# more): a direct evaluation of softmax(q K^T * scale) V with math.exp, no arrays.
# --------------------------------------------------------------------------------------
def _brute(q, k, v, lens, scale):
    B, n_q, d = len(q), len(q[0]), len(q[0][0])
    n_kv = len(k[0])
    out = [[[0.0] * d for _ in range(n_q)] for _ in range(B)]
    lse = [[0.0] * n_q for _ in range(B)]
    for b in range(B):
        for h in range(n_q):
            j = h * n_kv // n_q          # the pages' ceil(i * g / h) with 1-based i
            ws = []
            for t in range(lens[b]):
                s = scale * sum(q[b][h][i] * k[b][j][t][i] for i in range(d))
                ws.append(math.exp(s))
            z = sum(ws)
            lse[b][h] = math.log(z) if z > 0 else -math.inf
            for t in range(lens[b]):
                for i in range(d):
                    out[b][h][i] += ws[t] / z * v[b][j][t][i]
    return np.array(out), np.array(lse)


def pin_brute_force_tiny(lib):
    shapes = [(1, 2, 1, 2, 1), (1, 2, 1, 2, 2), (1, 2, 1, 2, 3), (2, 4, 2, 3, 3),
              (1, 6, 3, 2, 3), (2, 3, 3, 1, 2)]
    for i, (B, n_q, n_kv, d, T) in enumerate(shapes):
        q, k, v, lens = _gqa_case(400 + i, B=B, n_q=n_q, n_kv=n_kv, d=d, T=T)
        o, l = oracle.gqa_decode_f64(q, k, v, lens, 0.9, lib=lib)
        ob, lb = _brute(q.tolist(), k.tolist(), v.tolist(), lens.tolist(), 0.9)
        assert np.allclose(o, ob, atol=1e-13), (i, np.abs(o - ob).max())
        assert np.allclose(l, lb, atol=1e-13), (i, np.abs(l - lb).max())


# --------------------------------------------------------------------------------------
# Invariants.
# --------------------------------------------------------------------------------------
def pin_split_merge(lib):
    """Attention over [0,T) equals the log-sum-exp merge of attention over any partition
    of [0,T) into parts (empty parts included, lse = -inf, weight 0).  This is the
    identity the split-KV combine relies on."""
    q, k, v, _ = _gqa_case(500, B=1, n_q=4, n_kv=2, d=8, T=23)
    T = 23
    whole_o, whole_l = oracle.gqa_decode_f64(q, k, v, [T], 0.4, lib=lib)
    for cuts in ([0, 5, 5, 17, 23], [0, 1, 2, 3, 23], [0, 23], [0, 11, 23, 23]):
        parts = []
        for a, b in zip(cuts[:-1], cuts[1:]):
            ko = np.ascontiguousarray(k[:, :, a:b]); vo = np.ascontiguousarray(v[:, :, a:b])
            if b == a:
                ko = np.zeros((1, 2, 1, 8)); vo = np.zeros((1, 2, 1, 8))
            parts.append(oracle.gqa_decode_f64(q, ko, vo, [b - a], 0.4, lib=lib))
        lses = np.stack([p[1] for p in parts])          # [P, 1, n_q]
        m = lses.max(axis=0)
        total = m + np.log(np.exp(lses - m).sum(axis=0))
        merged = sum(np.exp(p[1] - total)[..., None] * p[0] for p in parts)
        assert np.allclose(total, whole_l, atol=1e-13)
        assert np.allclose(merged, whole_o, atol=1e-13)


def pin_permutation_invariance(lib):
    q, k, v, _ = _gqa_case(600, B=1, n_q=4, n_kv=2, d=8, T=19)
    perm = _rng(601).permutation(19)
    o1, l1 = oracle.gqa_decode_f64(q, k, v, [19], 0.6, lib=lib)
    o2, l2 = oracle.gqa_decode_f64(q, k[:, :, perm], v[:, :, perm], [19], 0.6, lib=lib)
    assert np.allclose(o1, o2, atol=1e-14) and np.allclose(l1, l2, atol=1e-13)


def pin_scale_equivariance(lib):
    """Multiplying q by a and the scale by 1/a leaves every score, hence the result, unchanged."""
    q, k, v, lens = _gqa_case(700)
    o1, l1 = oracle.gqa_decode_f64(q, k, v, lens, 0.5, lib=lib)
    o2, l2 = oracle.gqa_decode_f64(4.0 * q, k, v, lens, 0.125, lib=lib)
    assert np.allclose(o1, o2, atol=1e-14) and np.allclose(l1, l2, atol=1e-13)


# --------------------------------------------------------------------------------------
# MLA.
# --------------------------------------------------------------------------------------
def pin_mla_absorbed_equals_explicit(lib):
    """Absorbed MLA equals MLA with explicit per-head up-projections ("Attention
    variants: MQA, GQA, and MLA", section "MLA: cache a latent, not the keys and values",
    the score identity q.(c W_UK) = (q W_UK^T).c and the output identity
    sum_s w_s c_s W_UV = (sum_s w_s c_s) W_UV).  The explicit path below reconstructs
    per-head keys and values from the latents and never forms q W_UK^T."""
    r = _rng(800)
    H, d_c, d_h, d_r, T = 4, 24, 8, 6, 11
    W_uk = r.standard_normal((H, d_c, d_h)) / math.sqrt(d_c)
    W_uv = r.standard_normal((H, d_c, d_h)) / math.sqrt(d_c)
    q_head = r.standard_normal((H, d_h))
    q_rope = r.standard_normal((H, d_r))
    c = r.standard_normal((T, d_c))
    rr = r.standard_normal((T, d_r))
    scale = 1.0 / math.sqrt(d_h + d_r)
    # explicit: per-head K and V from the latents, RoPE key appended to K
    explicit = np.zeros((H, d_h))
    for h in range(H):
        k_h = np.concatenate([c @ W_uk[h], rr], axis=1)          # [T, d_h + d_r]
        v_h = c @ W_uv[h]                                        # [T, d_h]
        qh = np.concatenate([q_head[h], q_rope[h]])
        ref = F.scaled_dot_product_attention(torch.from_numpy(qh)[None, None, None],
                                             torch.from_numpy(k_h)[None, None],
                                             torch.from_numpy(v_h)[None, None], scale=scale)
        explicit[h] = ref[0, 0, 0].numpy()
    # absorbed: q_lat = W_UK q, attend over latents, then apply W_UV
    q_lat = np.einsum("hcd,hd->hc", W_uk, q_head)
    o_lat, _ = oracle.mla_decode_f64(q_lat[None], q_rope[None], c[None], rr[None], [T], scale,
                                     lib=lib)
    absorbed = np.einsum("hc,hcd->hd", o_lat[0], W_uv)
    assert np.allclose(absorbed, explicit, atol=1e-12), np.abs(absorbed - explicit).max()


def pin_mla_matches_sdpa(lib):
    """MLA is MQA whose key is [c || r] and whose value is c (the same latent): checked
    against SDPA with one KV head (values narrower than keys), fp64, atol 1e-12."""
    r = _rng(810)
    B, H, d_c, d_r, T = 2, 6, 16, 4, 9
    ql = r.standard_normal((B, H, d_c)); qr = r.standard_normal((B, H, d_r))
    c = r.standard_normal((B, T, d_c)); rr = r.standard_normal((B, T, d_r))
    lens = np.array([9, 4], dtype=np.int32)
    scale = 0.2
    o, _ = oracle.mla_decode_f64(ql, qr, c, rr, lens, scale, lib=lib)
    for b in range(B):
        L = int(lens[b])
        qfull = torch.from_numpy(np.concatenate([ql[b], qr[b]], axis=1))[None, :, None, :]
        kfull = torch.from_numpy(np.concatenate([c[b, :L], rr[b, :L]], axis=1))[None, None]
        val = torch.from_numpy(c[b, :L])[None, None]
        ref = F.scaled_dot_product_attention(qfull, kfull, val, scale=scale, enable_gqa=True)
        assert np.allclose(o[b], ref[0, :, 0].numpy(), atol=1e-12)


def pin_mla_without_rope_is_mqa(lib):
    """With no RoPE part, absorbed MLA is MQA with K = V = latent (one shared KV head)."""
    r = _rng(820)
    B, H, d_c, T = 2, 4, 12, 10
    ql = r.standard_normal((B, H, d_c)); c = r.standard_normal((B, T, d_c))
    lens = np.array([10, 6], dtype=np.int32)
    o1, l1 = oracle.mla_decode_f64(ql, np.zeros((B, H, 0)), c, np.zeros((B, T, 0)), lens, 0.3,
                                   lib=lib)
    o2, l2 = oracle.gqa_decode_f64(ql, c[:, None], c[:, None], lens, 0.3, lib=lib)
    assert np.allclose(o1, o2, atol=1e-14) and np.allclose(l1, l2, atol=1e-13)


# --------------------------------------------------------------------------------------
# Rotary position embedding (the textbook rotation of feature pairs; the pages name RoPE
# without its formula).  Pinned to mathematics, not to a retyped formula: position 0 is
# the identity, the angles of tiny cases are worked by hand (d = 2: one pair turning by
# p radians when base is anything, d = 4: the second pair turns by p / sqrt(base)),
# rotations keep every pair's length and compose (p then p' equals p + p'), the score
# of a rotated query and key depends only on the positions' difference, and the two
# pair layouts differ by a fixed permutation of the features.
# --------------------------------------------------------------------------------------
def pin_rope_identity_and_hand_cases(lib):
    r = _rng(31)
    x = r.standard_normal((5, 8))
    for inter in (0, 1):
        assert np.array_equal(oracle.rope_f64(x, np.zeros(5, np.int32), 10000.0, inter, lib=lib), x)
    # d = 2: (1, 0) at position p -> (cos p, sin p); (0, 1) -> (-sin p, cos p)
    for p in (1, 2, 7):
        y = oracle.rope_f64(np.array([[1.0, 0.0], [0.0, 1.0]]), [p, p], 10000.0, 1, lib=lib)
        assert np.allclose(y, [[math.cos(p), math.sin(p)], [-math.sin(p), math.cos(p)]], atol=1e-15), p
    # d = 4, base 100: pair 0 turns by p, pair 1 by p / 10
    p = 3
    y = oracle.rope_f64(np.array([[0.0, 0.0, 1.0, 0.0]]), [p], 100.0, 1, lib=lib)
    assert np.allclose(y, [[0.0, 0.0, math.cos(0.3), math.sin(0.3)]], atol=1e-15)
    y = oracle.rope_f64(np.array([[0.0, 1.0, 0.0, 0.0]]), [p], 100.0, 0, lib=lib)   # halves: pair 1 = (1, 3)
    assert np.allclose(y, [[0.0, math.cos(0.3), 0.0, math.sin(0.3)]], atol=1e-15)


def pin_rope_invariants(lib):
    r = _rng(32)
    d = 16
    x = r.standard_normal((6, d))
    pos = np.array([0, 1, 5, 100, 4095, 32767], np.int32)
    for inter in (0, 1):
        y = oracle.rope_f64(x, pos, 10000.0, inter, lib=lib)
        pairs = (lambda z: np.stack([z[:, 0::2], z[:, 1::2]], -1)) if inter else \
                (lambda z: np.stack([z[:, : d // 2], z[:, d // 2:]], -1))
        assert np.allclose(np.linalg.norm(pairs(y), axis=-1), np.linalg.norm(pairs(x), axis=-1), atol=1e-12)
        # composition
        a, b = np.array([3] * 6, np.int32), np.array([11] * 6, np.int32)
        twice = oracle.rope_f64(oracle.rope_f64(x, a, 10000.0, inter, lib=lib), b, 10000.0, inter, lib=lib)
        assert np.allclose(twice, oracle.rope_f64(x, a + b, 10000.0, inter, lib=lib), atol=1e-12)
        # relative position: <R_m q, R_n k> == <R_{m-n} q, k>
        q, k = r.standard_normal(d), r.standard_normal(d)
        for m, n in [(7, 2), (300, 299), (1000, 10)]:
            lhs = oracle.rope_f64(q[None], [m], 10000.0, inter, lib=lib)[0] @ \
                oracle.rope_f64(k[None], [n], 10000.0, inter, lib=lib)[0]
            rhs = oracle.rope_f64(q[None], [m - n], 10000.0, inter, lib=lib)[0] @ k
            assert abs(lhs - rhs) < 1e-9 * (1 + abs(rhs)), (m, n)
    # layouts: interleaved == halves under the permutation that interleaves the halves
    perm = np.empty(d, dtype=np.int64)
    perm[0::2] = np.arange(d // 2)
    perm[1::2] = np.arange(d // 2) + d // 2
    yi = oracle.rope_f64(x[:, perm], pos, 10000.0, 1, lib=lib)
    yh = oracle.rope_f64(x, pos, 10000.0, 0, lib=lib)
    assert np.allclose(yi, yh[:, perm], atol=1e-12)


# --------------------------------------------------------------------------------------
# Several new tokens per sequence with the causal mask ("Attention variants: MQA, GQA,
# and MLA", "Implementation, twice") and an optional sliding window.  Pinned to PyTorch
# SDPA in fp64 with an explicit boolean mask (the library routine the pages use), to
# the single-token routine on each query's visible slice, and to closed forms: a
# window of one token returns that token's value; a query before the cache's start
# sees nothing.
# --------------------------------------------------------------------------------------
def _multi_case(seed, B=3, L=4, n_q=8, n_kv=2, d=16, T=20):
    r = _rng(seed)
    q = r.standard_normal((B, L, n_q, d))
    k = r.standard_normal((B, n_kv, T, d))
    v = r.standard_normal((B, n_kv, T, d))
    return q, k, v


def pin_multi_token_sdpa(lib):
    q, k, v = _multi_case(41)
    B, L, n_q, d = q.shape
    n_kv, T = k.shape[1], k.shape[2]
    lens = np.array([20, 9, 4], np.int32)
    for window in (0, 1, 3, 6, 50):
        out, lse = oracle.gqa_decode_multi_f64(q, k, v, lens, 0.37, window=window, lib=lib)
        for b in range(B):
            n = int(lens[b])
            qt = torch.from_numpy(q[b]).permute(1, 0, 2)[None]              # [1, n_q, L, d]
            kt = torch.from_numpy(k[b, :, :n])[None]
            vt = torch.from_numpy(v[b, :, :n])[None]
            pos = torch.arange(n - L, n)[:, None]
            t = torch.arange(n)[None, :]
            vis = t <= pos
            if window > 0:
                vis &= t > pos - window
            ref = F.scaled_dot_product_attention(qt, kt, vt, attn_mask=vis, scale=0.37, enable_gqa=True)
            assert np.allclose(out[b], ref[0].permute(1, 0, 2).numpy(), atol=1e-12), (b, window)
            s = torch.einsum("hld,htd->hlt", qt[0], kt[0].repeat_interleave(n_q // n_kv, 0)) * 0.37
            s = s.masked_fill(~vis[None], float("-inf"))
            assert np.allclose(lse[b], torch.logsumexp(s, -1).permute(1, 0).numpy(), atol=1e-12), (b, window)


def pin_multi_token_reductions(lib):
    q, k, v = _multi_case(42, B=2, L=3)
    lens = np.array([11, 6], np.int32)
    L, n_q = q.shape[1], q.shape[2]
    g = n_q // k.shape[1]
    for window in (0, 4):
        out, lse = oracle.gqa_decode_multi_f64(q, k, v, lens, 0.5, window=window, lib=lib)
        for b in range(2):
            for i in range(L):
                pos = int(lens[b]) - L + i
                lo = max(0, pos + 1 - window) if window else 0
                # each query equals the single-token routine over its visible slice
                o1, l1 = oracle.gqa_decode_f64(q[b:b + 1, i], k[b:b + 1, :, lo:pos + 1], v[b:b + 1, :, lo:pos + 1],
                                               np.array([pos + 1 - lo], np.int32), 0.5, lib=lib)
                assert np.allclose(out[b, i], o1[0], atol=1e-14) and np.allclose(lse[b, i], l1[0], atol=1e-13)
    # window 1: the query sees only its own token
    out, lse = oracle.gqa_decode_multi_f64(q, k, v, lens, 0.5, window=1, lib=lib)
    for b in range(2):
        for i in range(L):
            pos = int(lens[b]) - L + i
            for h in range(n_q):
                assert np.allclose(out[b, i, h], v[b, h // g, pos], atol=1e-15)
                assert abs(lse[b, i, h] - 0.5 * q[b, i, h] @ k[b, h // g, pos]) < 1e-12
    # queries before the cache's first position see nothing
    out, lse = oracle.gqa_decode_multi_f64(q, k, v, np.array([2, 0], np.int32), 0.5, lib=lib)
    assert np.all(np.isneginf(lse[0, 0])) and np.all(out[0, 0] == 0) and np.all(np.isfinite(lse[0, 1:]))
    assert np.all(np.isneginf(lse[1])) and np.all(out[1] == 0)


# --------------------------------------------------------------------------------------
# Quantised (fp8) cache ("Attention variants: MQA, GQA, and MLA", section "Against the
# real libraries": quantised caches).  The codes follow the E4M3 format's definition:
# hand-worked values, every code against PyTorch's float8_e4m3fn conversion, the
# encoder's ties and saturation by hand, and the fp8 decode equal to the (separately
# pinned) decode over caches dequantised by PyTorch.
# --------------------------------------------------------------------------------------
E4M3_BY_HAND = {
    0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x0F: 1.875 * 2.0 ** -6,
    0x30: 0.5, 0x38: 1.0, 0x39: 1.125, 0x3F: 1.875, 0x40: 2.0, 0x78: 256.0, 0x7E: 448.0,
    0x80: -0.0, 0xB8: -1.0, 0xFE: -448.0,
}


def pin_e4m3_codes(lib):
    for c, v in E4M3_BY_HAND.items():
        got = oracle.e4m3_value(c, lib=lib)
        assert got == v and math.copysign(1.0, got) == math.copysign(1.0, v), (hex(c), got, v)
    assert math.isnan(oracle.e4m3_value(0x7F, lib=lib)) and math.isnan(oracle.e4m3_value(0xFF, lib=lib))
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = oracle.e4m3_dequant(codes, 1.0, lib=lib)
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert same.all(), np.nonzero(~same)


def pin_e4m3_encoder(lib):
    finite = [c for c in range(256) if c not in (0x7F, 0xFF)]
    # every finite value encodes to its own code
    vals = np.array([oracle.e4m3_value(c, lib=lib) for c in finite], np.float32)
    assert (oracle.e4m3_quant(vals, 1.0, lib=lib) == np.array(finite, np.uint8)).all()
    # midpoints between neighbours go to the even code; saturation; NaN
    hand = {1.0625: 0x38, 1.1875: 0x3A, 3 * 2.0 ** -10: 0x02, 2.0 ** -10: 0x00, 1.5 * 2.0 ** -9: 0x02,
            440.0: 0x7E, 448.0: 0x7E, 449.0: 0x7E, 1e30: 0x7E, -1e30: 0xFE, -1.0625: 0xB8, 17.0: 0x58, 19.0: 0x5A}
    for x, c in hand.items():
        got = int(oracle.e4m3_quant(np.array([x], np.float32), 1.0, lib=lib)[0])
        assert got == c, (x, hex(got), hex(c))
    assert int(oracle.e4m3_quant(np.array([np.nan], np.float32), 1.0, lib=lib)[0]) == 0x7F
    # in range, against PyTorch's round-to-nearest-even conversion
    x = torch.from_numpy(_rng(51).standard_normal(20000).astype(np.float32) * 60.0)
    x = x[x.abs() < 448]
    assert (oracle.e4m3_quant(x, 1.0, lib=lib) == x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()).all()
    # the division by the scale is taken in float
    s = np.float32(0.0371)
    y = (x.numpy() / s).astype(np.float32)
    y = np.clip(y, -447, 447)
    xs = (torch.from_numpy(y) * torch.tensor(float(s))).numpy()
    want = torch.from_numpy((xs / s).astype(np.float32)).clamp(-448, 448).to(torch.float8_e4m3fn)
    assert (oracle.e4m3_quant(xs, s, lib=lib) == want.view(torch.uint8).numpy()).all()


def _fp8_case(seed, B=2, n_q=8, n_kv=2, d=16, T=15):
    r = _rng(seed)
    q = r.standard_normal((B, n_q, d))
    codes = r.integers(0, 256, size=(2, B, n_kv, T, d), dtype=np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x3C      # no NaN codes
    return q, codes[0], codes[1]


def _torch_dequant(codes, s):
    return torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy() * s


def pin_fp8_decode_on_dequantised_cache(lib):
    q, kc, vc = _fp8_case(52)
    lens = np.array([15, 6], np.int32)
    for ks, vs in ((0.125, 4.0), (0.0371, 0.0213), (1.0, 1.0)):
        out, lse = oracle.gqa_decode_fp8(q, kc, vc, lens, 0.3, ks, vs, lib=lib)
        ro, rl = oracle.gqa_decode_f64(q, _torch_dequant(kc, ks), _torch_dequant(vc, vs), lens, 0.3, lib=lib)
        assert np.allclose(out, ro, rtol=1e-13, atol=1e-13) and np.allclose(lse, rl, rtol=1e-13, atol=1e-13), (ks, vs)
    # the value scale scales the output and leaves lse alone; the key scale is a score scale
    o1, l1 = oracle.gqa_decode_fp8(q, kc, vc, lens, 0.3, 0.5, 1.0, lib=lib)
    o2, l2 = oracle.gqa_decode_fp8(q, kc, vc, lens, 0.3, 0.5, 8.0, lib=lib)
    assert np.allclose(o2, 8.0 * o1, rtol=1e-13, atol=1e-13) and np.array_equal(l1, l2)
    o3, l3 = oracle.gqa_decode_fp8(q, kc, vc, lens, 0.15, 1.0, 1.0, lib=lib)
    assert np.allclose(o1, o3, rtol=1e-13, atol=1e-13) and np.allclose(l1, l3, rtol=1e-13, atol=1e-13)
    # several new tokens: the multi-token oracle on the dequantised cache
    r = _rng(53)
    qm = r.standard_normal((2, 3, 8, 16))
    out, lse = oracle.gqa_decode_fp8(qm, kc, vc, lens, 0.3, 0.25, 2.0, window=4, lib=lib)
    ro, rl = oracle.gqa_decode_multi_f64(qm, _torch_dequant(kc, 0.25), _torch_dequant(vc, 2.0), lens, 0.3,
                                         window=4, lib=lib)
    assert np.allclose(out, ro, atol=1e-13) and np.allclose(lse, rl, atol=1e-13)


ALL_PINS = [
    pin_gqa_equals_mha_on_repeated_kv, pin_sdpa_enable_gqa, pin_closed_forms,
    pin_empty_sequence, pin_brute_force_tiny, pin_split_merge, pin_permutation_invariance,
    pin_scale_equivariance, pin_mla_absorbed_equals_explicit, pin_mla_matches_sdpa,
    pin_mla_without_rope_is_mqa, pin_rope_identity_and_hand_cases, pin_rope_invariants,
    pin_multi_token_sdpa, pin_multi_token_reductions, pin_e4m3_codes, pin_e4m3_encoder,
    pin_fp8_decode_on_dequantised_cache,
]
