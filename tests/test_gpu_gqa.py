"""GPU parity of kvattn_gqa_decode against the fp64 oracle (B200).

Inputs are the seeded synthetic workloads; cache positions >= seq_len are filled with
NaN so that any read of them would show.  Small shapes are compared element by
element; the four full-size GQA/MHA/MQA workloads are compared on every sequence the
oracle evaluates (all of them for these sizes) in the launch configuration the bench
uses.
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


KERNELS = {"warp": 1, "tc": 2}   # warp-level MMA kernel, tcgen05 kernel
_forced = {"kernel": 0}


@pytest.fixture(autouse=True, params=list(KERNELS), ids=list(KERNELS))
def kernel(request):
    """Every test runs once per GQA kernel (the knob forces the choice)."""
    kb.kvattn_debug_set_workers(0, 0)
    kb.kvattn_debug_set_gqa_kernel(KERNELS[request.param])
    _forced["kernel"] = KERNELS[request.param]
    kb.kvattn_clear_device_flags()
    yield request.param
    kb.kvattn_debug_set_workers(0, 0)
    kb.kvattn_debug_set_gqa_kernel(0)
    _forced["kernel"] = 0
    assert kb.kvattn_read_device_flags() == 0, "a bounded wait ran out on the device"


def decode(cfg, dev):
    """kvattn_gqa_decode; skips the test when the forced kernel cannot serve the shape
    (the tcgen05 kernel only takes head_dim 128)."""
    if _forced["kernel"] == 2 and cfg.head_dim != 128:
        pytest.skip("tcgen05 GQA kernel: head_dim 128 only")
    return kb.kvattn_gqa_decode(dev["q"], dev["k_cache"], dev["v_cache"], dev["seq_lens"], cfg.scale)


def run_case(cfg, seed=0, poison=True, batch_ids=None, inputs=None):
    x = wl.make_gqa_inputs(cfg, seed=seed, poison_tail=poison) if inputs is None else inputs
    dev = {k: v.cuda() for k, v in x.items()}
    out, lse = decode(cfg, dev)
    torch.cuda.synchronize()
    ids = list(range(cfg.batch)) if batch_ids is None else list(batch_ids)
    ro, rl = oracle.gqa_decode(x["q"], x["k_cache"], x["v_cache"], x["seq_lens"], cfg.scale,
                               batch_ids=ids)
    assert_close(out.cpu().numpy()[ids], ro, f"{cfg.name} out")
    assert_close(lse.cpu().numpy()[ids], rl, f"{cfg.name} lse")
    return out, lse


def small(name, B, n_q, n_kv, d, T, lens=None, key_scale=1.0):
    return wl.GQAConfig(name, B, n_q, n_kv, d, T, 1.0 / math.sqrt(d),
                        seq_lens=tuple(lens) if lens is not None else None, key_scale=key_scale)


GROUPS = [(1, 1), (2, 1), (4, 1), (8, 2), (16, 2), (32, 1), (8, 8), (64, 2), (48, 1)]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("n_q,n_kv", [(g * k, k) for g, k in GROUPS],
                         ids=[f"g{g}_kv{k}" for g, k in GROUPS])
def test_group_sizes(d, n_q, n_kv):
    run_case(small(f"g{n_q // n_kv}", 3, n_q, n_kv, d, 300, lens=[300, 129, 1]))


@pytest.mark.parametrize("T", [1, 2, 15, 63, 64, 65, 127, 128, 129, 1000])
def test_lengths(T):
    run_case(small(f"T{T}", 2, 16, 4, 128, T, lens=[T, max(T // 2, 1)]))


def test_ragged_with_empty_sequences():
    run_case(small("ragged", 6, 32, 8, 128, 700, lens=[0, 1, 64, 65, 700, 0]))


def test_all_empty():
    out, lse = run_case(small("empty", 2, 8, 2, 64, 128, lens=[0, 0]))
    assert torch.all(out == 0) and torch.all(torch.isneginf(lse))


def test_small_problem_one_worker_per_unit():
    """A batch small enough for one worker per unit (every unit's cache <= 128 KB): empty,
    one-token, partial-tile and full sequences in one call, each unit finished in its own
    CTA with no combine."""
    run_case(small("unit_mode", 5, 8, 2, 64, 512, lens=[512, 0, 1, 100, 0]))
    run_case(small("unit_mode128", 3, 8, 4, 128, 256, lens=[0, 256, 65]))


@pytest.mark.parametrize("which", [1, 2], ids=["warp_kernel", "tcgen05_kernel"])
def test_many_short_sequences(which):
    """1000 sequences of 0-200 tokens (group 4, head_dim 128): many pieces per worker and
    many units cut by worker boundaries, on each kernel."""
    kb.kvattn_debug_set_gqa_kernel(which)
    try:
        lens = np.random.default_rng(34 + which).integers(0, 201, size=1000).tolist()
        run_case(small("many", 1000, 32, 8, 128, 200, lens=lens))
    finally:
        kb.kvattn_debug_set_gqa_kernel(0)


@pytest.mark.parametrize("B,n_q,n_kv,T", [(2, 32, 1, 128 * 37), (3, 16, 2, 1000), (1, 64, 8, 4096)],
                         ids=["2units_37tiles", "6units_8tiles", "8units_32tiles"])
def test_equal_units_in_parts(B, n_q, n_kv, T):
    """Equal lengths and no more units than workers on the tcgen05 kernel: each unit is
    cut into consecutive parts of its own (the last one shorter), merged by the combine."""
    kb.kvattn_debug_set_gqa_kernel(2)
    try:
        run_case(small("parts", B, n_q, n_kv, 128, T))
    finally:
        kb.kvattn_debug_set_gqa_kernel(0)


def test_sharp_softmax():
    # keys scaled by 8: a few tokens dominate each head (the P-rounding worst case)
    run_case(small("sharp", 2, 16, 2, 128, 200, lens=[200, 3], key_scale=8.0))


@pytest.mark.parametrize("workers,min_tiles", [(1, 1), (2, 1), (3, 1), (7, 1), (64, 1), (500, 1)])
def test_forced_splits(workers, min_tiles):
    """Force the worker count so that units are cut at many places and the combine
    merges up to hundreds of partials (empty sequences included)."""
    kb.kvattn_debug_set_workers(workers, min_tiles)
    run_case(small("split", 5, 32, 4, 128, 2000, lens=[2000, 1, 0, 777, 1500]))
    run_case(small("split64", 3, 8, 2, 64, 900, lens=[900, 64, 65]))


def test_repeat_invariance():
    """Result with n_kv < n_q equals the result with n_kv = n_q on the repeat-interleaved
    cache (the same kernel, other plan), up to the tolerance."""
    cfg = small("rep", 2, 16, 2, 128, 500, lens=[500, 77])
    x = wl.make_gqa_inputs(cfg, seed=5)
    d = {k: v.cuda() for k, v in x.items()}
    o1, l1 = decode(cfg, d)
    d2 = dict(d)
    d2["k_cache"] = d["k_cache"].repeat_interleave(8, dim=1).contiguous()
    d2["v_cache"] = d["v_cache"].repeat_interleave(8, dim=1).contiguous()
    o2, l2 = decode(cfg, d2)
    assert_close(o1.cpu().numpy(), o2.cpu().numpy().astype(np.float64), "repeat out")
    assert_close(l1.cpu().numpy(), l2.cpu().numpy().astype(np.float64), "repeat lse")


def test_nonzero_stream_and_reuse():
    cfg = small("stream", 4, 32, 8, 128, 1024)
    x = wl.make_gqa_inputs(cfg, seed=7)
    d = {k: v.cuda() for k, v in x.items()}
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        outs = [kb.kvattn_gqa_decode(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], cfg.scale,
                                     stream=s) for _ in range(3)]
        if _forced["kernel"] == 2:
            assert cfg.head_dim == 128
    s.synchronize()
    for o, l in outs[1:]:
        assert torch.equal(o, outs[0][0]) and torch.equal(l, outs[0][1])


@pytest.mark.parametrize("name", [n for n in wl.CONFIG_ORDER if isinstance(wl.CONFIGS[n], wl.GQAConfig)])
def test_workload_full_size(name):
    """The GQA/MHA/MQA workloads at full size, every sequence, bench launch configuration."""
    run_case(wl.CONFIGS[name], poison=True)


@pytest.mark.parametrize("direction", [1.0, -1.0], ids=["rising", "falling"])
def test_running_max_moves(direction):
    """Scores that ramp steeply along the sequence (about 20 in log2 units per 128
    tokens): with a rising ramp every tile raises every head's running max by far more
    than the rescale threshold, so O and the row sums are rescaled on most tiles; with a
    falling ramp the first tile holds the max and later weights underflow to zero."""
    cfg = small("ramp", 2, 32, 2, 128, 1500, lens=[1500, 700])
    g = torch.Generator().manual_seed(3)
    B, n_q, n_kv, d, T = cfg.batch, cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim, cfg.max_seq_len
    q = (0.5 + 0.1 * torch.randn(B, n_q, d, generator=g)).to(torch.bfloat16)
    t = torch.arange(T, dtype=torch.float32).view(1, 1, T, 1)
    ramp = 0.019 * (t if direction > 0 else (T - 1 - t))
    k = (ramp + 0.3 * torch.randn(B, n_kv, T, d, generator=g)).to(torch.bfloat16)
    v = torch.randn(B, n_kv, T, d, generator=g).to(torch.bfloat16)
    lens = torch.tensor(cfg.seq_lens, dtype=torch.int32)
    for b in range(B):
        k[b, :, lens[b]:] = float("nan")
        v[b, :, lens[b]:] = float("nan")
    run_case(cfg, inputs={"q": q, "k_cache": k, "v_cache": v, "seq_lens": lens})
