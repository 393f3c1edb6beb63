"""The benchmark's algorithmic byte and flop counts for the workload variants (CPU only):
the rows a windowed step must read and the (query, row) pairs it attends, against brute
force over the visibility rule; and the per-step byte counts, against hand-worked
values."""
import importlib
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from mla_kv_cache_b200 import workloads as wl  # noqa: E402


@pytest.fixture()
def bench():
    import bench as b
    b = importlib.reload(b)
    yield b
    b.KV8, b.QLEN, b.WINDOW, b.PAGED = False, 1, 0, 0


def _visible(n, L, w):
    """Set of (query i, row t) pairs: query i at n - L + i sees t <= its position and,
    with a window w > 0, the last w positions."""
    out = set()
    for i in range(L):
        p = n - L + i
        for t in range(n):
            if t <= p and (w == 0 or t > p - w):
                out.add((i, t))
    return out


@pytest.mark.parametrize("n", [0, 1, 2, 5, 17, 64])
@pytest.mark.parametrize("L,w", [(1, 0), (4, 0), (3, 1), (4, 5), (8, 100), (2, 3)])
def test_active_rows_and_pairs_brute_force(bench, n, L, w):
    bench.QLEN, bench.WINDOW = L, w
    vis = _visible(n, L, w)
    rows = {t for _, t in vis}
    assert bench.visible_pairs(n) == len(vis)
    if w == 0:
        assert bench.active_rows(n) == n                  # no window: the whole sequence
    else:
        # the step reads every row from the first visible one to the end of the sequence
        assert bench.active_rows(n) == (n - min(rows) if rows else 0)


def test_step_bytes_hand_worked(bench):
    cfg = wl.CONFIGS["gqa_b1_h8_kv2_d64_t512"]
    lens = [512]
    base = bench.step_bytes(cfg, lens)
    # q 8*64*2 + K,V 2*512*2*64*2 + out 8*64*4 + lse 8*4
    assert base["total"] == 1024 + 262144 + 2048 + 32
    bench.KV8 = True
    e = bench.step_bytes(cfg, lens)
    assert e["kv"] == 262144 // 2 and e["total"] == 1024 + 131072 + 2048 + 32
    bench.KV8, bench.QLEN, bench.WINDOW = False, 4, 100
    m = bench.step_bytes(cfg, lens)
    # rows 512 - (512 - 4 + 1 - 100) = 103 are read; q, out and lse carry the L axis
    assert m["kv"] == 2 * 103 * 2 * 64 * 2
    assert m["total"] == 4 * 1024 + 2 * 103 * 2 * 64 * 2 + 4 * 2048 + 4 * 32
    # flops: 4 * d per (query head, visible row)
    assert bench.step_flops(cfg, lens) == bench.visible_pairs(512) * 8 * 4 * 64


def test_variant_suffix(bench):
    bench.KV8, bench.QLEN, bench.WINDOW, bench.PAGED = True, 4, 4096, 128
    assert bench.variant_suffix() == "_e4m3_L4_w4096_paged128"
