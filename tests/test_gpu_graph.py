"""GPU parity of decode calls captured in a CUDA graph and replayed (B200).

A serving loop captures its decode step once and replays it every step, so a call's
kernels must compute the right result on every replay of the same launch parameters: the
work split is derived on the device from seq_lens, and the MLA kernel's merge counters
must count from zero again on each replay although the captured launch carries one and
the same call number.  Each case makes one call first (it sizes the workspace), captures
a second one, then replays it three times with the outputs NaN-filled before each replay
(a replay that left a block unwritten or unmerged would show) and with the sequence
lengths changed between replays; every replay must match the fp64 oracle.
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


def _replays(call, out, lse, dlens, lens_per_replay, check):
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        call()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        call()
    torch.cuda.synchronize()
    for lens in lens_per_replay:
        dlens.copy_(torch.tensor(lens, dtype=torch.int32))
        out.fill_(float("nan"))
        lse.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        check(lens, out.cpu().numpy(), lse.cpu().numpy())
    del g


@pytest.mark.parametrize("kv8", [False, True], ids=["bf16", "e4m3"])
def test_mla_graph_replays(kv8):
    B, H, T = 8, 128, 4096
    first = (4096,) * B                     # every sequence cut over several CTA pairs
    cfg = wl.MLAConfig("graph_mla", B, H, 512, 64, T, 1.0 / math.sqrt(192.0), seq_lens=first)
    x = wl.make_mla_inputs_fp8(cfg, seed=61) if kv8 else wl.make_mla_inputs(cfg, seed=61)
    d = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in x.items()}
    out = torch.empty((B, H, 512), dtype=torch.float32, device="cuda")
    lse = torch.empty((B, H), dtype=torch.float32, device="cuda")
    if kv8:
        call = lambda: kb.kvattn_mla_decode_fp8(d["q_latent"], d["q_rope"], d["latent_cache"], d["rope_cache"],
                                                d["seq_lens"], cfg.scale, d["latent_scale"], d["rope_scale"],
                                                out=out, lse=lse)
    else:
        call = lambda: kb.kvattn_mla_decode(d["q_latent"], d["q_rope"], d["latent_cache"], d["rope_cache"],
                                            d["seq_lens"], cfg.scale, out=out, lse=lse)

    def check(lens, o, l):
        lens_t = torch.tensor(lens, dtype=torch.int32)
        if kv8:
            ro, rl = oracle.mla_decode_fp8(x["q_latent"], x["q_rope"], x["latent_cache"], x["rope_cache"], lens_t,
                                           cfg.scale, x["latent_scale"], x["rope_scale"])
        else:
            ro, rl = oracle.mla_decode(x["q_latent"], x["q_rope"], x["latent_cache"], x["rope_cache"], lens_t,
                                       cfg.scale)
        assert_close(o, ro, f"replay {lens} out")
        assert_close(l, rl, f"replay {lens} lse")

    _replays(call, out, lse, d["seq_lens"], [first, first, (4096, 0, 1, 3000, 4096, 129, 2048, 4000)], check)


@pytest.mark.parametrize("n_q,n_kv,d_head", [(64, 8, 128), (32, 1, 128), (16, 2, 64)],
                         ids=["tc_g8", "tc_mqa", "warp_d64"])
def test_gqa_graph_replays(n_q, n_kv, d_head):
    B, T = 4, 8192
    first = (8192, 8192, 5000, 300)
    cfg = wl.GQAConfig("graph_gqa", B, n_q, n_kv, d_head, T, 1.0 / math.sqrt(d_head), seq_lens=first)
    x = wl.make_gqa_inputs(cfg, seed=67)
    d = {k: v.cuda() for k, v in x.items()}
    out = torch.empty((B, n_q, d_head), dtype=torch.float32, device="cuda")
    lse = torch.empty((B, n_q), dtype=torch.float32, device="cuda")
    call = lambda: kb.kvattn_gqa_decode(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], cfg.scale,
                                        out=out, lse=lse)

    def check(lens, o, l):
        ro, rl = oracle.gqa_decode(x["q"], x["k_cache"], x["v_cache"], torch.tensor(lens, dtype=torch.int32),
                                   cfg.scale)
        assert_close(o, ro, f"replay {lens} out")
        assert_close(l, rl, f"replay {lens} lse")

    _replays(call, out, lse, d["seq_lens"], [first, first, (1, 8192, 0, 7777)], check)
