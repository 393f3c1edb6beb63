"""Seeded synthetic inputs for decode attention -- shared by the tests, the bench and
the oracle checks.

This module only draws random numbers and lays them out; it holds none of the
attention arithmetic.  Every tensor is produced on the CPU from a torch.Generator
seeded by the caller (default 0), in a fixed draw order, and rounded once to bf16
(round to nearest even) after any scaling or offset, so the stored bf16 values are
the ground truth for both the CUDA path and the oracle.

Draw order for one workload:
  GQA: seq_lens (ragged configs only), q, k, v, then spike positions (spiky configs).
  MLA: seq_lens (ragged configs only), q_latent, q_rope, latent_cache, rope_cache.
Caches are drawn one sequence at a time (batch-major), so a workload's values do not
depend on how much memory the host has.
"""
import math
from dataclasses import dataclass
from typing import Optional, Sequence, Tuple

import torch


@dataclass(frozen=True)
class GQAConfig:
    """One GQA/MQA/MHA decode workload: q [B, n_q, d], caches [B, n_kv, max_seq_len, d]."""
    name: str
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    max_seq_len: int
    scale: float
    # None: every sequence has max_seq_len tokens; (lo, hi): uniform integers in [lo, hi];
    # an explicit tuple of ints with one entry per sequence is also accepted.
    seq_len_range: Optional[Tuple[int, int]] = None
    seq_lens: Optional[Tuple[int, ...]] = None
    key_scale: float = 1.0          # k = bf16(key_scale * N(0,1) [+ spikes])
    spike_fraction: float = 0.0     # fraction of positions per sequence given a key offset
    spike_value: float = 0.0

    @property
    def group_size(self):
        return self.n_q_heads // self.n_kv_heads


@dataclass(frozen=True)
class MLAConfig:
    """One absorbed-MLA decode workload (latent 512 + RoPE 64 in the DeepSeek shape)."""
    name: str
    batch: int
    n_heads: int
    latent_dim: int
    rope_dim: int
    max_seq_len: int
    scale: float
    seq_len_range: Optional[Tuple[int, int]] = None
    seq_lens: Optional[Tuple[int, ...]] = None


# The five workloads of the headline measurement, in their published order.
CONFIGS = {
    # batch 1, 8 query heads, 2 KV heads (group 4), head_dim 64, context 512, scale 1/8
    "gqa_b1_h8_kv2_d64_t512": GQAConfig(
        "gqa_b1_h8_kv2_d64_t512", 1, 8, 2, 64, 512, 1.0 / 8.0),
    # Llama-2-7B-shaped MHA layer: batch 32, 32/32 heads, d 128, context 4096
    "mha_b32_h32_d128_t4096": GQAConfig(
        "mha_b32_h32_d128_t4096", 32, 32, 32, 128, 4096, 1.0 / math.sqrt(128.0)),
    # 70B-shaped GQA layer: batch 16, 64 q / 8 kv heads, d 128, ragged contexts in
    # [1024, 8192], keys scaled by 2 to sharpen the softmax
    "gqa_b16_h64_kv8_d128_ragged8192": GQAConfig(
        "gqa_b16_h64_kv8_d128_ragged8192", 16, 64, 8, 128, 8192, 1.0 / math.sqrt(128.0),
        seq_len_range=(1024, 8192), key_scale=2.0),
    # long-context MQA: batch 4, 32 q heads, 1 KV head, d 128, context 32768, 1% of key
    # positions given a +4 offset spike
    "mqa_b4_h32_d128_t32768": GQAConfig(
        "mqa_b4_h32_d128_t32768", 4, 32, 1, 128, 32768, 1.0 / math.sqrt(128.0),
        spike_fraction=0.01, spike_value=4.0),
    # DeepSeek-shaped absorbed MLA: batch 32, 128 heads, latent 512 + RoPE 64, context
    # 4096, scale 1/sqrt(192)
    "mla_b32_h128_c512_r64_t4096": MLAConfig(
        "mla_b32_h128_c512_r64_t4096", 32, 128, 512, 64, 4096, 1.0 / math.sqrt(192.0)),
}
CONFIG_ORDER = list(CONFIGS)


def _draw_lens(cfg, g):
    B, T = cfg.batch, cfg.max_seq_len
    if cfg.seq_lens is not None:
        assert len(cfg.seq_lens) == B
        return torch.tensor(cfg.seq_lens, dtype=torch.int32)
    if cfg.seq_len_range is not None:
        lo, hi = cfg.seq_len_range
        return torch.randint(lo, hi + 1, (B,), generator=g, dtype=torch.int64).to(torch.int32)
    return torch.full((B,), T, dtype=torch.int32)


def _normal_bf16(shape, g, scale=1.0):
    x = torch.randn(shape, generator=g, dtype=torch.float32)
    if scale != 1.0:
        x = x * scale
    return x.to(torch.bfloat16)


def _poison(cache, lens, seq_axis):
    """Fill every position >= seq_lens[b] with NaN (tests prove those are never read)."""
    for b, L in enumerate(lens.tolist()):
        idx = [b] + [slice(None)] * (cache.dim() - 1)
        idx[seq_axis] = slice(int(L), None)
        cache[tuple(idx)] = float("nan")


def make_gqa_inputs(cfg: GQAConfig, seed: int = 0, poison_tail: bool = False):
    """Returns dict(q, k_cache, v_cache, seq_lens) as CPU tensors (bf16, int32)."""
    g = torch.Generator().manual_seed(seed)
    B, Hq, Hk, d, T = cfg.batch, cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim, cfg.max_seq_len
    lens = _draw_lens(cfg, g)
    q = _normal_bf16((B, Hq, d), g)
    k = torch.empty((B, Hk, T, d), dtype=torch.bfloat16)
    v = torch.empty((B, Hk, T, d), dtype=torch.bfloat16)
    need_fp32_keys = cfg.spike_fraction > 0
    k32 = torch.empty((B, Hk, T, d), dtype=torch.float32) if need_fp32_keys else None
    for b in range(B):
        kb = torch.randn((Hk, T, d), generator=g, dtype=torch.float32)
        if cfg.key_scale != 1.0:
            kb = kb * cfg.key_scale
        if need_fp32_keys:
            k32[b] = kb
        else:
            k[b] = kb.to(torch.bfloat16)
    for b in range(B):
        v[b] = _normal_bf16((Hk, T, d), g)
    if need_fp32_keys:
        n_spikes = int(math.floor(cfg.spike_fraction * T))
        for b in range(B):
            pos = torch.randperm(T, generator=g)[:n_spikes]
            k32[b][:, pos, :] += cfg.spike_value
            k[b] = k32[b].to(torch.bfloat16)
        del k32
    if poison_tail:
        _poison(k, lens, 2)
        _poison(v, lens, 2)
    return {"q": q, "k_cache": k, "v_cache": v, "seq_lens": lens}


def quantize_e4m3(x, seq_lens=None, seq_axis=2):
    """Synthesises an fp8 (E4M3) cache from a bf16 one: scale = max|x| / 448 (float32),
    codes = the nearest E4M3 values of x / scale (PyTorch's conversion).  Rows past
    seq_lens[b] (NaN in a poisoned cache) get the NaN code.  Returns (codes as a
    float8_e4m3fn tensor, scale)."""
    finite = x[~torch.isnan(x)] if torch.isnan(x).any() else x
    amax = float(finite.abs().max().float()) if finite.numel() else 1.0
    scale = float(torch.tensor(amax / 448.0 if amax > 0 else 1.0, dtype=torch.float32))
    codes = torch.empty(x.shape, dtype=torch.float8_e4m3fn)
    s32 = torch.tensor(scale, dtype=torch.float32)
    for b in range(x.shape[0]):
        xb = x[b].float() / s32
        codes[b] = xb.clamp(-448.0, 448.0).to(torch.float8_e4m3fn)
    if seq_lens is not None:
        raw = codes.view(torch.uint8)
        for b, n in enumerate(seq_lens.tolist()):
            idx = [b] + [slice(None)] * (x.dim() - 1)
            idx[seq_axis] = slice(int(n), None)
            raw[tuple(idx)] = 0x7F
    return codes, scale


def make_gqa_inputs_fp8(cfg: GQAConfig, seed: int = 0, poison_tail: bool = False):
    """The bf16 workload of make_gqa_inputs (same draws), with its caches stored as
    E4M3 codes and one float scale per cache tensor.  Returns dict(q, k_cache, v_cache,
    seq_lens, k_scale, v_scale); the caches are float8_e4m3fn tensors."""
    x = make_gqa_inputs(cfg, seed, poison_tail=False)
    lens = x["seq_lens"] if poison_tail else None
    k8, ks = quantize_e4m3(x["k_cache"], lens)
    del x["k_cache"]
    v8, vs = quantize_e4m3(x["v_cache"], lens)
    del x["v_cache"]
    return {"q": x["q"], "k_cache": k8, "v_cache": v8, "seq_lens": x["seq_lens"], "k_scale": ks, "v_scale": vs}


def make_mla_inputs(cfg: MLAConfig, seed: int = 0, poison_tail: bool = False):
    """Returns dict(q_latent, q_rope, latent_cache, rope_cache, seq_lens) (CPU tensors)."""
    g = torch.Generator().manual_seed(seed)
    B, H, dc, dr, T = cfg.batch, cfg.n_heads, cfg.latent_dim, cfg.rope_dim, cfg.max_seq_len
    lens = _draw_lens(cfg, g)
    q_lat = _normal_bf16((B, H, dc), g)
    q_rope = _normal_bf16((B, H, dr), g)
    lat = torch.empty((B, T, dc), dtype=torch.bfloat16)
    rope = torch.empty((B, T, dr), dtype=torch.bfloat16)
    for b in range(B):
        lat[b] = _normal_bf16((T, dc), g)
    for b in range(B):
        rope[b] = _normal_bf16((T, dr), g)
    if poison_tail:
        _poison(lat, lens, 1)
        _poison(rope, lens, 1)
    return {"q_latent": q_lat, "q_rope": q_rope, "latent_cache": lat, "rope_cache": rope,
            "seq_lens": lens}


def make_mla_inputs_fp8(cfg: MLAConfig, seed: int = 0, poison_tail: bool = False):
    """The bf16 workload of make_mla_inputs (same draws), with the latent and RoPE caches
    stored as E4M3 codes and one float scale per cache tensor.  Returns dict(q_latent,
    q_rope, latent_cache, rope_cache, seq_lens, latent_scale, rope_scale); the caches are
    float8_e4m3fn tensors."""
    x = make_mla_inputs(cfg, seed, poison_tail=False)
    lens = x["seq_lens"] if poison_tail else None
    lat8, ls = quantize_e4m3(x["latent_cache"], lens, seq_axis=1)
    del x["latent_cache"]
    rope8, rs = quantize_e4m3(x["rope_cache"], lens, seq_axis=1)
    del x["rope_cache"]
    return {"q_latent": x["q_latent"], "q_rope": x["q_rope"], "latent_cache": lat8, "rope_cache": rope8,
            "seq_lens": x["seq_lens"], "latent_scale": ls, "rope_scale": rs}


def make_inputs(cfg, seed: int = 0, poison_tail: bool = False):
    if isinstance(cfg, MLAConfig):
        return make_mla_inputs(cfg, seed, poison_tail)
    return make_gqa_inputs(cfg, seed, poison_tail)


def sample_batch_ids(batch: int, n: int, seed: int = 1) -> Sequence[int]:
    """A seeded subset of batch indices (always including the first and the last)."""
    if n >= batch:
        return list(range(batch))
    g = torch.Generator().manual_seed(seed)
    mid = torch.randperm(max(batch - 2, 1), generator=g)[: max(n - 2, 0)] + 1
    return sorted(set([0, batch - 1] + [int(x) for x in mid.tolist()]))
