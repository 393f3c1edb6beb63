"""Decode-attention benchmark: one JSON line on stdout (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kvattn|reference]
                    [--config NAME] [--no-extra-configs] [--cpu-sample-s S]
                    [--paged PAGE_SIZE] [--kv-dtype bf16|e4m3] [--q-len L] [--window W]

A step is one library call covering every sequence of one layer's decode step for the
workload (all of its query heads, out and lse complete, split-KV combine included).
The headline workload is the Llama-2-7B-shaped MHA layer (batch 32, 32/32 heads,
head_dim 128, context 4096); the other workloads are measured on the same line under
"configs".  Inputs are seeded synthetic tensors resident in HBM before the timed
region; L2 is flushed before every timed step (a 256 MiB device write, then a read of
the same buffer so no dirty line is left to write back) and the flush is outside the
step's CUDA-event interval.  With N > 1 (torchrun, one rank per GPU)
every rank runs its own independent batch (replicas: the units of this path are
independent sequences, there is no collective on the data path); the time is the
maximum over ranks and the value is the bytes of all ranks over that time.

Metric: decode-attention time per step, bytes per second and fraction of the measured
HBM peak.  Bytes per step are the algorithmic minimum: q + the touched K/V (or latent +
RoPE) cache rows + fp32 out + fp32 lse.  Variants of the GQA workloads: an E4M3 cache
(--kv-dtype e4m3, one byte per cached value), L new tokens per sequence with the causal
mask (--q-len) and a sliding window (--window: only the rows some query can see are
touched).
"""
import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

from mla_kv_cache_b200 import workloads as wl

ROOT = os.path.dirname(os.path.abspath(__file__))
HEADLINE = "mha_b32_h32_d128_t4096"
METRIC = "decode-attention µs/step, KV-cache GB/s and % of B200 HBM roofline"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
HOST_HIDE_CYCLES = 200_000      # ~0.1 ms of GPU spin before each timed step


# ----------------------------------------------------------------------------- variants
PAGED = 0   # --paged: rows per page of a paged cache layout (0: contiguous cache)
KV8 = False  # --kv-dtype e4m3: E4M3 cache codes, one scale per tensor
QLEN = 1    # --q-len: new tokens per sequence (causal among them)
WINDOW = 0  # --window: sliding window in tokens (0: none)


def variant_suffix():
    return (("_e4m3" if KV8 else "") + (f"_L{QLEN}" if QLEN > 1 else "") +
            (f"_w{WINDOW}" if WINDOW else "") + (f"_paged{PAGED}" if PAGED else ""))


def active_rows(n):
    """Rows of a sequence of n cached tokens that some query can see."""
    if WINDOW <= 0:
        return n
    return n - max(0, n - QLEN + 1 - WINDOW)


def visible_pairs(n):
    """(query, cached row) pairs that take part in attention for one head of a sequence."""
    tot = 0
    for i in range(QLEN):
        hi = n - QLEN + i + 1
        lo = max(0, hi - WINDOW) if WINDOW > 0 else 0
        tot += max(0, hi - lo)
    return tot


# ----------------------------------------------------------------------------- bytes / flops
def step_bytes(cfg, lens):
    """Algorithmic bytes of one step: q + touched cache rows + out (fp32) + lse (fp32)."""
    lens = [min(max(int(x), 0), cfg.max_seq_len) for x in lens]
    if isinstance(cfg, wl.MLAConfig):
        q = QLEN * cfg.batch * cfg.n_heads * (cfg.latent_dim + cfg.rope_dim) * 2
        kv = sum(lens) * (cfg.latent_dim + cfg.rope_dim) * (1 if KV8 else 2)
        out = QLEN * cfg.batch * cfg.n_heads * cfg.latent_dim * 4
        lse = QLEN * cfg.batch * cfg.n_heads * 4
    else:
        q = QLEN * cfg.batch * cfg.n_q_heads * cfg.head_dim * 2
        kv = 2 * sum(active_rows(n) for n in lens) * cfg.n_kv_heads * cfg.head_dim * (1 if KV8 else 2)
        out = QLEN * cfg.batch * cfg.n_q_heads * cfg.head_dim * 4
        lse = QLEN * cfg.batch * cfg.n_q_heads * 4
    return {"total": q + kv + out + lse, "kv": kv, "q": q, "out": out + lse}


def step_flops(cfg, lens):
    """Algorithmic flops: 2 per multiply-add of the score and the value products."""
    lens = [min(max(int(x), 0), cfg.max_seq_len) for x in lens]
    if isinstance(cfg, wl.MLAConfig):
        vis = sum(max(0, n - QLEN + 1 + i) for n in lens for i in range(QLEN))
        return vis * cfg.n_heads * 2 * ((cfg.latent_dim + cfg.rope_dim) + cfg.latent_dim)
    return sum(visible_pairs(n) for n in lens) * cfg.n_q_heads * 4 * cfg.head_dim


def variant_fields():
    return {"kv_dtype": "e4m3 (one scale per tensor)" if KV8 else "bf16", "q_len": QLEN, "window": WINDOW}


def workload_fields(cfg):
    if isinstance(cfg, wl.MLAConfig):
        return {"batch": cfg.batch, "n_heads": cfg.n_heads, "latent_dim": cfg.latent_dim,
                "rope_dim": cfg.rope_dim, "seq_len": cfg.max_seq_len}
    return {"batch": cfg.batch, "n_q_heads": cfg.n_q_heads, "n_kv_heads": cfg.n_kv_heads,
            "head_dim": cfg.head_dim, "seq_len": cfg.max_seq_len}


def config_fields(name, cfg, nb, world):
    """The line's "config" object; both arms print the same one for the same workload."""
    if isinstance(cfg, wl.MLAConfig):
        layout = "contiguous latent [B, T, 512] + RoPE key [B, T, 64]"
    else:
        layout = "contiguous [B, n_kv, T, d]"
    return {"workload": name + variant_suffix(), **workload_fields(cfg), **variant_fields(),
            "bytes_per_step": nb["total"],
            "cache_layout": f"paged: {PAGED}-row pages in a shuffled pool, block table" if PAGED else layout,
            "l2": "flushed before every timed step (256 MiB device write + read-back, outside the timed interval)",
            "parallelism": f"replicas x{world}: one independent batch per GPU, no collective"}


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "source": "measured (MEASURED_PEAKS.json)"}
    except Exception:
        return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
                "source": "fallback (profiling recipe)"}


def kernel_sources_sha(names):
    import hashlib
    h = hashlib.sha256()
    for name in names:
        path = os.path.join(ROOT, "mla_kv_cache_b200", "csrc", name)
        if os.path.exists(path):
            h.update(open(path, "rb").read())
    return h.hexdigest()


def recorded_traffic(workload):
    """DRAM bytes per launch from the committed ncu summary, or None when the kernel
    sources changed since those counters were taken."""
    try:
        rec = json.load(open(os.path.join(ROOT, "profiles", "traffic.json"))).get(workload)
    except Exception:
        return None
    if not rec or rec.get("source_sha256") != kernel_sources_sha(rec.get("sources", [])):
        return None
    return rec.get("bytes")


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        rows = []
        try:
            for line in open(self.path):
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        except Exception:
            pass
        finally:
            try:
                os.unlink(self.path)
            except Exception:
                pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


def physical_gpu_id():
    """nvidia-smi id (index or UUID) of the current CUDA device."""
    cur = torch.cuda.current_device()
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        if cur < len(ids):
            return ids[cur]
    return str(cur)


# ----------------------------------------------------------------------------- distributed
def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return rank, world, local


def dist_max(x):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dev = torch.device("cuda") if torch.cuda.is_available() else torch.device("cpu")
        t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())
    return float(x)


def dist_barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


# ----------------------------------------------------------------------------- GPU arm


def to_pages(cache, page_size, seq_axis, perm):
    """A contiguous cache [B, ..., T, ...] (T at seq_axis) laid out as a shuffled pool of
    pages: page b * M + lp of the natural order goes to slot perm[b * M + lp]."""
    B, T = cache.shape[0], cache.shape[seq_axis]
    M = T // page_size
    if seq_axis == 2:    # [B, n_kv, T, d] -> [B * M, n_kv, S, d]
        pages = cache.view(B, cache.shape[1], M, page_size, cache.shape[3]).permute(0, 2, 1, 3, 4)
        pages = pages.reshape(B * M, cache.shape[1], page_size, cache.shape[3])
    else:                # [B, T, c] -> [B * M, S, c]
        pages = cache.view(B * M, page_size, cache.shape[2])
    pool = torch.empty_like(pages)
    pool[perm] = pages
    return pool


def host_inputs(cfg, seed):
    """The workload's seeded inputs (CPU) with the variant applied."""
    if WINDOW and isinstance(cfg, wl.MLAConfig):
        raise ValueError("windows: GQA workloads only")
    if isinstance(cfg, wl.MLAConfig):
        x = wl.make_mla_inputs_fp8(cfg, seed=seed) if KV8 else wl.make_mla_inputs(cfg, seed=seed)
        if QLEN > 1:
            g = torch.Generator().manual_seed(seed + 29)
            x["q_latent"] = torch.randn((cfg.batch, QLEN, cfg.n_heads, cfg.latent_dim),
                                        generator=g).to(torch.bfloat16)
            x["q_rope"] = torch.randn((cfg.batch, QLEN, cfg.n_heads, cfg.rope_dim), generator=g).to(torch.bfloat16)
        return x
    x = wl.make_gqa_inputs_fp8(cfg, seed=seed) if KV8 else wl.make_inputs(cfg, seed=seed)
    if QLEN > 1:
        g = torch.Generator().manual_seed(seed + 29)
        x["q"] = torch.randn((cfg.batch, QLEN, cfg.n_q_heads, cfg.head_dim), generator=g).to(torch.bfloat16)
    elif WINDOW and not KV8:
        x["q"] = x["q"][:, None].contiguous()     # the multi-token entry point's layout, L = 1
    return x


def q4d():
    """The variant's query carries an L axis (and so do out and lse)."""
    return QLEN > 1 or (WINDOW > 0 and not KV8)


def device_inputs(cfg, seed):
    x = host_inputs(cfg, seed)
    d = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in x.items()}
    if PAGED:
        T = cfg.max_seq_len
        if T % PAGED:
            raise ValueError(f"--paged {PAGED} does not divide the cache capacity {T}")
        M = T // PAGED
        g = torch.Generator().manual_seed(seed + 17)
        perm = torch.randperm(cfg.batch * M, generator=g).cuda()
        d["block_table"] = perm.view(cfg.batch, M).to(torch.int32).contiguous()
        names = ("latent_cache", "rope_cache") if isinstance(cfg, wl.MLAConfig) else ("k_cache", "v_cache")
        axis = 1 if isinstance(cfg, wl.MLAConfig) else 2
        for n in names:
            d[n + "_pages"] = to_pages(d.pop(n), PAGED, axis, perm)
        torch.cuda.empty_cache()
    return x, d


def make_call(cfg, d, out, lse, stream):
    from mla_kv_cache_b200 import binding as kb
    if QLEN > 1 and isinstance(cfg, wl.MLAConfig):
        if PAGED:
            raise ValueError("the MLA multi-token entry point takes a contiguous cache")
        return lambda: kb.kvattn_mla_decode_multi(d["q_latent"], d["q_rope"], d["latent_cache"], d["rope_cache"],
                                                  d["seq_lens"], cfg.scale, d.get("latent_scale"),
                                                  d.get("rope_scale"), out=out, lse=lse, stream=stream)
    if KV8 and isinstance(cfg, wl.MLAConfig):
        if PAGED:
            return lambda: kb.kvattn_mla_decode_fp8_paged(d["q_latent"], d["q_rope"], d["latent_cache_pages"],
                                                          d["rope_cache_pages"], d["block_table"], d["seq_lens"],
                                                          cfg.scale, d["latent_scale"], d["rope_scale"], out=out,
                                                          lse=lse, stream=stream)
        return lambda: kb.kvattn_mla_decode_fp8(d["q_latent"], d["q_rope"], d["latent_cache"], d["rope_cache"],
                                                d["seq_lens"], cfg.scale, d["latent_scale"], d["rope_scale"],
                                                out=out, lse=lse, stream=stream)
    if KV8 and PAGED:
        if QLEN > 1 or WINDOW:
            raise ValueError("the paged E4M3 entry point takes one new token and no window")
        return lambda: kb.kvattn_gqa_decode_fp8_paged(d["q"], d["k_cache_pages"], d["v_cache_pages"],
                                                      d["block_table"], d["seq_lens"], cfg.scale, d["k_scale"],
                                                      d["v_scale"], out=out, lse=lse, stream=stream)
    if KV8:
        return lambda: kb.kvattn_gqa_decode_fp8(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], cfg.scale,
                                                d["k_scale"], d["v_scale"], window=WINDOW, out=out, lse=lse,
                                                stream=stream)
    if QLEN > 1 or WINDOW:
        if PAGED:
            raise ValueError("the paged entry points take one new token and no window")
        return lambda: kb.kvattn_gqa_decode_multi(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], cfg.scale,
                                                  window=WINDOW, out=out, lse=lse, stream=stream)
    if PAGED:
        if isinstance(cfg, wl.MLAConfig):
            return lambda: kb.kvattn_mla_decode_paged(d["q_latent"], d["q_rope"], d["latent_cache_pages"],
                                                      d["rope_cache_pages"], d["block_table"], d["seq_lens"],
                                                      cfg.scale, out=out, lse=lse, stream=stream)
        return lambda: kb.kvattn_gqa_decode_paged(d["q"], d["k_cache_pages"], d["v_cache_pages"],
                                                  d["block_table"], d["seq_lens"], cfg.scale, out=out,
                                                  lse=lse, stream=stream)
    if isinstance(cfg, wl.MLAConfig):
        return lambda: kb.kvattn_mla_decode(d["q_latent"], d["q_rope"], d["latent_cache"],
                                            d["rope_cache"], d["seq_lens"], cfg.scale, out=out,
                                            lse=lse, stream=stream)
    return lambda: kb.kvattn_gqa_decode(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], cfg.scale,
                                        out=out, lse=lse, stream=stream)


def out_shapes(cfg):
    if isinstance(cfg, wl.MLAConfig):
        if QLEN > 1:
            return (cfg.batch, QLEN, cfg.n_heads, cfg.latent_dim), (cfg.batch, QLEN, cfg.n_heads)
        return (cfg.batch, cfg.n_heads, cfg.latent_dim), (cfg.batch, cfg.n_heads)
    if q4d():
        return (cfg.batch, QLEN, cfg.n_q_heads, cfg.head_dim), (cfg.batch, QLEN, cfg.n_q_heads)
    return (cfg.batch, cfg.n_q_heads, cfg.head_dim), (cfg.batch, cfg.n_q_heads)


def oracle_step(cfg, x, ids):
    """The oracle on sequences `ids` of the workload (variant applied)."""
    import oracle
    if isinstance(cfg, wl.MLAConfig) and QLEN > 1:
        lat, rope = x["latent_cache"], x["rope_cache"]
        if KV8:
            lat = oracle.e4m3_dequant(lat, x["latent_scale"])
            rope = oracle.e4m3_dequant(rope, x["rope_scale"])
        sel = list(ids)
        return oracle.mla_decode_multi(x["q_latent"][sel], x["q_rope"][sel], lat[sel], rope[sel],
                                       x["seq_lens"][sel], cfg.scale)
    if isinstance(cfg, wl.MLAConfig):
        if KV8:
            return oracle.mla_decode_fp8(x["q_latent"], x["q_rope"], x["latent_cache"], x["rope_cache"],
                                         x["seq_lens"], cfg.scale, x["latent_scale"], x["rope_scale"],
                                         batch_ids=ids)
        return oracle.mla_decode(x["q_latent"], x["q_rope"], x["latent_cache"], x["rope_cache"],
                                 x["seq_lens"], cfg.scale, batch_ids=ids)
    if KV8:
        for b in ids:
            oracle.gqa_decode_fp8(x["q"][b:b + 1], x["k_cache"][b:b + 1], x["v_cache"][b:b + 1],
                                  x["seq_lens"][b:b + 1], cfg.scale, x["k_scale"], x["v_scale"], window=WINDOW)
        return None
    if QLEN > 1 or WINDOW:
        q = x["q"] if x["q"].dim() == 4 else x["q"][:, None]
        for b in ids:
            oracle.gqa_decode_multi(q[b:b + 1], x["k_cache"][b:b + 1], x["v_cache"][b:b + 1],
                                    x["seq_lens"][b:b + 1], cfg.scale, window=WINDOW)
        return None
    return oracle.gqa_decode(x["q"], x["k_cache"], x["v_cache"], x["seq_lens"], cfg.scale, batch_ids=ids)


def is_mla(cfg):
    """The MLA path is one kernel per call; the GQA paths launch a decode and a combine kernel."""
    return isinstance(cfg, wl.MLAConfig)


def flush_l2(buf):
    """Evict the step's data from L2: write a buffer twice the L2 size, then read it
    back, so that L2 holds clean lines (no dirty write-back of the flush itself lands
    inside the next timed step)."""
    buf.zero_()
    buf.view(torch.int64).amax()


def time_device(call, stream, steps, warmup, flush):
    """Per-step CUDA-event time (ms) of `call`, L2 flushed before each step (outside the
    event interval).  Returns the list of step times."""
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            flush_l2(flush)
            call()
    torch.cuda.synchronize()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    with torch.cuda.stream(stream):
        for i in range(steps):
            flush_l2(flush)
            # Keep the GPU busy (outside the timed interval) while the host enqueues the
            # step, so host-side Python latency is not counted as device time.
            torch.cuda._sleep(HOST_HIDE_CYCLES)
            starts[i].record(stream)
            call()
            ends[i].record(stream)
    torch.cuda.synchronize()
    return [s.elapsed_time(e) for s, e in zip(starts, ends)]


def time_e2e(cfg, d, stream, steps, warmup, flush):
    """End to end through the public API: every step copies the step's host inputs (q and
    seq_lens, pinned) to the device, calls the library and reads out and lse back into
    pinned host memory.  The KV cache is the decode loop's resident state in HBM."""
    from mla_kv_cache_b200 import binding as kb
    if isinstance(cfg, wl.MLAConfig):
        names = ["q_latent", "q_rope", "seq_lens"]
    else:
        names = ["q", "seq_lens"]
    host = {n: d[n].cpu().pin_memory() for n in names}
    o_shape, l_shape = out_shapes(cfg)
    out_h = torch.empty(o_shape, dtype=torch.float32).pin_memory()
    lse_h = torch.empty(l_shape, dtype=torch.float32).pin_memory()
    dev = dict(d)
    out = torch.empty(o_shape, dtype=torch.float32, device="cuda")
    lse = torch.empty(l_shape, dtype=torch.float32, device="cuda")
    call = make_call(cfg, dev, out, lse, stream)

    def step():
        for n in names:
            dev[n].copy_(host[n], non_blocking=True)
        call()
        out_h.copy_(out, non_blocking=True)
        lse_h.copy_(lse, non_blocking=True)

    times = time_device(step, stream, steps, warmup, flush)
    h2d = sum(host[n].numel() * host[n].element_size() for n in names)
    d2h = out_h.numel() * 4 + lse_h.numel() * 4
    return times, h2d, d2h


def cpu_baseline(cfg, x, budget_s):
    """The fp64 oracle, as it stands, on a bounded sample of the workload's sequences."""
    import oracle
    lens = x["seq_lens"].tolist()
    order = list(range(cfg.batch))
    done, t_used = [], 0.0
    t0 = time.perf_counter()
    for b in order:
        oracle_step(cfg, x, [b])
        done.append(b)
        t_used = time.perf_counter() - t0
        if t_used >= budget_s:
            break
    sample_lens = [lens[b] for b in done]
    sub = (wl.MLAConfig if isinstance(cfg, wl.MLAConfig) else wl.GQAConfig)
    nbytes = step_bytes(cfg, lens)["total"] * (sum(sample_lens) / max(sum(lens), 1))
    return {"value": nbytes / t_used / 1e9, "unit": "GB/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"{len(done)} of {cfg.batch} sequences of {cfg.name} (all their heads), "
                      f"{t_used:.1f} s of fp64 CPU work incl. exact conversion to fp64; "
                      f"bytes scaled by the sample's share of tokens",
            "us_per_step_extrapolated": t_used * 1e6 * sum(lens) / max(sum(sample_lens), 1)}


def measure_config(cfg, steps, warmup, flush, stream, seed, pk, world):
    x, d = device_inputs(cfg, seed)
    o_shape, l_shape = out_shapes(cfg)
    out = torch.empty(o_shape, dtype=torch.float32, device="cuda")
    lse = torch.empty(l_shape, dtype=torch.float32, device="cuda")
    call = make_call(cfg, d, out, lse, stream)
    dist_barrier()
    torch.cuda.synchronize()
    times = time_device(call, stream, steps, warmup, flush)
    torch.cuda.synchronize()
    dist_barrier()
    ms = dist_max(sum(times) / len(times))
    lens = x["seq_lens"].tolist()
    nb = step_bytes(cfg, lens)
    fl = step_flops(cfg, lens)
    gbs = nb["total"] / (ms * 1e-3) / 1e9
    res = {"us_per_step": ms * 1e3, "us_min": min(times) * 1e3, "gb_per_s": gbs,
           "kv_gb_per_s": nb["kv"] / (ms * 1e-3) / 1e9, "bytes_per_step": nb["total"],
           "hbm_frac": gbs / pk["hbm_gbs"], "tflops": fl / (ms * 1e-3) / 1e12,
           "flops_per_step": fl}
    if isinstance(cfg, wl.MLAConfig):
        t_hbm = nb["total"] / (pk["hbm_gbs"] * 1e9)
        # E4M3 operands: the tensor pipe's fp8 rate, twice the measured bf16 one (the
        # nominal dense ratio, 4.5 / 2.25 PFLOP/s)
        t_tc = fl / (pk["bf16_tflops"] * (2.0 if KV8 else 1.0) * 1e12)
        res["roofline_us"] = max(t_hbm, t_tc) * 1e6
        res["roofline_bound"] = "hbm" if t_hbm >= t_tc else "tensor"
        res["roofline_frac"] = res["roofline_us"] / res["us_per_step"]
    return x, d, res, times


def gpu_arm(args):
    rank, world, local = dist_setup(args.gpus)
    from mla_kv_cache_b200 import binding as kb
    kb.lib()
    pk = peaks()
    stream = torch.cuda.Stream()
    l2 = torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size
    flush = torch.empty(max(256 << 20, 2 * l2), dtype=torch.uint8, device="cuda")
    seed = 0 + rank * 1000   # each replica its own batch

    head_cfg = wl.CONFIGS[args.config]
    extras = {}
    if not args.no_extra_configs:
        for name in wl.CONFIG_ORDER:
            if name == args.config:
                continue
            try:
                _, _, res, _ = measure_config(wl.CONFIGS[name], max(args.steps // 10, 20),
                                              args.warmup, flush, stream, seed, pk, world)
            except Exception as e:  # an unsupported workload is reported, not hidden
                res = {"error": str(e).splitlines()[0][:200]}
            extras[name] = res
            torch.cuda.empty_cache()

    x, d, res, _ = measure_config(head_cfg, 20, args.warmup, flush, stream, seed, pk, world)
    o_shape, l_shape = out_shapes(head_cfg)
    out = torch.empty(o_shape, dtype=torch.float32, device="cuda")
    lse = torch.empty(l_shape, dtype=torch.float32, device="cuda")
    call = make_call(head_cfg, d, out, lse, stream)
    # the timed region proper: exactly K steps, barrier + synchronize on both sides
    with ClockSampler(physical_gpu_id()) as clk:
        dist_barrier()
        torch.cuda.synchronize()
        times = time_device(call, stream, args.steps, args.warmup, flush)
        torch.cuda.synchronize()
        dist_barrier()
    clocks = clk.summary()
    # the library's own count of the kernels one step enqueues (decode, and a combine only
    # when units are cut between workers)
    from mla_kv_cache_b200 import binding as kb
    n0 = kb.kvattn_kernel_launches()
    call()
    torch.cuda.synchronize()
    launches_per_step = kb.kvattn_kernel_launches() - n0
    ms = dist_max(sum(times) / len(times))
    lens = x["seq_lens"].tolist()
    nb = step_bytes(head_cfg, lens)
    value = nb["total"] * world / (ms * 1e-3) / 1e9
    e2e_times, h2d, d2h = time_e2e(head_cfg, d, stream, max(args.steps // 10, 20), args.warmup, flush)
    e2e_ms = dist_max(sum(e2e_times) / len(e2e_times))
    achieved = nb["total"] / (ms * 1e-3) / 1e9
    traffic = recorded_traffic(args.config + variant_suffix())
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "us_per_step": ms * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3 operands, fp32 accumulate" if KV8 else "bf16",
        "data": "synthetic (seeded N(0,1) bf16, shapes of the workload" +
                ("; cache stored as E4M3 codes, scale = max|x| / 448)" if KV8 else ")"),
        "config": config_fields(args.config, head_cfg, nb, world),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / pk["hbm_gbs"], "traffic": traffic,
                     "peak_source": pk["source"] + " burst copy bandwidth",
                     "timed_unit": "one library call: " + (("the decode kernel (partials merged inside it)"
                                                            + (" after the virtual-batch kernel"
                                                               if launches_per_step > 1 else ""))
                                                           if is_mla(head_cfg) else
                                                           "decode kernel + PDL-chained combine kernel"
                                                           if launches_per_step > 1 else
                                                           "the decode kernel (no unit cut: no combine)")},
        "e2e": {"value": nb["total"] * world / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
                "us_per_step": e2e_ms * 1e3, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "note": "per step: pinned host q/seq_lens -> device, library call, out/lse -> pinned host; KV cache resident in HBM"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
        "configs": dict(extras, **{args.config: res}),
    }
    if rank == 0 and world == 1 and args.cpu_sample_s > 0:
        line["cpu_baseline"] = cpu_baseline(head_cfg, x, args.cpu_sample_s)
    if rank == 0:
        print(json.dumps(line), flush=True)
    _finish()


def reference_arm(args):
    """The oracle on the host cores: same workload, metric and unit; each step is a
    bounded sample of the workload (a few sequences), scaled by its share of tokens."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    cfg = wl.CONFIGS[args.config]
    x = host_inputs(cfg, seed=0)
    lens = x["seq_lens"].tolist()
    nb = step_bytes(cfg, lens)
    per_step_seqs = max(1, min(cfg.batch, args.ref_sequences))
    times, shares = [], []
    for s in range(args.warmup + args.steps):
        ids = [(s * per_step_seqs + i) % cfg.batch for i in range(per_step_seqs)]
        t0 = time.perf_counter()
        oracle_step(cfg, x, ids)
        dt = time.perf_counter() - t0
        if s >= args.warmup:
            times.append(dt)
            shares.append(sum(lens[i] for i in ids) / max(sum(lens), 1))
    # seconds for a whole step, extrapolated from the sampled share of tokens
    full_s = statistics.mean(t / sh for t, sh in zip(times, shares))
    value = nb["total"] / full_s / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": full_s * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) bf16, shapes of the workload)",
        "config": config_fields(args.config, cfg, nb, world),
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": oracle.num_threads(),
                         "kind": "oracle",
                         "sample": f"{per_step_seqs} of {cfg.batch} sequences per step (all heads), "
                                   f"time scaled by their share of tokens"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def _finish():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="kvattn", choices=["kvattn", "reference"])
    ap.add_argument("--config", default=HEADLINE, choices=wl.CONFIG_ORDER)
    ap.add_argument("--no-extra-configs", action="store_true")
    ap.add_argument("--cpu-sample-s", type=float, default=10.0)
    ap.add_argument("--ref-sequences", type=int, default=2)
    ap.add_argument("--paged", type=int, default=0, metavar="PAGE_SIZE",
                    help="time the paged-cache entry points, the cache cut into pages of this "
                         "many rows (a multiple of 64) and shuffled over a pool")
    ap.add_argument("--kv-dtype", default="bf16", choices=["bf16", "e4m3"],
                    help="cache storage: bf16, or E4M3 codes with one scale per tensor (GQA workloads)")
    ap.add_argument("--q-len", type=int, default=1, help="new tokens per sequence (causal among them)")
    ap.add_argument("--window", type=int, default=0, help="sliding window in tokens (0: none)")
    args = ap.parse_args()
    global PAGED, KV8, QLEN, WINDOW
    PAGED = args.paged
    KV8 = args.kv_dtype == "e4m3"
    QLEN = args.q_len
    WINDOW = args.window
    if QLEN < 1 or WINDOW < 0:
        ap.error("--q-len must be >= 1 and --window >= 0")
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        reference_arm(args)
    else:
        gpu_arm(args)


if __name__ == "__main__":
    main()
