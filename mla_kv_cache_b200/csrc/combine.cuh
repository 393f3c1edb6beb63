// combine.cuh -- merge of split-KV partial results by log-sum-exp.
//
// Attention over a token range [0, T) is the log-sum-exp merge of attention over any
// partition of that range: with per-part normalised outputs o_s and log-sum-exps
// lse_s,  lse = log sum_s exp(lse_s)  and  out = sum_s exp(lse_s - lse) * o_s.  An empty
// part has lse_s = -inf and weight 0.  The decode kernels leave one partial (o_s, lse_s)
// per worker that touched a unit cut by a worker boundary; this kernel merges them.
//
// Launched right after the decode kernel with programmatic dependent launch: the CTAs
// may start early but wait (griddepcontrol.wait) until the decode grid has finished
// and its writes are visible.  One CTA per (unit, head row); units covered entirely by
// one worker were finished by that worker and are skipped; empty sequences get
// out = 0, lse = -inf here.
#pragma once
#include "common.cuh"
#include "schedule.cuh"

namespace kvattn {

struct CombineParams {
    const void *ws_meta;
    const float *ws_lse;   // [workers, 2, heads_per_unit]
    const float *ws_o;     // [workers, 2, heads_per_unit, D]
    float *out;            // [B, n_q, D]
    float *lse;            // [B, n_q]
    int B, n_q;
    int units_per_seq;     // U
    int heads_per_unit;    // rows of one unit's output block (HEADS of the decode kernel)
    int n_hb;              // head blocks per group (GQA); 1 for MLA
    int n_kv;              // KV heads (GQA); 1 for MLA
    int g;                 // query heads per KV head (GQA); n_heads for MLA
};

// VEC floats per thread, D / VEC threads per CTA.
template <int D, int VEC>
__global__ void __launch_bounds__(D / VEC) combine_kernel(const CombineParams p) {
    pdl_wait_primary();
    const int u = blockIdx.x;                // unit = b * U + i
    const int r = blockIdx.y;                // row within the unit's head block
    const int b = u / p.units_per_seq;
    const int i = u % p.units_per_seq;
    const int j = i / p.n_hb;
    const int hb = i % p.n_hb;
    const int hg = hb * p.heads_per_unit + r;
    if (hg >= p.g) return;
    const size_t gh = (size_t)b * p.n_q + (size_t)j * p.g + hg;
    const int col = threadIdx.x * VEC;

    const MetaView mv = meta_view(const_cast<void *>(p.ws_meta));
    const long long W = mv.w_total[0];
    const int n_tiles = mv.prefix[b + 1] - mv.prefix[b];
    if (n_tiles == 0) {
#pragma unroll
        for (int v = 0; v < VEC; ++v) p.out[gh * D + col + v] = 0.f;
        if (threadIdx.x == 0) p.lse[gh] = -INFINITY;
        return;
    }
    const long long ustart = (long long)mv.prefix[b] * p.units_per_seq + (long long)i * n_tiles;
    const long long c_first = ustart / W;
    const long long c_last = (ustart + n_tiles - 1) / W;
    if (c_first == c_last) return;            // finished by its only worker

    float M = -INFINITY;
    for (long long c = c_first; c <= c_last; ++c) {
        const int slot = (ustart <= c * W) ? 0 : 1;
        M = fmaxf(M, p.ws_lse[((size_t)c * 2 + slot) * p.heads_per_unit + r]);
    }
    float acc[VEC];
#pragma unroll
    for (int v = 0; v < VEC; ++v) acc[v] = 0.f;
    float S = 0.f;
    for (long long c = c_first; c <= c_last; ++c) {
        const int slot = (ustart <= c * W) ? 0 : 1;
        const size_t part = ((size_t)c * 2 + slot) * p.heads_per_unit + r;
        const float w = __expf(p.ws_lse[part] - M);
        S += w;
        const float *src = p.ws_o + part * D + col;
        if (VEC == 4) {
            const float4 x = *reinterpret_cast<const float4 *>(src);
            acc[0] += w * x.x; acc[1] += w * x.y; acc[2] += w * x.z; acc[3] += w * x.w;
        } else {
#pragma unroll
            for (int v = 0; v < VEC; ++v) acc[v] += w * src[v];
        }
    }
    const float inv = 1.f / S;
#pragma unroll
    for (int v = 0; v < VEC; ++v) p.out[gh * D + col + v] = acc[v] * inv;
    if (threadIdx.x == 0) p.lse[gh] = M + __logf(S);
}

}  // namespace kvattn
