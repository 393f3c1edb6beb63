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
// and its writes are visible.  Before that wait each CTA derives the work split from
// seq_lens itself (the same integer arithmetic as the decode kernels, schedule.cuh), so
// that after it the partials' loads go out at once.  One CTA per (unit, head row);
// units covered entirely by one worker were finished by that worker and are skipped;
// empty sequences get out = 0, lse = -inf here.  The CTA's warps take the partials
// round robin, each keeps a running (max, sum, weighted output) -- the same online
// rescaling as the decode kernels -- with up to eight partials' loads in flight, and the
// warps' states are merged at the end through shared memory.
#pragma once
#include "common.cuh"
#include "schedule.cuh"

namespace kvattn {

struct CombineParams {
    const int32_t *seq_lens;
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
    int T_max;             // cache capacity per sequence
    int tile;              // tokens per tile of the decode kernel
    int workers;           // decode workers (CTAs or CTA pairs)
    int min_tiles;         // the decode kernel's minimum tiles per worker
    int q_len;             // new tokens per sequence (rows of a unit: q_len x g)
    int window;            // sliding window (0: none)
    int unit_split;        // the decode kernel cuts equal units into parts (unit_part_tiles)
};

// D columns, D / 32 floats per lane; NW warps share the partials of one output row.
template <int D, int NW>
__global__ void __launch_bounds__(NW * 32) combine_kernel(const CombineParams p) {
    constexpr int kCombineWarps = NW;
    constexpr int VEC = D / 32;
    __shared__ float s_m[kCombineWarps], s_s[kCombineWarps];
    __shared__ float s_acc[kCombineWarps][D];

    const int u = blockIdx.x;                // unit = b * U + i
    const int r = blockIdx.y;                // row within the unit's head block
    const int b = u / p.units_per_seq;
    const int i = u % p.units_per_seq;
    const int j = i / p.n_hb;
    const int hb = i % p.n_hb;
    // row of the unit: query position qi and head hg of the group (qi-major)
    const int vr = hb * p.heads_per_unit + r;
    if (vr >= p.g * p.q_len) return;
    const int qi = vr / p.g, hg = vr - qi * p.g;
    const size_t gh = ((size_t)b * p.q_len + qi) * p.n_q + (size_t)j * p.g + hg;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int col = lane * VEC;

    // ---- the work split, from seq_lens (an input: readable before the decode grid ends)
    const int l0 = clamp_len(__ldg(p.seq_lens), p.T_max);
    const int t0 = tiles_of(l0 - active_start(l0, p.q_len, p.window), p.tile);
    int before = 0, all = 0, same = 1;
    for (int x = threadIdx.x; x < p.B; x += blockDim.x) {
        const int lx = clamp_len(__ldg(p.seq_lens + x), p.T_max);
        const int t = tiles_of(lx - active_start(lx, p.q_len, p.window), p.tile);
        all += t;
        same &= t == t0;
        if (x < b) before += t;
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
        before += __shfl_xor_sync(0xffffffffu, before, off);
        all += __shfl_xor_sync(0xffffffffu, all, off);
        same &= __shfl_xor_sync(0xffffffffu, same, off);
    }
    __shared__ int s_sum[3][kCombineWarps];
    if (lane == 0) { s_sum[0][warp] = before; s_sum[1][warp] = all; s_sum[2][warp] = same; }
    __syncthreads();
    before = 0;
    all = 0;
#pragma unroll
    for (int w = 0; w < kCombineWarps; ++w) { before += s_sum[0][w]; all += s_sum[1][w]; same &= s_sum[2][w]; }
    const int len_b = clamp_len(__ldg(p.seq_lens + b), p.T_max);
    const int n_tiles = tiles_of(len_b - active_start(len_b, p.q_len, p.window), p.tile);
    const long long W = tiles_per_worker((long long)all * p.units_per_seq, p.workers, p.min_tiles);
    if (n_tiles == 0) {
        // nothing of this unit was touched by the decode kernel
        for (int c = threadIdx.x; c < D; c += blockDim.x) p.out[gh * D + c] = 0.f;
        if (threadIdx.x == 0) p.lse[gh] = -INFINITY;
        return;
    }
    const long long ustart = (long long)before * p.units_per_seq + (long long)i * n_tiles;
    long long c_first = ustart / W;
    long long c_last = (ustart + n_tiles - 1) / W;
    bool parts = false;   // the decode kernel's unit parts: workers u k .. u k + ceil(n / Wu) - 1, slot 0
    if (p.unit_split && same) {
        int k = 0;
        const long long Wu = unit_part_tiles(t0, (long long)p.B * p.units_per_seq, p.workers, p.min_tiles, &k);
        if (Wu > 0) {
            parts = true;
            c_first = (long long)u * k;
            c_last = c_first + (t0 + Wu - 1) / Wu - 1;
        }
    }
    if (c_first == c_last) return;            // finished by its only worker

    pdl_wait_primary();
    float m = -INFINITY, S = 0.f;
    float acc[VEC];
#pragma unroll
    for (int v = 0; v < VEC; ++v) acc[v] = 0.f;
    constexpr int UNROLL = D >= 512 ? 4 : 8;
    for (long long c0 = c_first + warp; c0 <= c_last; c0 += (long long)kCombineWarps * UNROLL) {
        float ls[UNROLL];
        float ov[UNROLL][VEC];
#pragma unroll
        for (int q = 0; q < UNROLL; ++q) {
            const long long c = c0 + (long long)q * kCombineWarps;
            ls[q] = -INFINITY;
            if (c <= c_last) {
                const int slot = (parts || ustart <= c * W) ? 0 : 1;
                const size_t part = ((size_t)c * 2 + slot) * p.heads_per_unit + r;
                ls[q] = p.ws_lse[part];
                const float4 *src = reinterpret_cast<const float4 *>(p.ws_o + part * D + col);
#pragma unroll
                for (int v = 0; v < VEC / 4; ++v) {
                    const float4 x = src[v];
                    ov[q][4 * v] = x.x; ov[q][4 * v + 1] = x.y; ov[q][4 * v + 2] = x.z; ov[q][4 * v + 3] = x.w;
                }
                if (VEC % 4 != 0)
                    for (int v = (VEC / 4) * 4; v < VEC; ++v) ov[q][v] = p.ws_o[part * D + col + v];
            } else {
#pragma unroll
                for (int v = 0; v < VEC; ++v) ov[q][v] = 0.f;
            }
        }
#pragma unroll
        for (int q = 0; q < UNROLL; ++q) {
            if (ls[q] == -INFINITY) continue;
            const float mn = fmaxf(m, ls[q]);
            const float a = __expf(m - mn);       // 0 while m is still -inf
            const float w = __expf(ls[q] - mn);
            S = S * a + w;
#pragma unroll
            for (int v = 0; v < VEC; ++v) acc[v] = acc[v] * a + w * ov[q][v];
            m = mn;
        }
    }
    if (lane == 0) { s_m[warp] = m; s_s[warp] = S; }
#pragma unroll
    for (int v = 0; v < VEC; ++v) s_acc[warp][col + v] = acc[v];
    __syncthreads();
    if (warp != 0) return;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kCombineWarps; ++w) M = fmaxf(M, s_m[w]);
    float tot = 0.f;
    float res[VEC];
#pragma unroll
    for (int v = 0; v < VEC; ++v) res[v] = 0.f;
#pragma unroll
    for (int w = 0; w < kCombineWarps; ++w) {
        const float f = (s_m[w] == -INFINITY) ? 0.f : __expf(s_m[w] - M);
        tot += s_s[w] * f;
#pragma unroll
        for (int v = 0; v < VEC; ++v) res[v] += s_acc[w][col + v] * f;
    }
    // a row may have no visible position in any partial (a new token before the cache's
    // start): out 0, lse -inf
    const float inv = tot > 0.f ? 1.f / tot : 0.f;
#pragma unroll
    for (int v = 0; v < VEC; ++v) p.out[gh * D + col + v] = res[v] * inv;
    if (lane == 0) p.lse[gh] = tot > 0.f ? M + __logf(tot) : -INFINITY;
}

}  // namespace kvattn
