// gqa_decode.cuh -- split-KV decode attention for MHA / GQA / MQA on sm_100a.
//
// Each CTA is one persistent worker (schedule.cuh) that streams its range of KV tiles
// through shared memory once, whatever the group size: the K and V tiles of a KV head
// are loaded a single time and every query head of the group reads them there
// ("Attention variants: MQA, GQA, and MLA", section "Against the real libraries": index
// each query head into its group's KV tile instead of materialising the repeat).
//
// Warp roles (160 threads; 288 when the group needs two m-tiles):
//   last warp, lane 0  producer: TMA tiled loads (128-byte swizzle, no multicast) of the K
//                   and V tiles into an NST-stage ring guarded by full/empty mbarriers;
//                   the KV stream is tagged evict-first in L2.
//   other warps     consumers: the group's query heads are the M rows of warp-level
//                   m16n8k16 bf16 MMAs (16 heads per m-tile, zero rows when g < 16).
//                   Scores S = Q K^T and the update O += P V run on the tensor path;
//                   the online softmax (running max m, running sum l, rescale of O by
//                   2^(m_old - m_new)) runs in registers with quad shuffles.  P is split
//                   into a bf16 high part and a bf16 remainder and both are multiplied
//                   by V, which keeps the weights to ~16 significant bits.
// Warps split each tile's tokens (token slots); at the end of a piece their (m, l, O)
// are merged through shared memory and written as the final out/lse of the unit or as
// a partial for the combine kernel.
#pragma once
#include "common.cuh"
#include "schedule.cuh"

namespace kvattn {

struct GqaParams {
    const __nv_bfloat16 *q;     // [B, n_q, D]
    const int32_t *seq_lens;    // [B]
    float *out;                 // [B, n_q, D]
    float *lse;                 // [B, n_q]
    void *ws_meta;              // published decomposition (schedule.cuh)
    float *ws_lse;              // [workers, 2, HEADS]
    float *ws_o;                // [workers, 2, HEADS, D]
    int B, n_q, n_kv, T_max;
    int g;                      // group size n_q / n_kv
    int n_hb;                   // head blocks per group (ceil(g / HEADS))
    int workers;                // gridDim.x
    int min_tiles;
    float scale_log2;           // scale * log2(e)
    const int32_t *block_table; // [B, max_pages] physical pages (paged cache); null: contiguous
    int max_pages;              // block-table columns
    int page_size;              // rows per page (T_max when contiguous)
    int q_len;                  // new tokens per sequence (1: single-token decode)
    int window;                 // sliding window in tokens (0: none)
    float k_scale, v_scale;     // E4M3 cache: value = code * scale (1 for a bf16 cache)
    int unit_mode;              // warp kernel: worker u takes exactly unit u (no partials, no combine)
    int unit_split;             // tcgen05 kernel: unit parts when every unit has the same tiles
};

template <int D, int MT>
struct GqaCfg {
    static constexpr int TILE = 64;                       // tokens per pipeline stage
    static constexpr int NST = (D == 128) ? (MT == 1 ? 5 : 4) : 8;   // pipeline depth
    static constexpr int NCW = 4 * MT;                    // consumer warps (16 tokens each)
    static constexpr int NTHREADS = (NCW + 1) * 32;
    static constexpr int NTS = NCW / MT;                  // token slots per tile
    static constexpr int TOK_PER_WARP = TILE / NTS;       // 16 or 32
    static constexpr int HEADS = 16 * MT;                 // query heads per CTA
    static constexpr int CB = D / 64;                     // 128-byte column blocks
    static constexpr int KV_TILE_BYTES = TILE * D * 2;
    static constexpr int STAGE_BYTES = 2 * KV_TILE_BYTES;
    static constexpr int MERGE_FLOATS_PER_WARP = 16 * D + 32;
    static constexpr int MERGE_BYTES = NCW * MERGE_FLOATS_PER_WARP * 4 + HEADS * (NTS + 1) * 4;
    static constexpr int OFF_MERGE = NST * STAGE_BYTES;
    static constexpr int OFF_BARS = OFF_MERGE + MERGE_BYTES;
    static constexpr int OFF_CBAR = OFF_BARS + 2 * NST * 8;          // consumer barrier
    static constexpr int OFF_ABORT = OFF_CBAR + 8;
    static constexpr int OFF_PREFIX = OFF_ABORT + 16;
    static constexpr int smem_bytes(int B) { return 1024 + OFF_PREFIX + (B + 1) * 4; }
    static_assert(TOK_PER_WARP % 16 == 0, "token slot must hold whole 16-token MMA blocks");
};

// Byte address of element (row, col) of a [TILE x D] bf16 tile stored as D/64 column
// blocks of TILE rows x 128 bytes with the TMA 128-byte swizzle (16-byte chunk index
// XOR row % 8).  col must be a multiple of 8.
template <int TILE>
__device__ __forceinline__ uint32_t swz_addr(uint32_t base, int row, int col) {
    const int blk = col >> 6;
    const int chunk = (col & 63) >> 3;
    return base + blk * (TILE * 128) + row * 128 + ((chunk ^ (row & 7)) << 4);
}

template <int D, int MT>
__global__ void __launch_bounds__(GqaCfg<D, MT>::NTHREADS, 1)
gqa_decode_kernel(const GqaParams p, const __grid_constant__ CUtensorMap kmap,
                  const __grid_constant__ CUtensorMap vmap) {
    using C = GqaCfg<D, MT>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float *merge = reinterpret_cast<float *>(smem + C::OFF_MERGE);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::OFF_BARS);
    uint64_t *empty = full + C::NST;
    uint64_t *cbar = reinterpret_cast<uint64_t *>(smem + C::OFF_CBAR);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_ABORT);
    int *s_prefix = reinterpret_cast<int *>(smem + C::OFF_PREFIX);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int U = p.n_kv * p.n_hb;

    if (tid == 0) {
        for (int s = 0; s < C::NST; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], C::NCW);
        }
        mbar_init(cbar, C::NCW * 32);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) build_tile_prefix(p.seq_lens, p.B, p.T_max, C::TILE, s_prefix, lane);
    if (warp == C::NCW && lane == 0) {
        prefetch_tensormap(&kmap);
        prefetch_tensormap(&vmap);
    }
    __syncthreads();

    const long long total = (long long)s_prefix[p.B] * U;
    const long long W = tiles_per_worker(total, p.workers, p.min_tiles);
    if (blockIdx.x == 0 && !p.unit_mode) {
        MetaView mv = meta_view(p.ws_meta);
        if (tid == 0) { mv.w_total[0] = W; mv.w_total[1] = total; }
        for (int i = tid; i <= p.B; i += C::NTHREADS) mv.prefix[i] = s_prefix[i];
    }
    // The combine kernel may be scheduled now; it waits for this grid to finish.
    pdl_launch_dependents();

    long long p0 = (long long)blockIdx.x * W;
    long long p1 = (p0 + W < total) ? p0 + W : total;
    if (p.unit_mode) {
        // one worker per unit (B * U workers): the unit's own tile range, so that every
        // piece is the whole unit and is written as the final result; a unit without
        // tiles writes out = 0, lse = -inf for its rows
        const int u = blockIdx.x, b = u / U, i = u % U;
        const int n = s_prefix[b + 1] - s_prefix[b];
        p0 = (long long)s_prefix[b] * U + (long long)i * n;
        p1 = p0 + n;
        if (n == 0) {
            const int j = i / p.n_hb, hb = i % p.n_hb;
            for (int e = tid; e < C::HEADS * D; e += C::NTHREADS) {
                const int r = e / D, col = e - r * D;
                const int hg = hb * C::HEADS + r;
                if (hg >= p.g) continue;
                const size_t gh = (size_t)b * p.n_q + (size_t)j * p.g + hg;
                p.out[gh * D + col] = 0.f;
                if (col == 0) p.lse[gh] = -INFINITY;
            }
            return;
        }
    }
    if (p0 >= total) return;

    if (warp == C::NCW) {
        // ------------------------------------------------------------ producer
        if (lane != 0) return;
        const uint64_t pol = l2_policy_evict_first();
        int k = 0;
        bool ok = true;
        for (long long pos = p0; pos < p1 && ok;) {
            const Piece pc = piece_at(s_prefix, p.B, U, pos, p1, p0);
            const int len = clamp_len(__ldg(p.seq_lens + pc.b), p.T_max);
            const int j = pc.i / p.n_hb;
            for (int lt = pc.lt0; lt < pc.lt1; ++lt, ++k) {
                const int stage = k % C::NST;
                const uint32_t ph = (uint32_t)(k / C::NST) & 1u;
                if (!mbar_wait(&empty[stage], ph ^ 1u, FLAG_EMPTY_WAIT, abort_flag)) { ok = false; break; }
                mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
                const TileSrc src = tile_source(p.block_table, p.max_pages, p.page_size, pc.b, lt, C::TILE, len);
                const int y = src.y;
                const int z = src.page * p.n_kv + j;
                uint8_t *kt = smem + stage * C::STAGE_BYTES;
                uint8_t *vt = kt + C::KV_TILE_BYTES;
#pragma unroll
                for (int cb = 0; cb < C::CB; ++cb)
                    tma_load_3d(kt + cb * C::TILE * 128, &kmap, &full[stage], cb * 64, y, z, pol);
#pragma unroll
                for (int cb = 0; cb < C::CB; ++cb)
                    tma_load_3d(vt + cb * C::TILE * 128, &vmap, &full[stage], cb * 64, y, z, pol);
            }
            pos = pc.ustart + pc.lt1;
        }
        if (!ok) {
            // Let the copies already issued land before the CTA can exit.
            for (int kk = (k > C::NST ? k - C::NST : 0); kk < k; ++kk)
                mbar_wait(&full[kk % C::NST], (uint32_t)(kk / C::NST) & 1u, FLAG_FULL_WAIT, nullptr);
        }
        return;
    }

    // ---------------------------------------------------------------- consumers
    const int mt = warp % MT;
    const int ts = warp / MT;
    const int gid = lane >> 2;
    const int tig = lane & 3;
    const int mi = lane >> 3;
    const int rr = lane & 7;
    float *my_merge = merge + warp * C::MERGE_FLOATS_PER_WARP;   // O[16][D], m[16], l[16]
    float *wts = merge + C::NCW * C::MERGE_FLOATS_PER_WARP;      // [HEADS][NTS] weights, [HEADS] lse

    // Bounded barrier over the consumer warps (an mbarrier phase per use).
    uint32_t cbar_uses = 0;
    auto consumer_sync = [&]() -> bool {
        mbar_arrive(cbar);
        return __all_sync(0xffffffffu, mbar_wait(cbar, (cbar_uses++) & 1u, FLAG_FULL_WAIT, abort_flag)) != 0;
    };

    int k = 0;
    for (long long pos = p0; pos < p1;) {
        const Piece pc = piece_at(s_prefix, p.B, U, pos, p1, p0);
        pos = pc.ustart + pc.lt1;
        const int len = clamp_len(__ldg(p.seq_lens + pc.b), p.T_max);
        const int j = pc.i / p.n_hb;
        const int hb = pc.i % p.n_hb;
        const int head0 = hb * C::HEADS + mt * 16;     // first head of this m-tile, in the group

        // Q fragments (A operand) of this m-tile: rows = heads, cols = head dim.
        uint32_t qa[D / 16][4];
        {
            const int h0 = head0 + gid, h1 = head0 + gid + 8;
            const bool v0 = h0 < p.g, v1 = h1 < p.g;
            const uint32_t *q0 = reinterpret_cast<const uint32_t *>(
                p.q + ((size_t)pc.b * p.n_q + (size_t)j * p.g + (v0 ? h0 : 0)) * D);
            const uint32_t *q1 = reinterpret_cast<const uint32_t *>(
                p.q + ((size_t)pc.b * p.n_q + (size_t)j * p.g + (v1 ? h1 : 0)) * D);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const int c = (kk * 16 + tig * 2) >> 1;
                qa[kk][0] = v0 ? __ldg(q0 + c) : 0u;
                qa[kk][1] = v1 ? __ldg(q1 + c) : 0u;
                qa[kk][2] = v0 ? __ldg(q0 + c + 4) : 0u;
                qa[kk][3] = v1 ? __ldg(q1 + c + 4) : 0u;
            }
        }

        float o[D / 8][4];
#pragma unroll
        for (int nt = 0; nt < D / 8; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
        float m_run[2] = {-INFINITY, -INFINITY};
        float l_run[2] = {0.f, 0.f};
        bool aborted = false;

        for (int lt = pc.lt0; lt < pc.lt1; ++lt, ++k) {
            const int stage = k % C::NST;
            const uint32_t ph = (uint32_t)(k / C::NST) & 1u;
            // warp-uniform: the warp goes on to ldmatrix / mma.sync (warp-collective)
            if (!__all_sync(0xffffffffu, mbar_wait(&full[stage], ph, FLAG_FULL_WAIT, abort_flag))) {
                aborted = true;
                break;
            }
            const int y = min(lt * C::TILE, len - C::TILE);
            const int tok_lo = lt * C::TILE - y;                       // valid tile rows
            const int tok_hi = min((lt + 1) * C::TILE, len) - y;
            const uint32_t kbase = smem_u32(smem + stage * C::STAGE_BYTES);
            const uint32_t vbase = kbase + C::KV_TILE_BYTES;

#pragma unroll
            for (int sb = 0; sb < C::TOK_PER_WARP / 16; ++sb) {
                const int r0 = ts * C::TOK_PER_WARP + sb * 16;
                if (r0 >= tok_hi || r0 + 16 <= tok_lo) continue;      // warp-uniform
                // ---- S = Q K^T for 16 heads x 16 tokens
                float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    uint32_t b0, b1, b2, b3;
                    ldmatrix_x4(swz_addr<C::TILE>(kbase, r0 + (mi >> 1) * 8 + rr, kk * 16 + (mi & 1) * 8),
                                b0, b1, b2, b3);
                    mma_bf16_16816(s[0], qa[kk], b0, b1);
                    mma_bf16_16816(s[1], qa[kk], b2, b3);
                }
                // ---- scale, mask, online softmax (rows gid and gid + 8)
                float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const int row = r0 + nt * 8 + tig * 2 + (c & 1);
                        const bool valid = row >= tok_lo && row < tok_hi;
                        s[nt][c] = valid ? s[nt][c] * p.scale_log2 : -INFINITY;
                        mx[c >> 1] = fmaxf(mx[c >> 1], s[nt][c]);
                    }
                float alpha[2], mu[2];
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
                    mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
                    const float mnew = fmaxf(m_run[r], mx[r]);
                    mu[r] = (mnew == -INFINITY) ? 0.f : mnew;
                    alpha[r] = fast_exp2(m_run[r] - mu[r]);
                    m_run[r] = mnew;
                }
                float ls[2] = {0.f, 0.f};
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        s[nt][c] = fast_exp2(s[nt][c] - mu[c >> 1]);
                        ls[c >> 1] += s[nt][c];
                    }
                l_run[0] = l_run[0] * alpha[0] + ls[0];
                l_run[1] = l_run[1] * alpha[1] + ls[1];
#pragma unroll
                for (int nt = 0; nt < D / 8; ++nt) {
                    o[nt][0] *= alpha[0]; o[nt][1] *= alpha[0];
                    o[nt][2] *= alpha[1]; o[nt][3] *= alpha[1];
                }
                // ---- P as two bf16 A operands (high part + remainder)
                uint32_t pa_hi[4], pa_lo[4];
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    const float h0 = bf16_round(s[nt][0]), h1 = bf16_round(s[nt][1]);
                    const float h2 = bf16_round(s[nt][2]), h3 = bf16_round(s[nt][3]);
                    pa_hi[nt * 2 + 0] = pack_bf16x2(h0, h1);
                    pa_hi[nt * 2 + 1] = pack_bf16x2(h2, h3);
                    pa_lo[nt * 2 + 0] = pack_bf16x2(s[nt][0] - h0, s[nt][1] - h1);
                    pa_lo[nt * 2 + 1] = pack_bf16x2(s[nt][2] - h2, s[nt][3] - h3);
                }
                // ---- O += P V
#pragma unroll
                for (int nn = 0; nn < D / 16; ++nn) {
                    uint32_t b0, b1, b2, b3;
                    ldmatrix_x4_trans(swz_addr<C::TILE>(vbase, r0 + (mi & 1) * 8 + rr, nn * 16 + (mi >> 1) * 8),
                                      b0, b1, b2, b3);
                    mma_bf16_16816(o[2 * nn], pa_hi, b0, b1);
                    mma_bf16_16816(o[2 * nn], pa_lo, b0, b1);
                    mma_bf16_16816(o[2 * nn + 1], pa_hi, b2, b3);
                    mma_bf16_16816(o[2 * nn + 1], pa_lo, b2, b3);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage]);
        }
        if (aborted) return;

        // ---- merge the token slots of each m-tile and write the piece's result
        l_run[0] += __shfl_xor_sync(0xffffffffu, l_run[0], 1);
        l_run[0] += __shfl_xor_sync(0xffffffffu, l_run[0], 2);
        l_run[1] += __shfl_xor_sync(0xffffffffu, l_run[1], 1);
        l_run[1] += __shfl_xor_sync(0xffffffffu, l_run[1], 2);
#pragma unroll
        for (int nt = 0; nt < D / 8; ++nt) {
            *reinterpret_cast<float2 *>(my_merge + gid * D + nt * 8 + tig * 2) = make_float2(o[nt][0], o[nt][1]);
            *reinterpret_cast<float2 *>(my_merge + (gid + 8) * D + nt * 8 + tig * 2) = make_float2(o[nt][2], o[nt][3]);
        }
        if (tig == 0) {
            my_merge[16 * D + gid] = m_run[0];
            my_merge[16 * D + gid + 8] = m_run[1];
            my_merge[16 * D + 16 + gid] = l_run[0];
            my_merge[16 * D + 16 + gid + 8] = l_run[1];
        }
        if (!consumer_sync()) return;

        const int ctid = tid;   // 0 .. NCW*32-1
        if (ctid < C::HEADS) {
            const int r = ctid, rmt = r >> 4, rrow = r & 15;
            float M = -INFINITY;
#pragma unroll
            for (int t = 0; t < C::NTS; ++t)
                M = fmaxf(M, merge[(t * MT + rmt) * C::MERGE_FLOATS_PER_WARP + 16 * D + rrow]);
            const float Mu = (M == -INFINITY) ? 0.f : M;
            float L = 0.f;
            float w[C::NTS];
#pragma unroll
            for (int t = 0; t < C::NTS; ++t) {
                const float *mb = merge + (t * MT + rmt) * C::MERGE_FLOATS_PER_WARP + 16 * D;
                w[t] = fast_exp2(mb[rrow] - Mu);
                L += mb[16 + rrow] * w[t];
            }
            const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
            for (int t = 0; t < C::NTS; ++t) wts[r * C::NTS + t] = w[t] * inv;
            // natural-log lse of the (scaled) scores: (M + log2 L) * ln 2
            wts[C::HEADS * C::NTS + r] = L > 0.f ? (Mu + __log2f(L)) * 0.69314718055994531f : -INFINITY;
        }
        if (!consumer_sync()) return;

        const int j_heads = j * p.g;
        const size_t part = ((size_t)blockIdx.x * 2 + pc.slot) * C::HEADS;
        for (int idx = ctid; idx < C::HEADS * D; idx += C::NCW * 32) {
            const int r = idx / D, col = idx % D;
            const int hg = hb * C::HEADS + r;
            if (hg >= p.g) continue;
            const int rmt = r >> 4, rrow = r & 15;
            float v = 0.f;
#pragma unroll
            for (int t = 0; t < C::NTS; ++t)
                v += wts[r * C::NTS + t] * merge[(t * MT + rmt) * C::MERGE_FLOATS_PER_WARP + rrow * D + col];
            if (pc.whole) {
                const size_t gh = (size_t)pc.b * p.n_q + j_heads + hg;
                p.out[gh * D + col] = v;
                if (col == 0) p.lse[gh] = wts[C::HEADS * C::NTS + r];
            } else {
                p.ws_o[(part + r) * D + col] = v;
                if (col == 0) p.ws_lse[part + r] = wts[C::HEADS * C::NTS + r];
            }
        }
        if (!consumer_sync()) return;
    }
}

}  // namespace kvattn
