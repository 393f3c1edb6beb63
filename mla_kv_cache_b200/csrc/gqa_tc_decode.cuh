// gqa_tc_decode.cuh -- decode attention for query-head groups that share a KV head
// (GQA, MQA) on the sm_100a tensor cores (tcgen05, accumulators in tensor memory), with
// the cached tokens on the MMA rows.
//
// What it computes is what gqa_decode.cuh computes ("Attention variants: MQA, GQA, and
// MLA", sections "MQA: one KV head for everyone" and "GQA: interpolating with groups";
// "Grouped-Query Attention: Fewer KV Heads, Same Quality", "The Unified View"):
//     out[b, h] = softmax(scale * q[b, h] . K[b, j]^T) V[b, j],   j = h / g.
//
// Orientation.  A decode step has one query token per head, so the query side of a
// group is g rows while the token side of a KV tile is long.  Both products are taken
// transposed so that the 128 tokens of a tile fill the M = 128 rows of tcgen05.mma:
//     S^T[t, h]  = K[t, :] . q[h, :]          A = K tile (K-major), B = query block (K-major)
//     O^T[d, h] += sum_t V[t, d] P^T[t, h]    A = V tile read MN-major, B = P^T (MN-major)
// S^T and O^T live in tensor memory: TMEM lane t holds token t's scores for every head
// of the unit, lane d holds output dimension d of every head.  A unit is up to 64 query
// heads of one group (the N of the value product); the score product uses
// N = max(16, NR) where NR is the number of head columns the kernel processes.
//
// Per 128-token tile (one CTA per SM, persistent, stream-K over tiles, schedule.cuh):
//   producer (warp 0)   TMA loads of the K and V tiles (two 128-byte-swizzled boxes of
//                       [128 tokens x 64] each) into a 3-stage ring; the unit's query
//                       block once per piece, double-buffered when it has <= 32 heads.
//                       No multicast.
//   MMA (warp 1)        the score product of the next tile (8 MMAs 128 x N x 16) into one
//                       of two TMEM score buffers, then the value product of this tile
//                       (16 MMAs 128 x 64 x 16) into O^T; completion by tcgen05.commit.
//   softmax (warps 2-5) one thread per TMEM lane.  Per tile: scale and mask its token's
//                       scores, reduce the per-head maxima over the 128 tokens (a
//                       transposed shuffle reduction inside the warp, then the four warps
//                       through shared memory), let the owner thread of each head update
//                       its running max, and write P^T = 2^(s - m) into the K half of the
//                       stage (the score product is done with it) as a bf16 high part and
//                       a bf16 remainder; the value product multiplies V by both, so the
//                       weights keep ~16 significant bits.  The running max moves lazily:
//                       only when a head's tile maximum exceeds it by more than 2^8, and
//                       then that head's column of O^T and its row sums are rescaled.
// E4M3 cache (KV8).  A tile of K or V is one 128-byte-swizzled box of [128 tokens x 128
// codes]; the ring holds six 32 KB stages.  Both products run as kind::f8f6f4 MMAs on
// E4M3 operands straight from the TMA'd tiles, so nothing is converted per tile:
//   - the query block is split, once per piece and in place by the MMA warp, into an
//     E4M3 high part and an E4M3 remainder after scaling by 2^e (the block's largest
//     magnitude lands in [128, 256)); K times both parts, summed in the accumulator,
//     is K times the query to ~8 significant bits.  The score scale folds in the key
//     scale and 2^-e;
//   - P^T is written as an E4M3 high part and remainder of 64 * 2^(s - m) (the running
//     max moves once a head's tile maximum exceeds it by 2^2, so the weights stay in
//     E4M3's range), in the plain (unswizzled) MN-major layout: 16 heads x 128 tokens
//     per 2 KB block, one 16-byte row per token;
//   - V^T is the V tile read MN-major (128 dimensions = one 128-byte row per token);
//     the value scale and 1/64 fold into the final 1 / row sum.
// Each thread keeps its token slot's partial row sums per head; at the end of a piece
// they are reduced the same way and every thread writes its output dimension of every
// head (final output, or the worker's partial for the split combine).
//
// Every wait is bounded (common.cuh), including the softmax warps' own group barrier,
// which is an mbarrier rather than a named barrier so that it can give up.
#pragma once
#include "common.cuh"
#include "gqa_decode.cuh"
#include "schedule.cuh"
#include "tc05.cuh"

namespace kvattn {
namespace gqatc {

constexpr int TILE = 128;                 // tokens per tile = MMA M
constexpr int D = 128;                    // head dimension
constexpr int HB = 64;                    // query heads per unit (value-product N)
constexpr int CHUNK = TILE * 128;         // one [128 tokens x 128 bytes] box: 16 KB
constexpr int RING = 12 * CHUNK;          // the stage ring: 192 KB
constexpr int QREGION = 2 * HB * 128;     // query blocks: 16 KB (one of 64 heads or two of <= 32)
constexpr int NTHREADS_MAX = 320;         // producer, MMA, up to two groups of 4 softmax warps
constexpr uint32_t TM_S = 0;              // two score buffers
constexpr int NST_MAX = 6;
constexpr float P8_LOG2 = 6.f;            // E4M3 P^T holds 2^6 * 2^(s - m)

// Per cache type: bf16 (a tile is two [128 x 64] boxes, 3 stages of 64 KB) or E4M3
// (one [128 x 128] box, 6 stages of 32 KB).
template <bool KV8>
struct Kv {
    static constexpr int KV_BYTES = KV8 ? CHUNK : 2 * CHUNK;     // a K or V tile
    static constexpr int STAGE = 2 * KV_BYTES;                   // K then V
    static constexpr int NST = RING / STAGE;
    // the running max moves when a head's tile maximum exceeds it by 2^RESCALE
    static constexpr float RESCALE = KV8 ? 2.f : 8.f;
    // tensor memory: two score buffers (E4M3: the query's high-part and remainder
    // products side by side, 2 x NQ columns each), then O^T as two halves -- the value
    // product of the weights' high part and of their remainder -- summed at the end
    static constexpr uint32_t S_STRIDE = KV8 ? 128 : 64;
    static constexpr uint32_t TM_O = 2 * S_STRIDE;
    static constexpr uint32_t TM_COLS = KV8 ? 512 : 256;
    static_assert(NST <= NST_MAX, "stage barriers");
};

constexpr int OFF_ST = 0;
constexpr int OFF_Q = OFF_ST + RING;               // 196608
constexpr int OFF_RED = OFF_Q + QREGION;              // [4][4][64] fp32: tile maxima of groups 0/1, piece-end sums
constexpr int OFF_MS = OFF_RED + 4 * 4 * HB * 4;   // [2][64] running max after a group's latest tile
constexpr int OFF_ASO = OFF_MS + 2 * HB * 4;       // [2][64] rescale of O^T since the previous tile
constexpr int OFF_ASL = OFF_ASO + 2 * HB * 4;      // [2][64] rescale of a group's row sums
constexpr int OFF_NFO = OFF_ASL + 2 * HB * 4;      // [2][64] bytes: O^T column rescaled this tile
constexpr int OFF_NFL = OFF_NFO + 2 * HB;          // [2][64] bytes: row sum rescaled this tile
constexpr int OFF_MFIN = OFF_NFL + 2 * HB;         // [2][64] each group's last max (piece end)
constexpr int OFF_LINV = OFF_MFIN + 2 * HB * 4;    // [64] 1 / row sum
constexpr int OFF_QS = OFF_LINV + HB * 4;          // [2] fp32: 2^-e of each E4M3 query buffer
constexpr int OFF_BARS = OFF_QS + 16;
constexpr int OFF_TMEMPTR = OFF_BARS + 256;
constexpr int OFF_ABORT = OFF_TMEMPTR + 16;
constexpr int OFF_PREFIX = OFF_ABORT + 16;
constexpr int smem_bytes(int B) { return 1024 + OFF_PREFIX + (B + 1) * 4; }

struct Bars {
    uint64_t full[NST_MAX], empty[NST_MAX];
    uint64_t qfull[2];    // a query block landed (buffer = piece % NQB)
    uint64_t qempty[2];   // every score MMA of that piece has read it
    uint64_t qconv[2];    // E4M3 cache: the MMA warp has split that block (and its 2^-e)
    uint64_t sready[2];   // scores of a tile in TMEM buffer (tile & 1)
    uint64_t sfree[2];    // the softmax threads have read that buffer
    uint64_t pready[4];   // P^T of tile kt (index kt & 3) written, O^T rescaled: its value product may run
    uint64_t ofree;       // the epilogue has read O^T
    uint64_t grp[2];      // barrier of a softmax group's four warps
    uint64_t hand[2];     // running max after a tile of group g published (two groups)
    uint64_t all;         // barrier of every softmax warp (piece end)
};
static_assert(sizeof(Bars) <= 256, "barrier block overflows its slot");

template <int NR, bool KV8 = false>
struct Cfg {
    static_assert(NR == 8 || NR == 16 || NR == 32 || NR == 64, "head columns per unit");
    static constexpr int NQ = NR < 16 ? 16 : NR;           // score-product N (and columns read)
    static constexpr int RW = NR >= 32 ? NR / 32 : 1;      // values a lane holds after the reduction
    static constexpr int LPH = NR >= 32 ? 1 : 32 / NR;     // lanes holding the same head after it
    static constexpr int QCHUNK = NQ * 128;                // [NQ heads x 64] bf16 box
    static constexpr int QBLOCK = 2 * QCHUNK;              // one query block (head_dim 128)
    // query buffers: two when they fit, so that the next piece's block loads while the
    // current piece still reads its own
    static constexpr int NQB = 2 * QBLOCK <= QREGION ? 2 : 1;
    // softmax groups: two, taking alternate tiles, for 16 and 32 columns (where one
    // group's per-tile work paces the kernel) and for 8 over an E4M3 cache (half the bytes
    // per tile: 52.2 vs 56.3 us on the ragged GQA workload, 189 vs 200 us on MHA); one for
    // 8 over bf16 (the data's arrival paces it, measured) and for 64 (a thread's registers
    // do not allow 320 threads)
    static constexpr int NG = (NR == 16 || NR == 32 || (KV8 && NR == 8)) ? 2 : 1;
    static constexpr int NTHREADS = 64 + 128 * NG;
};

struct Ctx {
    uint8_t *smem;
    Bars *bars;
    volatile int *abort_flag;
    const int *s_prefix;
    uint32_t tmem;
    int U;
    long long p0, p1;
};

// One halving step of the transposed reduction: lanes whose bit `m` is set keep the
// upper W values, the others the lower W, and each adds (or takes the max of) the half
// its partner gave away.
template <int W, bool MAX>
__device__ __forceinline__ void xr_step(float *v, bool upper, int m) {
#pragma unroll
    for (int i = 0; i < W; ++i) {
        const float send = upper ? v[i] : v[W + i];
        const float keep = upper ? v[W + i] : v[i];
        const float got = __shfl_xor_sync(0xffffffffu, send, m);
        v[i] = MAX ? fmaxf(keep, got) : keep + got;
    }
}
// Reduces NR per-lane values over the 32 lanes of the warp, per column.  Afterwards
// lane l holds in v[i] the result for column RW * l + i (NR >= 32), or in v[0] the
// result for column l / LPH (NR < 32).  NR - 1 shuffles for NR >= 32.
template <int NR, bool MAX>
__device__ __forceinline__ void warp_xreduce(float (&v)[NR], int lane) {
    if constexpr (NR >= 2) xr_step<NR / 2, MAX>(v, (lane & 16) != 0, 16);
    if constexpr (NR >= 4) xr_step<NR / 4, MAX>(v, (lane & 8) != 0, 8);
    if constexpr (NR >= 8) xr_step<NR / 8, MAX>(v, (lane & 4) != 0, 4);
    if constexpr (NR >= 16) xr_step<NR / 16, MAX>(v, (lane & 2) != 0, 2);
    if constexpr (NR >= 32) xr_step<NR / 32, MAX>(v, (lane & 1) != 0, 1);
    if constexpr (NR < 32) {
#pragma unroll
        for (int m = 16 / NR; m >= 1; m >>= 1) {
            const float got = __shfl_xor_sync(0xffffffffu, v[0], m);
            v[0] = MAX ? fmaxf(v[0], got) : v[0] + got;
        }
    }
}
// Stores the warp's reduced columns into row[0..NR).
template <int NR>
__device__ __forceinline__ void store_reduced(float *row, const float (&v)[NR], int lane) {
    using C = Cfg<NR>;
    if constexpr (NR >= 32) {
#pragma unroll
        for (int i = 0; i < C::RW; ++i) row[C::RW * lane + i] = v[i];
    } else {
        if ((lane & (C::LPH - 1)) == 0) row[lane / C::LPH] = v[0];
    }
}

// One arrival per warp on a barrier the softmax warps share (initialised with a count of
// warps): the lanes meet first, so every lane's earlier writes and fences are ordered
// before lane 0's arrival, which releases them.  (128 single-thread arrivals on one
// barrier word cost several hundred cycles per barrier.)
__device__ __forceinline__ void warp_arrive(uint64_t *bar, int lane) {
    __syncwarp();
    if (lane == 0) mbar_arrive(bar);
}

// NQ consecutive TMEM columns of this thread's lane.
template <int NQ>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&v)[NQ]) {
    if constexpr (NQ == 16) {
        tmem_ld16(taddr, v);
    } else if constexpr (NQ == 32) {
        tmem_ld32(taddr, v);
    } else {
        uint32_t a[32], b[32];
        tmem_ld32(taddr, a);
        tmem_ld32(taddr + 32, b);
#pragma unroll
        for (int i = 0; i < 32; ++i) { v[i] = a[i]; v[32 + i] = b[i]; }
    }
}
// ------------------------------------------------------------------ producer (warp 0, lane 0)
template <int NR, bool KV8>
__device__ __forceinline__ void producer(const GqaParams &p, const CUtensorMap *kmap, const CUtensorMap *vmap,
                                         const CUtensorMap *qmap, const Ctx &c) {
    using C = Cfg<NR>;
    using L = Kv<KV8>;
    constexpr int NST = L::NST;
    Bars *bars = c.bars;
    const uint64_t pol = l2_policy_evict_first();
    int k = 0, pi = 0;
    bool ok = true;
    for (long long pos = c.p0; pos < c.p1 && ok; ++pi) {
        const Piece pc = piece_at(c.s_prefix, p.B, c.U, pos, c.p1, c.p0);
        pos = pc.ustart + pc.lt1;
        const int len = clamp_len(__ldg(p.seq_lens + pc.b), p.T_max);
        const int j = pc.i / p.n_hb, hb = pc.i % p.n_hb;
        const int qb = pi % C::NQB, qu = pi / C::NQB;
        if (qu > 0 && !mbar_wait(&bars->qempty[qb], (uint32_t)(qu - 1) & 1u, FLAG_EMPTY_WAIT, c.abort_flag)) {
            ok = false;
            break;
        }
        const int qrow = j * p.g + hb * HB;
        uint8_t *qdst = c.smem + OFF_Q + qb * C::QBLOCK;
        if (p.q_len == 1) {
            mbar_arrive_expect_tx(&bars->qfull[qb], C::QBLOCK);
            tma_load_3d(qdst, qmap, &bars->qfull[qb], 0, qrow, pc.b, pol);
            tma_load_3d(qdst + C::QCHUNK, qmap, &bars->qfull[qb], 64, qrow, pc.b, pol);
        } else {
            // several new tokens: rows (position qi, head h) = the g heads of the group at
            // each of the q_len positions, qi-major (a 4-D box of q[B, q_len, n_q, d])
            const uint32_t bytes = 2u * (uint32_t)(p.g * p.q_len) * 128u;
            mbar_arrive_expect_tx(&bars->qfull[qb], bytes);
            tma_load_4d(qdst, qmap, &bars->qfull[qb], 0, j * p.g, 0, pc.b, pol);
            tma_load_4d(qdst + C::QCHUNK, qmap, &bars->qfull[qb], 64, j * p.g, 0, pc.b, pol);
        }
        const int start = active_start(len, p.q_len, p.window);
        for (int lt = pc.lt0; lt < pc.lt1; ++lt, ++k) {
            const int s = k % NST;
            const uint32_t ph = (uint32_t)(k / NST) & 1u;
            if (!mbar_wait(&bars->empty[s], ph ^ 1u, FLAG_EMPTY_WAIT, c.abort_flag)) { ok = false; break; }
            mbar_arrive_expect_tx(&bars->full[s], L::STAGE);
            const TileSrc src = tile_source(p.block_table, p.max_pages, p.page_size, pc.b, lt, TILE, len, start);
            const int y = src.y;
            const int z = src.page * p.n_kv + j;
            uint8_t *st = c.smem + OFF_ST + s * L::STAGE;
            if constexpr (KV8) {
                // one 128-byte box per tile (the map sees a row as 64 two-byte elements)
                tma_load_3d(st, kmap, &bars->full[s], 0, y, z, pol);
                tma_load_3d(st + L::KV_BYTES, vmap, &bars->full[s], 0, y, z, pol);
            } else {
                tma_load_3d(st, kmap, &bars->full[s], 0, y, z, pol);
                tma_load_3d(st + CHUNK, kmap, &bars->full[s], 64, y, z, pol);
                tma_load_3d(st + L::KV_BYTES, vmap, &bars->full[s], 0, y, z, pol);
                tma_load_3d(st + L::KV_BYTES + CHUNK, vmap, &bars->full[s], 64, y, z, pol);
            }
        }
    }
    if (!ok) {
        // Let every copy already issued land before the CTA can exit.
        for (int kk = (k > NST ? k - NST : 0); kk < k; ++kk)
            mbar_wait_sleep(&bars->full[kk % NST], (uint32_t)(kk / NST) & 1u, FLAG_FULL_WAIT, nullptr);
        for (int pp = (pi > C::NQB ? pi - C::NQB : 0); pp < pi; ++pp)
            mbar_wait_sleep(&bars->qfull[pp % C::NQB], (uint32_t)(pp / C::NQB) & 1u, FLAG_FULL_WAIT, nullptr);
    }
}

// ------------------------------------------------------------------ E4M3 query split (warp 1)
// Splits the bf16 query block at qbase (two 128-byte-swizzled [NQ x 64] boxes) in place
// into two E4M3 blocks of [NQ x 128] in the same swizzle: the high parts where the first
// box was, the remainders where the second was.  Every value is first multiplied by
// 2^e, e chosen so that the block's largest magnitude lands in [128, 256).  Run by the
// 32 lanes of one warp; returns 2^-e.  Row h of both boxes holds only row h's data, so
// rows are independent: lanes take eight rows at a time (four lanes a row, 32
// dimensions each), read everything they need, meet, then write.
template <int NQ>
__device__ __forceinline__ float split_query_e4m3(uint8_t *qbase, int lane) {
    constexpr int QCHUNK = NQ * 128;
    float amax = 0.f;
    const uint4 *src = reinterpret_cast<const uint4 *>(qbase);
    for (int i = lane; i < 2 * QCHUNK / 16; i += 32) {
        const uint4 u = src[i];
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(w[t])), fabsf(bf16_hi(w[t]))));
    }
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, m));
    int e = 0;
    if (amax > 0.f && amax <= 3.0e38f) {
        int x;
        frexpf(amax, &x);                 // amax in [2^(x-1), 2^x)
        e = min(max(8 - x, -126), 126);
    }
    const float up = __int_as_float((127 + e) << 23);
    const float down = __int_as_float((127 - e) << 23);
    const int m = lane & 3;               // dimensions 32m .. 32m + 31
    const int chunk = m >> 1;             // in bf16 box m / 2, 16-byte units 4 (m & 1) .. + 3
#pragma unroll 1
    for (int g0 = 0; g0 < NQ; g0 += 8) {
        const int h = g0 + (lane >> 2);
        const int sw = h & 7;
        const uint8_t *row = qbase + chunk * QCHUNK + h * 128;
        uint4 in[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) in[j] = *reinterpret_cast<const uint4 *>(row + (((4 * (m & 1) + j) ^ sw) << 4));
        __syncwarp();
        uint32_t hw[8], lw[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t w[4] = {in[j].x, in[j].y, in[j].z, in[j].w};
#pragma unroll
            for (int t = 0; t < 4; t += 2) {
                uint16_t h0, l0, h1, l1;
                split_e4m3x2(bf16_lo(w[t]) * up, bf16_hi(w[t]) * up, h0, l0);
                split_e4m3x2(bf16_lo(w[t + 1]) * up, bf16_hi(w[t + 1]) * up, h1, l1);
                hw[2 * j + t / 2] = (uint32_t)h0 | ((uint32_t)h1 << 16);
                lw[2 * j + t / 2] = (uint32_t)l0 | ((uint32_t)l1 << 16);
            }
        }
        // E4M3 16-byte units 2m and 2m + 1 of row h (dimensions 32m .. 32m + 31)
        uint8_t *hrow = qbase + h * 128;
        uint8_t *lrow = qbase + QCHUNK + h * 128;
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int slot = ((2 * m + u) ^ sw) << 4;
            *reinterpret_cast<uint4 *>(hrow + slot) = make_uint4(hw[4 * u], hw[4 * u + 1], hw[4 * u + 2], hw[4 * u + 3]);
            *reinterpret_cast<uint4 *>(lrow + slot) = make_uint4(lw[4 * u], lw[4 * u + 1], lw[4 * u + 2], lw[4 * u + 3]);
        }
        __syncwarp();
    }
    return down;
}

// ------------------------------------------------------------------ MMA issuer (warp 1, lane 0)
// Score product of tile kt into TMEM buffer (kt & 1).  The caller has seen the tile
// land and the buffer freed.
template <int NR, bool KV8>
__device__ __forceinline__ void issue_scores(const Ctx &c, int kt, int qbuf) {
    using C = Cfg<NR>;
    using L = Kv<KV8>;
    const int s = kt % L::NST, sb = kt & 1;
    tc_fence_after();
    const uint32_t st = smem_u32(c.smem + OFF_ST + s * L::STAGE);
    const uint32_t qb = smem_u32(c.smem + OFF_Q + qbuf * C::QBLOCK);
    if constexpr (KV8) {
        // K (E4M3, [128 tokens x 128], K-major) times the query's high part and its
        // remainder at once: the two blocks are consecutive 128-byte rows, so N = 2 NQ
        // and the tile is read once (4 MMAs of K = 32); TMEM columns [0, NQ) get the
        // high-part scores, [NQ, 2 NQ) the remainder's
        constexpr uint32_t idesc = idesc_e4m3(128, 2 * Cfg<NR>::NQ, 0, 0);
#pragma unroll
        for (int kk = 0; kk < D / 32; ++kk) {
            const uint64_t a = smem_desc_sw128(st + kk * 32, 16, 1024);
            const uint64_t b = smem_desc_sw128(qb + kk * 32, 16, 1024);
            umma_ss_f8(c.tmem + TM_S + L::S_STRIDE * sb, a, b, idesc, kk ? 1u : 0u);
        }
    } else {
        constexpr uint32_t idesc = idesc_f16_major(128, Cfg<NR>::NQ, 1, 1, 0, 0);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t blk = kk >> 2, in = (kk & 3) * 32;
            const uint64_t a = smem_desc_sw128(st + blk * CHUNK + in, 16, 1024);
            const uint64_t b = smem_desc_sw128(qb + blk * C::QCHUNK + in, 16, 1024);
            umma_ss(c.tmem + TM_S + L::S_STRIDE * sb, a, b, idesc, kk > 0 ? 1u : 0u);
        }
    }
    umma_commit(&c.bars->sready[sb]);
}

// Value product of tile kt into O^T (first = the piece's first tile: overwrite).
template <int NR, bool KV8>
__device__ __forceinline__ void issue_values(const Ctx &c, int kt, bool first) {
    using L = Kv<KV8>;
    const int s = kt % L::NST;
    tc_fence_after();
    const uint32_t st = smem_u32(c.smem + OFF_ST + s * L::STAGE);
    if constexpr (KV8) {
        // V^T: M = 128 dimensions (one 128-byte row per token, MN-major), K = 32 tokens;
        // P^T: N = 2 NQ columns -- the high parts' 16-head blocks, then the remainders',
        // 2 KB apart, 16 bytes per token (plain MN-major: 8-token core matrices 128
        // bytes apart); the tile is read once (4 MMAs)
        constexpr int NQ = Cfg<NR>::NQ;
        constexpr uint32_t idesc_pv = idesc_e4m3(128, 2 * NQ, 1, 1);
#pragma unroll
        for (int kk = 0; kk < TILE / 32; ++kk) {
            const uint64_t a = smem_desc_sw128(st + L::KV_BYTES + kk * 4096, CHUNK, 1024);
            const uint64_t b = smem_desc_plain(st + kk * 512, 128, 2048);
            umma_ss_f8(c.tmem + L::TM_O, a, b, idesc_pv, (!first || kk) ? 1u : 0u);
        }
    } else {
        constexpr uint32_t idesc_pv = idesc_f16_major(128, 2 * HB, 1, 1, 1, 1);
#pragma unroll
        for (int kk = 0; kk < TILE / 16; ++kk) {
            // V^T: M = 128 dimensions in two 64-wide blocks 16 KB apart, K = 16 tokens
            const uint64_t a = smem_desc_sw128(st + L::KV_BYTES + kk * 2048, CHUNK, 1024);
            // P^T (in the K half of the stage): N = 128 columns, the high part's 64 heads
            // and the remainder's 64, two 64-wide blocks 16 KB apart; the tile is read once
            const uint64_t b = smem_desc_sw128(st + kk * 2048, CHUNK, 1024);
            umma_ss(c.tmem + L::TM_O, a, b, idesc_pv, (!first || kk > 0) ? 1u : 0u);
        }
    }
    umma_commit(&c.bars->empty[s]);   // frees the stage; also tells the softmax that O^T has this tile
}

// The issuer never blocks on one product while the other could go: it tests whether
// the next score product (its tile landed, its TMEM buffer free) or the next value
// product (P^T written; at a piece start, O^T read out) may run and issues whatever is
// ready.  Score products run at most three tiles ahead of value products, so a softmax
// group finds its next tile's scores waiting when it finishes a tile (the two TMEM score
// buffers are guarded by sfree); with four P^T-ready barriers (tile & 3) every tested
// barrier stays within one phase of the tested parity.  A value product ends with one
// commit, on its stage's empty barrier, which the softmax warps also wait on before they
// touch O^T (a commit costs the issuing thread ~300 cycles).  Idle time is bounded like
// every other wait.  The whole warp runs the
// loop over pieces (with an E4M3 cache its 32 lanes split each query block); lane 0
// alone issues.
template <int NR, bool KV8>
__device__ __forceinline__ void mma_issuer(const GqaParams &p, const Ctx &c, int lane) {
    using L = Kv<KV8>;
    constexpr int NST = L::NST;
    Bars *bars = c.bars;
    int k = 0, pi = 0;
    for (long long pos = c.p0; pos < c.p1; ++pi) {
        const Piece pc = piece_at(c.s_prefix, p.B, c.U, pos, c.p1, c.p0);
        pos = pc.ustart + pc.lt1;
        const int nt = pc.lt1 - pc.lt0;
        const int qb = pi % Cfg<NR>::NQB, qu = pi / Cfg<NR>::NQB;
        if (!warp_all(mbar_wait(&bars->qfull[qb], (uint32_t)qu & 1u, FLAG_FULL_WAIT, c.abort_flag))) return;
        if constexpr (KV8) {
            const float down = split_query_e4m3<Cfg<NR>::NQ>(c.smem + OFF_Q + qb * Cfg<NR>::QBLOCK, lane);
            if (lane == 0) reinterpret_cast<float *>(c.smem + OFF_QS)[qb] = down;
            fence_proxy_async_smem();
            mbar_arrive(&bars->qconv[qb]);
            __syncwarp();
        }
        int failed = 0;
        if (lane == 0) {
            int nq = 0, nv = 0;
            long long idle_since = clock64();
            while (nv < nt) {
                bool progressed = false;
                if (nq < nt && nq < nv + 3) {
                    const int kt = k + nq;
                    if (mbar_test(&bars->full[kt % NST], (uint32_t)(kt / NST) & 1u) &&
                        (kt < 2 || mbar_test(&bars->sfree[kt & 1], (uint32_t)((kt >> 1) - 1) & 1u))) {
                        issue_scores<NR, KV8>(c, kt, qb);
                        ++nq;
                        if (nq == nt) umma_commit(&bars->qempty[qb]);
                        progressed = true;
                    }
                }
                if (nv < nq) {
                    const int kt = k + nv;
                    if (mbar_test(&bars->pready[kt & 3], (uint32_t)(kt >> 2) & 1u) &&
                        (nv > 0 || pi == 0 || mbar_test(&bars->ofree, (uint32_t)(pi - 1) & 1u))) {
                        issue_values<NR, KV8>(c, kt, nv == 0);
                        ++nv;
                        progressed = true;
                    }
                }
                if (progressed) {
                    idle_since = clock64();
                } else {
                    if (*c.abort_flag) { failed = 1; break; }
                    if (clock64() - idle_since > kWaitLimitCycles) {
                        atomicOr(&g_device_flags, FLAG_MMA_WAIT);
                        *c.abort_flag = 1;
                        failed = 1;
                        break;
                    }
                }
            }
        }
        if (__shfl_sync(0xffffffffu, failed, 0)) return;
        k += nt;
    }
}

// ------------------------------------------------------------------ softmax (warps 2 ..)
// NG groups of four warps (one thread per TMEM lane each).  With two groups, group g
// takes the tiles kt with kt % 2 == g (and the score buffer g), so one group's tile
// overlaps the other's; the running max of each column is handed from group to group
// through shared memory (ms[g]) and the hand[g] barriers -- the one serial step.  Each
// group keeps its own row sums, relative to the max it last used; at the end of a piece
// they are merged at the final max.  O^T is rescaled, in tile order, by the factor
// between consecutive tiles' maxima.
// MULTI: several new tokens or a window (the per-column visibility mask and the
// (position, head) output rows); without it the kernel keeps the single-token forms --
// a compile-time split, because the multi-token code in the same kernel costs the
// single-token MQA workload ~4 us per step (measured) even where it does not run.
template <int NR, bool KV8, bool MULTI>
__device__ __forceinline__ void softmax_warps(const GqaParams &p, const Ctx &c, int warp, int lane) {
    using C = Cfg<NR, KV8>;
    using L = Kv<KV8>;
    constexpr int NQ = C::NQ;
    constexpr int NST = L::NST;
    constexpr int NG = C::NG;
    constexpr int NOWN = (NR + 31) / 32;            // warps holding owner threads
    constexpr uint32_t O_LO = KV8 ? NQ : HB;     // column of O^T's remainder half
    Bars *bars = c.bars;
    const int g = (warp - 2) >> 2;        // group
    const int wg = (warp - 2) & 3;        // warp within the group
    const int q = warp & 3;               // TMEM lane quadrant
    const int r = 32 * q + lane;          // token row of a tile / output dimension
    const int st_id = wg * 32 + lane;     // owner index (column) within the group
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    float *red = reinterpret_cast<float *>(c.smem + OFF_RED);
    float *ms = reinterpret_cast<float *>(c.smem + OFF_MS);
    float *aso = reinterpret_cast<float *>(c.smem + OFF_ASO);
    float *asl = reinterpret_cast<float *>(c.smem + OFF_ASL);
    uint8_t *nfo = c.smem + OFF_NFO;
    uint8_t *nfl = c.smem + OFF_NFL;
    float *mfin = reinterpret_cast<float *>(c.smem + OFF_MFIN);
    float *linv = reinterpret_cast<float *>(c.smem + OFF_LINV);
    uint32_t grp_uses = 0, all_uses = 0;
    auto grp_sync = [&]() -> bool {
        warp_arrive(&bars->grp[g], lane);
        const bool ok = mbar_wait(&bars->grp[g], grp_uses & 1u, FLAG_FULL_WAIT, c.abort_flag);
        ++grp_uses;
        return warp_all(ok);
    };
    auto all_sync = [&]() -> bool {
        warp_arrive(&bars->all, lane);
        const bool ok = mbar_wait(&bars->all, all_uses & 1u, FLAG_FULL_WAIT, c.abort_flag);
        ++all_uses;
        return warp_all(ok);
    };

    int k = 0, pi = 0;
    for (long long pos = c.p0; pos < c.p1; ++pi) {
        const Piece pc = piece_at(c.s_prefix, p.B, c.U, pos, c.p1, c.p0);
        pos = pc.ustart + pc.lt1;
        const int len = clamp_len(__ldg(p.seq_lens + pc.b), p.T_max);
        const int j = pc.i / p.n_hb, hb = pc.i % p.n_hb;
        const int nt = pc.lt1 - pc.lt0;
        const int start = active_start(len, p.q_len, p.window);
        // columns of one query position (the group's heads); all columns of the unit
        const uint64_t group_bits = (!MULTI || p.g >= 64) ? ~0ull : ((1ull << p.g) - 1ull);
        // score scale (log2 units); with an E4M3 cache also the key scale and the 2^-e
        // of the split query block
        float cs = p.scale_log2;
        if constexpr (KV8) {
            const int qb = pi % C::NQB, qu = pi / C::NQB;
            if (!warp_all(mbar_wait(&bars->qconv[qb], (uint32_t)qu & 1u, FLAG_MMA_WAIT, c.abort_flag))) return;
            cs *= p.k_scale * reinterpret_cast<const float *>(c.smem + OFF_QS)[qb];
        }
        float m_own = -INFINITY;              // max of column st_id this group last used (owners)
        float l_part[NR];
#pragma unroll
        for (int h = 0; h < NR; ++h) l_part[h] = 0.f;

        for (int t = NG == 1 ? 0 : ((g - k) & 1); t < nt; t += NG) {
            const int kt = k + t;
            const int s = kt % NST, sb = kt & 1;
            const int lt = pc.lt0 + t;
            // tile row r holds position y + r (the last tile is shifted back to end at len;
            // its rows before tok0 belong to the previous tile)
            const int tok0 = start + lt * TILE;
            const int y = min(tok0, len - TILE);
            const int posr = y + r;
            // the columns (query position qi, head) that may see this token: query qi sits
            // at len - q_len + qi and sees [that + 1 - window, that] (causal, windowed)
            uint64_t vis = 0;
            const bool in_tile = posr >= tok0 && posr < len;
            if constexpr (MULTI) {
                if (in_tile) {
                    for (int qi = 0; qi < p.q_len; ++qi) {
                        const int hi = len - p.q_len + qi + 1;
                        const int lo = p.window > 0 ? hi - p.window : 0;
                        if (posr < hi && posr >= lo) vis |= group_bits << (qi * p.g);
                    }
                }
            }
            // ---- this token's scores
            if (!warp_all(mbar_wait(&bars->sready[sb], (uint32_t)(kt >> 1) & 1u, FLAG_MMA_WAIT, c.abort_flag)))
                return;
            tc_fence_after();
            uint32_t sv[NQ];
            if constexpr (KV8) {
                // high-part and remainder scores, added (16 columns at a time)
#pragma unroll
                for (int c0 = 0; c0 < NQ; c0 += 16) {
                    uint32_t a16[16], b16[16];
                    tmem_ld16(c.tmem + lane_base + TM_S + L::S_STRIDE * sb + c0, a16);
                    tmem_ld16(c.tmem + lane_base + TM_S + L::S_STRIDE * sb + NQ + c0, b16);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        sv[c0 + i] = __float_as_uint(__uint_as_float(a16[i]) + __uint_as_float(b16[i]));
                }
            } else {
                tmem_ld_cols<NQ>(c.tmem + lane_base + TM_S + L::S_STRIDE * sb, sv);
                tmem_wait_ld();
            }
            tc_fence_before();
            warp_arrive(&bars->sfree[sb], lane);
            float sc[NR], v[NR];
#pragma unroll
            for (int h = 0; h < NR; ++h) {
                const bool see = MULTI ? ((vis >> h) & 1ull) != 0 : in_tile;
                sc[h] = see ? __uint_as_float(sv[h]) * cs : -INFINITY;
                v[h] = sc[h];
            }
            // ---- per-column maximum over the tile's 128 tokens
            warp_xreduce<NR, true>(v, lane);
            store_reduced<NR>(red + (g * 4 + q) * HB, v, lane);
            if (!grp_sync()) return;
            // ---- owners: the running max after this tile (from the previous tile's, which
            //      the other group handed over), the rescale of O^T since the previous
            //      tile and of this group's row sums since its own previous tile
            if (st_id < NR) {
                const float tm = fmaxf(fmaxf(red[(g * 4 + 0) * HB + st_id], red[(g * 4 + 1) * HB + st_id]),
                                       fmaxf(red[(g * 4 + 2) * HB + st_id], red[(g * 4 + 3) * HB + st_id]));
                float m_prev = m_own;
                if (NG == 2 && t > 0) {
                    if (!mbar_wait(&bars->hand[g ^ 1], (uint32_t)((kt - 1) >> 1) & 1u, FLAG_FULL_WAIT, c.abort_flag))
                        m_prev = -INFINITY;   // (abandoned: the group's next wait fails too)
                    else
                        m_prev = ms[(g ^ 1) * HB + st_id];
                }
                const float m_new = (t == 0 || tm > m_prev + L::RESCALE) ? tm : m_prev;
                const bool need_o = t > 0 && m_new != m_prev;
                const bool need_l = m_own != m_new && m_own != -INFINITY;
                ms[g * HB + st_id] = m_new;
                aso[g * HB + st_id] = need_o ? fast_exp2(m_prev - m_new) : 1.f;
                asl[g * HB + st_id] = need_l ? fast_exp2(m_own - m_new) : 1.f;
                nfo[g * HB + st_id] = need_o;
                nfl[g * HB + st_id] = need_l;
                m_own = m_new;
            }
            if (NG == 2 && wg < NOWN) warp_arrive(&bars->hand[g], lane);
            if (!grp_sync()) return;
            if (*c.abort_flag) return;
            // ---- weights: P^T row r, high part and remainder, into the stage's K half
            uint32_t any_o = 0, any_l = 0;
#pragma unroll
            for (int h = 0; h < NR; h += 4) {
                any_o |= *reinterpret_cast<const uint32_t *>(nfo + g * HB + h);
                any_l |= *reinterpret_cast<const uint32_t *>(nfl + g * HB + h);
            }
            if (any_l != 0) {
                const float *a = asl + g * HB;
#pragma unroll
                for (int h = 0; h < NR; h += 4) {
                    const float4 x = *reinterpret_cast<const float4 *>(a + h);
                    l_part[h] *= x.x; l_part[h + 1] *= x.y; l_part[h + 2] *= x.z; l_part[h + 3] *= x.w;
                }
            }
            const float *msg = ms + g * HB;
            uint8_t *st = c.smem + OFF_ST + s * L::STAGE;
            if constexpr (KV8) {
                // 16 heads per 16-byte row of a 2 KB block, the remainders' blocks after the
                // high parts' (NQ / 16 blocks each); heads past NR are zero
#pragma unroll
                for (int cb = 0; cb < NQ / 16; ++cb) {
                    uint32_t hw[4] = {0u, 0u, 0u, 0u}, lw[4] = {0u, 0u, 0u, 0u};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int h = 16 * cb + 4 * e;
                        if (h < NR) {
                            float a[4];
#pragma unroll
                            for (int u = 0; u < 4; ++u) {
                                const float mu = msg[h + u];
                                // 2^6 * 2^(s - m), summed in the same units
                                a[u] = fast_exp2(sc[h + u] - (mu == -INFINITY ? 0.f : mu) + P8_LOG2);
                                l_part[h + u] += a[u];
                            }
                            uint16_t h0, l0, h1, l1;
                            split_e4m3x2(a[0], a[1], h0, l0);
                            split_e4m3x2(a[2], a[3], h1, l1);
                            hw[e] = (uint32_t)h0 | ((uint32_t)h1 << 16);
                            lw[e] = (uint32_t)l0 | ((uint32_t)l1 << 16);
                        }
                    }
                    *reinterpret_cast<uint4 *>(st + cb * 2048 + r * 16) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                    *reinterpret_cast<uint4 *>(st + NQ * 128 + cb * 2048 + r * 16) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
                }
            } else {
                uint8_t *hrow = st + r * 128;
                uint8_t *lrow = st + CHUNK + r * 128;
#pragma unroll
                for (int cc = 0; cc < NR / 8; ++cc) {
                    uint32_t hw[4], lw[4];
                    const float4 m0 = *reinterpret_cast<const float4 *>(msg + 8 * cc);
                    const float4 m1 = *reinterpret_cast<const float4 *>(msg + 8 * cc + 4);
                    // (a column with no visible token so far has max -inf; its weights are 0)
                    float mh[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
#pragma unroll
                    for (int e = 0; e < 8; ++e) mh[e] = mh[e] == -INFINITY ? 0.f : mh[e];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int h = 8 * cc + 2 * e;
                        const float a = fast_exp2(sc[h] - mh[2 * e]);
                        const float b = fast_exp2(sc[h + 1] - mh[2 * e + 1]);
                        l_part[h] += a;
                        l_part[h + 1] += b;
                        split_bf16x2(a, b, hw[e], lw[e]);
                    }
                    const int slot = (cc ^ (r & 7)) << 4;
                    *reinterpret_cast<uint4 *>(hrow + slot) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                    *reinterpret_cast<uint4 *>(lrow + slot) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
                }
            }
            fence_proxy_async_smem();
            // ---- rescale the affected columns of O^T (after the previous tile's value product)
            if (any_o != 0) {
                if (!warp_all(mbar_wait(&bars->empty[(kt - 1) % NST], (uint32_t)((kt - 1) / NST) & 1u, FLAG_MMA_WAIT,
                                        c.abort_flag)))
                    return;
                tc_fence_after();
                const float *a = aso + g * HB;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
#pragma unroll
                    for (int c0 = 0; c0 < NQ; c0 += 16) {
                        const uint32_t col = L::TM_O + half * O_LO + c0;
                        uint32_t ov[16];
                        tmem_ld16(c.tmem + lane_base + col, ov);
                        tmem_wait_ld();
#pragma unroll
                        for (int h = 0; h < 16; h += 4) {
                            if (c0 + h < NR) {
                                const float4 x = *reinterpret_cast<const float4 *>(a + c0 + h);
                                ov[h] = __float_as_uint(__uint_as_float(ov[h]) * x.x);
                                ov[h + 1] = __float_as_uint(__uint_as_float(ov[h + 1]) * x.y);
                                ov[h + 2] = __float_as_uint(__uint_as_float(ov[h + 2]) * x.z);
                                ov[h + 3] = __float_as_uint(__uint_as_float(ov[h + 3]) * x.w);
                            }
                        }
                        tmem_st16(c.tmem + lane_base + col, ov);
                    }
                }
                tmem_wait_st();
            }
            tc_fence_before();
            warp_arrive(&bars->pready[kt & 3], lane);
        }
        k += nt;

        // ---- end of the piece: the groups' row sums (merged at the final max), lse, output
        float v[NR];
#pragma unroll
        for (int h = 0; h < NR; ++h) v[h] = l_part[h];
        warp_xreduce<NR, false>(v, lane);
        store_reduced<NR>(red + ((2 + g) * 4 + q) * HB, v, lane);
        if (st_id < NR) mfin[g * HB + st_id] = m_own;
        if (!all_sync()) return;
        // columns of the unit: (query position qi, head h of the group), qi-major; output
        // row of column cc in out [B, q_len, n_q, d] / lse [B, q_len, n_q]
        const int h_real = min(HB, p.g * p.q_len - hb * HB);
        const size_t part = ((size_t)blockIdx.x * 2 + pc.slot) * HB;
        auto out_row = [&](int cc) -> size_t {
            if constexpr (!MULTI) return (size_t)pc.b * p.n_q + (size_t)j * p.g + (size_t)hb * HB + cc;
            const int vr = hb * HB + cc;
            const int qi = vr / p.g;
            return ((size_t)pc.b * p.q_len + qi) * p.n_q + (size_t)j * p.g + (vr - qi * p.g);
        };
        if (g == 0 && st_id < NR) {
            float M = -INFINITY, l = 0.f, lg[NG], mg[NG];
#pragma unroll
            for (int x = 0; x < NG; ++x) {
                lg[x] = red[((2 + x) * 4 + 0) * HB + st_id] + red[((2 + x) * 4 + 1) * HB + st_id] +
                        red[((2 + x) * 4 + 2) * HB + st_id] + red[((2 + x) * 4 + 3) * HB + st_id];
                mg[x] = mfin[x * HB + st_id];
                M = fmaxf(M, mg[x]);
            }
#pragma unroll
            for (int x = 0; x < NG; ++x)
                if (lg[x] > 0.f) l += mg[x] == M ? lg[x] : lg[x] * fast_exp2(mg[x] - M);
            // (E4M3 cache: l and O^T both carry 2^6; the value scale enters here)
            linv[st_id] = l > 0.f ? (KV8 ? p.v_scale : 1.f) / l : 0.f;
            const float lse_v =
                l > 0.f ? (M + __log2f(l) - (KV8 ? P8_LOG2 : 0.f)) * 0.69314718055994531f : -INFINITY;
            if (st_id < h_real) {
                if (pc.whole)
                    p.lse[out_row(st_id)] = lse_v;
                else
                    p.ws_lse[part + st_id] = lse_v;
            }
        }
        if (!all_sync()) return;
        const int klast = k - 1;
        if (!warp_all(mbar_wait(&bars->empty[klast % NST], (uint32_t)(klast / NST) & 1u, FLAG_MMA_WAIT, c.abort_flag)))
            return;
        tc_fence_after();
        // 16-column chunks of O^T, taken by the groups in turn
#pragma unroll
        for (int c0 = 0; c0 < NQ; c0 += 16) {
            if ((c0 / 16) % NG != g) continue;
            uint32_t ov[16], ol[16];
            tmem_ld16(c.tmem + lane_base + L::TM_O + c0, ov);
            tmem_ld16(c.tmem + lane_base + L::TM_O + O_LO + c0, ol);
            tmem_wait_ld();
#pragma unroll
            for (int h = 0; h < 16; ++h) {
                const int cc = c0 + h;
                if (cc < NR && cc < h_real) {
                    float *dst = pc.whole ? p.out + out_row(cc) * D : p.ws_o + (part + cc) * D;
                    dst[r] = (__uint_as_float(ov[h]) + __uint_as_float(ol[h])) * linv[cc];
                }
            }
        }
        tc_fence_before();
        warp_arrive(&bars->ofree, lane);
    }
}

}  // namespace gqatc

template <int NR, bool KV8, bool MULTI>
__global__ void __launch_bounds__(gqatc::Cfg<NR, KV8>::NTHREADS, 1)
gqa_tc_decode_kernel(const GqaParams p, const __grid_constant__ CUtensorMap kmap,
                     const __grid_constant__ CUtensorMap vmap, const __grid_constant__ CUtensorMap qmap) {
    using namespace gqatc;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Bars *bars = reinterpret_cast<Bars *>(smem + OFF_BARS);
    uint32_t *tmem_ptr = reinterpret_cast<uint32_t *>(smem + OFF_TMEMPTR);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + OFF_ABORT);
    int *s_prefix = reinterpret_cast<int *>(smem + OFF_PREFIX);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int U = p.n_kv * p.n_hb;

    if (tid == 0) {
        for (int s = 0; s < Kv<KV8>::NST; ++s) {
            mbar_init(&bars->full[s], 1);
            mbar_init(&bars->empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars->qfull[i], 1);
            mbar_init(&bars->qempty[i], 1);
            mbar_init(&bars->qconv[i], 32);
        }
        constexpr int NG = Cfg<NR, KV8>::NG;
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars->sready[i], 1);
            mbar_init(&bars->sfree[i], 4);        // the four warps of the tile's group
            mbar_init(&bars->pready[i], 4);
            mbar_init(&bars->pready[2 + i], 4);
            mbar_init(&bars->grp[i], 4);
            mbar_init(&bars->hand[i], (NR + 31) / 32);   // the group's warps holding owners
        }
        mbar_init(&bars->ofree, 4 * NG);
        mbar_init(&bars->all, 4 * NG);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_ptr), Kv<KV8>::TM_COLS);
        tmem_relinquish();
    }
    if (warp == 2) build_tile_prefix(p.seq_lens, p.B, p.T_max, TILE, s_prefix, lane, p.q_len, p.window);
    // query buffers start zeroed: rows a unit's block does not fill stay finite (a
    // single-token block is a full box: the TMA fills its rows past the heads with zeros)
    if constexpr (MULTI)
        for (int i = tid; i < QREGION / 16; i += Cfg<NR, KV8>::NTHREADS)
            reinterpret_cast<uint4 *>(smem + OFF_Q)[i] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&kmap);
        prefetch_tensormap(&vmap);
        prefetch_tensormap(&qmap);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    Ctx c;
    c.smem = smem;
    c.bars = bars;
    c.abort_flag = abort_flag;
    c.s_prefix = s_prefix;
    c.tmem = *tmem_ptr;
    c.U = U;
    const long long total = (long long)s_prefix[p.B] * U;
    const long long W = tiles_per_worker(total, p.workers, p.min_tiles);
    if (blockIdx.x == 0) {
        MetaView mv = meta_view(p.ws_meta);
        if (tid == 0) { mv.w_total[0] = W; mv.w_total[1] = total; }
        for (int i = tid; i <= p.B; i += Cfg<NR, KV8>::NTHREADS) mv.prefix[i] = s_prefix[i];
    }
    // The combine kernel may be scheduled now; it waits for this grid to finish.
    pdl_launch_dependents();
    c.p0 = (long long)blockIdx.x * W;
    c.p1 = (c.p0 + W < total) ? c.p0 + W : total;
    if (p.unit_split) {   // equal units: consecutive parts of one unit per worker (schedule.cuh)
        const int n_uni = uniform_tile_count(s_prefix, p.B);
        const long long units = (long long)p.B * U;
        int k = 0;
        const long long Wu = unit_part_tiles(n_uni, units, p.workers, p.min_tiles, &k);
        if (Wu > 0) {
            const long long u = blockIdx.x / k, i = blockIdx.x % k, ub = u * n_uni;
            c.p0 = total;
            c.p1 = total;
            if (u < units && i * Wu < n_uni) {
                c.p0 = ub + i * Wu;
                c.p1 = (i + 1) * Wu < n_uni ? c.p0 + Wu : ub + n_uni;
            }
        }
    }

    if (c.p0 < total) {
        if (warp == 0) {
            if (lane == 0) producer<NR, KV8>(p, &kmap, &vmap, &qmap, c);
        } else if (warp == 1) {
            mma_issuer<NR, KV8>(p, c, lane);
        } else {
            softmax_warps<NR, KV8, MULTI>(p, c, warp, lane);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(c.tmem, Kv<KV8>::TM_COLS);
    }
}

}  // namespace kvattn
