// mla_decode.cuh -- absorbed multi-head latent attention decode (latent 512 + RoPE 64)
// on sm_100a tensor cores (tcgen05, accumulators and operands in tensor memory).
//
// What it computes ("Attention variants: MQA, GQA, and MLA", section "MLA: cache a
// latent, not the keys and values"): with the key up-projection folded into the query,
// head h of sequence b scores every cached token t as
//     s[h,t] = scale * (q_lat[h] . c_t + q_rope[h] . r_t)
// and returns out[h] = sum_t softmax(s[h])_t * c_t, a 512-wide latent (the value
// up-projection is applied by the caller) -- one shared 576-wide key row per token,
// whose first 512 elements are also the value.
//
// Why a CTA pair.  The fp32 accumulator of 128 heads x 512 latent columns is 256 KB,
// all of one SM's tensor memory.  A 2-CTA cluster therefore splits the latent columns:
// CTA r holds columns [256r, 256r + 256) of every cached row (CTA 0 also the 64 RoPE
// columns) and the accumulator O_r = P * C[:, 256r..] (128 x 256 fp32, 256 TMEM columns).
// Each CTA computes partial scores over its part of the 576-wide contraction, stages
// them in a local send buffer, and one bulk copy per tile (distributed shared memory,
// issued by warp 2) moves them into the other CTA's receive buffer, completing its
// mbarrier's transaction count; both CTAs add the two partials in the same order and run
// the identical online softmax, so P, the rescale factors and the row sums never cross
// the pair.  Every cached byte is loaded from HBM once; every MMA is M = 128.
//
// Tensor memory of a CTA (512 columns): O_r [0, 256), the partial scores S_r of one
// tile [256, 320), the latent part of Q_r as bf16 pairs [320, 448), and P of one tile
// [448, 512): its bf16 high part (32 columns, the top 16 bits of each fp32 weight) and
// bf16 remainder (32 columns).  The
// value product runs twice, O_r += P_hi C_r + P_lo C_r, so the weights keep ~16
// significant bits while the cache stays in its bf16 form (no conversion pass).
//
// Per 64-token tile and CTA:
//   TMA (warp 0)       4 (CTA 0: 5) 128-byte-swizzled boxes [64 tokens x 64 columns]
//                      into a 3-stage ring; CTA 0 also the q_rope block once per piece.
//   send (warp 2)      one bulk copy per tile of the staged partial scores to the peer.
//   MMA (warp 1)       S_r = Q_r C_r^T: 16 MMAs 128x64x16 with A from TMEM (CTA 0: 4 more
//                      with the RoPE query from shared memory); O_r += P C_r: 8 MMAs
//                      128x256x16 with A = P from TMEM and C_r read MN-major from the same
//                      swizzled tile.  It issues whichever product is ready.
//   softmax (warps 4-11) two warpgroups (one per TMEM lane quadrant) take the
//                      tiles in turn, so one group's exchange and exponentials overlap
//                      the other's.  A thread owns one head row of its group's tiles: it
//                      reads the row's 64 partial scores, sends them to the peer, adds the
//                      peer's, masks, and takes the tile maximum.  The running max is
//                      handed from group to group through shared memory (the only serial
//                      step); it moves lazily, only when a tile's maximum exceeds it by
//                      more than 2^8, and then this row of O_r is rescaled in TMEM.  The
//                      thread writes P = 2^(s - m) into TMEM and keeps its group's row sum.
// At the end of a piece the two groups merge their row sums, and each normalises half
// of the row's 256 output columns from TMEM and writes the final result or the worker's
// partial for the split combine.
#pragma once
#include "common.cuh"
#include "schedule.cuh"
#include "tc05.cuh"

namespace kvattn {
namespace mla {

constexpr int TILE = 64;                 // tokens per tile (the MMA N of the score product)
constexpr int HR = 128;                  // head rows (MMA M)
constexpr int NCH = 5;                   // 64-column chunks per stage slot (CTA 0 uses 5)
constexpr int NST = 3;                   // pipeline stages
constexpr int CHUNK_T = TILE * 128;      // one [64 tokens x 64 cols] bf16 box: 8 KB
constexpr int STAGE = NCH * CHUNK_T;     // 40 KB
constexpr int QROPE = HR * 128;          // q_rope block [128 heads x 64] bf16: 16 KB
constexpr int NTHREADS = 384;            // warpgroup 0: producer, MMA, sender (1 idle warp); 1, 2: softmax groups
constexpr int REGS_WG0 = 96;             // registers per thread after reallocation: warpgroup 0
constexpr int REGS_SOFTMAX = 200;        //   softmax warpgroups (128 x 96 + 256 x 200 <= 384 x 168)
constexpr int NGROUP = 128;              // threads per softmax group
constexpr int MAX_BATCH = 1024;
constexpr uint32_t TM_O = 0;             // TMEM columns [0, 256): O_r
constexpr uint32_t TM_S = 256;           // [256, 320): partial scores of one tile
constexpr uint32_t TM_Q = 320;           // [320, 448): latent part of Q_r (bf16 pairs)
constexpr uint32_t TM_P = 448;           // [448, 480): P high part, [480, 512): remainder
constexpr uint32_t TM_COLS = 512;
constexpr float RESCALE_LOG2 = 8.f;      // rescale O only when the row max grows by > 2^8
constexpr uint32_t RECV_BYTES = HR * TILE * 4;   // the peer's partial scores of one tile

constexpr int OFF_ST = 0;
constexpr int OFF_QROPE = OFF_ST + NST * STAGE;          // 122880
constexpr int OFF_RECV = OFF_QROPE + QROPE;              // 139264: [128 heads][64] fp32 from the peer
constexpr int OFF_SEND = OFF_RECV + (int)RECV_BYTES;     // 172032: [128 heads][64] fp32 to the peer
constexpr int OFF_MREF = OFF_RECV + 2 * (int)RECV_BYTES; // 204800: [2][128] running max
constexpr int OFF_LX = OFF_MREF + 2 * HR * 4;            // [2][128] row sums of the groups
constexpr int OFF_BARS = OFF_LX + 2 * HR * 4;            // 206848
constexpr int OFF_TMEMPTR = OFF_BARS + 256;
constexpr int OFF_ABORT = OFF_TMEMPTR + 16;     // abort flag; +8: tiles whose send buffer the sender has read
constexpr int OFF_PREFIX = OFF_ABORT + 16;
constexpr int smem_bytes(int B) { return 1024 + OFF_PREFIX + (B + 1) * 4; }

struct Bars {
    uint64_t full[NST], empty[NST];
    uint64_t qready;       // latent part of Q_r written into TMEM (both groups)
    uint64_t qrope_full;   // q_rope block landed in shared memory (TMA, CTA 0)
    uint64_t qempty;       // every score MMA of the piece has read Q
    uint64_t sready[2];    // partial scores of a tile (parity) in TMEM
    uint64_t sfree;        // the tile's group has read them
    uint64_t recv_full[2]; // the peer's partial scores of a tile of group g landed (armed by g)
    uint64_t peer_rfree;   // the peer has consumed the tile this CTA last sent (4 remote arrivals)
    uint64_t staged;       // a tile's partial scores written into the send buffer (4 warps)
    uint64_t hand[2];      // running max of a tile (parity) published
    uint64_t pready;       // P of a tile in TMEM and O rescaled: the value product may run
    uint64_t odone[2];     // value product of a tile (parity) finished
    uint64_t ofree;        // the epilogue has read O
    uint64_t lx;           // the groups' row sums exchanged (end of a piece)
};
static_assert(sizeof(Bars) <= 256, "barrier block overflows its slot");

}  // namespace mla

struct MlaParams {
    const __nv_bfloat16 *q_latent;   // [B, H, 512]
    const __nv_bfloat16 *q_rope;     // [B, H, 64]
    const int32_t *seq_lens;
    float *out;        // [B, H, 512]
    float *lse;        // [B, H]
    void *ws_meta;
    float *ws_lse;     // [workers, 2, 128]
    float *ws_o;       // [workers, 2, 128, 512]
    int B, H, T_max;
    int workers;       // clusters
    int min_tiles;
    float scale_log2;
    const int32_t *block_table; // [B, max_pages] physical pages (paged cache); null: contiguous
    int max_pages;              // block-table columns
    int page_size;              // rows per page (T_max when contiguous)
};

struct MlaMaps {
    CUtensorMap lat, rope, qlat, qrope;
};

namespace mla {

struct Ctx {
    uint8_t *smem;
    Bars *bars;
    volatile int *abort_flag;
    const int *s_prefix;
    uint32_t tmem;
    uint32_t r, peer;
    int worker;
    long long p0, p1;
};

// ------------------------------------------------------------------ producer (warp 0, lane 0)
__device__ __forceinline__ void producer(const MlaParams &p, const MlaMaps &m, const Ctx &c) {
    Bars *bars = c.bars;
    const uint64_t pol = l2_policy_evict_first();
    const int nch = c.r == 0 ? 5 : 4;
    int k = 0, pi = 0;
    bool ok = true;
    for (long long pos = c.p0; pos < c.p1 && ok; ++pi) {
        const Piece pc = piece_at(c.s_prefix, p.B, 1, pos, c.p1, c.p0);
        pos = pc.ustart + pc.lt1;
        const int len = clamp_len(__ldg(p.seq_lens + pc.b), p.T_max);
        if (c.r == 0) {
            // the RoPE part of this sequence's queries (the score MMAs read it from here)
            if (pi > 0 && !mbar_wait(&bars->qempty, (uint32_t)(pi - 1) & 1u, FLAG_EMPTY_WAIT, c.abort_flag)) {
                ok = false;
                break;
            }
            mbar_arrive_expect_tx(&bars->qrope_full, QROPE);
            tma_load_3d(c.smem + OFF_QROPE, &m.qrope, &bars->qrope_full, 0, 0, pc.b, pol);
        }
        for (int lt = pc.lt0; lt < pc.lt1; ++lt, ++k) {
            const int s = k % NST;
            const uint32_t ph = (uint32_t)(k / NST) & 1u;
            if (!mbar_wait(&bars->empty[s], ph ^ 1u, FLAG_EMPTY_WAIT, c.abort_flag)) { ok = false; break; }
            mbar_arrive_expect_tx(&bars->full[s], nch * CHUNK_T);
            const TileSrc src = tile_source(p.block_table, p.max_pages, p.page_size, pc.b, lt, TILE, len);
            uint8_t *st = c.smem + OFF_ST + s * STAGE;
            for (int ch = 0; ch < 4; ++ch)
                tma_load_3d(st + ch * CHUNK_T, &m.lat, &bars->full[s], 256 * (int)c.r + 64 * ch, src.y, src.page,
                            pol);
            if (c.r == 0) tma_load_3d(st + 4 * CHUNK_T, &m.rope, &bars->full[s], 0, src.y, src.page, pol);
        }
    }
    if (!ok) {
        // Let every copy already issued land before the CTA can exit.
        for (int kk = (k > NST ? k - NST : 0); kk < k; ++kk)
            mbar_wait_sleep(&bars->full[kk % NST], (uint32_t)(kk / NST) & 1u, FLAG_FULL_WAIT, nullptr);
        if (c.r == 0 && pi > 0) mbar_wait_sleep(&bars->qrope_full, (uint32_t)(pi - 1) & 1u, FLAG_FULL_WAIT, nullptr);
    }
}

// ------------------------------------------------------------------ MMA issuer (warp 1, lane 0)
// Partial scores of tile kt: latent chunks with A = Q_r from TMEM, the RoPE chunk (CTA 0)
// with A = q_rope from shared memory.  The caller has seen the tile land and S freed.
__device__ __forceinline__ void issue_scores(const Ctx &c, int kt) {
    const int s = kt % NST;
    tc_fence_after();
    constexpr uint32_t idesc = idesc_f16(128, TILE, 1, 1, 0);
    const uint32_t st = smem_u32(c.smem + OFF_ST + s * STAGE);
    for (int ch = 0; ch < 4; ++ch)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            const uint64_t bd = smem_desc_sw128(st + ch * CHUNK_T + kk * 32, 16, 1024);
            umma_ts(c.tmem + TM_S, c.tmem + TM_Q + ch * 32 + kk * 8, bd, idesc, (ch | kk) != 0);
        }
    if (c.r == 0) {
        const uint32_t qr = smem_u32(c.smem + OFF_QROPE);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = smem_desc_sw128(qr + kk * 32, 16, 1024);
            const uint64_t bd = smem_desc_sw128(st + 4 * CHUNK_T + kk * 32, 16, 1024);
            umma_ss(c.tmem + TM_S, ad, bd, idesc, 1u);
        }
    }
    umma_commit(&c.bars->sready[kt & 1]);
}

// O_r += P C_r for tile kt: 4 token blocks of 16, high part then remainder of P.
__device__ __forceinline__ void issue_values(const Ctx &c, int kt, bool first) {
    const int s = kt % NST;
    tc_fence_after();
    constexpr uint32_t idesc = idesc_f16(128, 256, 1, 1, 1);
    const uint32_t st = smem_u32(c.smem + OFF_ST + s * STAGE);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
        const uint64_t bd = smem_desc_sw128(st + kk * 2048, CHUNK_T, 1024);
        umma_ts(c.tmem + TM_O, c.tmem + TM_P + kk * 8, bd, idesc, (!first || kk > 0) ? 1u : 0u);
        umma_ts(c.tmem + TM_O, c.tmem + TM_P + 32 + kk * 8, bd, idesc, 1u);
    }
    umma_commit(&c.bars->empty[s]);
    umma_commit(&c.bars->odone[kt & 1]);
}

// Issues the value product of the oldest scored tile (P written; at a piece start, O
// read out) or the score product of the next tile (tile landed, the previous tile's
// scores read), whichever is ready -- the value product first, it is on the softmax
// groups' critical path -- never blocking on one while the other could go.
// Idle time is bounded like every other wait.
__device__ __forceinline__ void mma_issuer(const MlaParams &p, const Ctx &c) {
    Bars *bars = c.bars;
    int k = 0, pi = 0;
    for (long long pos = c.p0; pos < c.p1; ++pi) {
        const Piece pc = piece_at(c.s_prefix, p.B, 1, pos, c.p1, c.p0);
        pos = pc.ustart + pc.lt1;
        const int nt = pc.lt1 - pc.lt0;
        if (!mbar_wait(&bars->qready, (uint32_t)pi & 1u, FLAG_FULL_WAIT, c.abort_flag)) return;
        if (c.r == 0 && !mbar_wait(&bars->qrope_full, (uint32_t)pi & 1u, FLAG_FULL_WAIT, c.abort_flag)) return;
        int nq = 0, nv = 0;
        long long idle_since = clock64();
        while (nv < nt) {
            bool progressed = false;
            if (nv < nq) {
                const int kt = k + nv;
                if (mbar_test(&bars->pready, (uint32_t)kt & 1u) &&
                    (nv > 0 || pi == 0 || mbar_test(&bars->ofree, (uint32_t)(pi - 1) & 1u))) {
                    issue_values(c, kt, nv == 0);
                    ++nv;
                    progressed = true;
                }
            }
            if (nq < nt && nq < nv + NST) {
                const int kt = k + nq;
                if (mbar_test(&bars->full[kt % NST], (uint32_t)(kt / NST) & 1u) &&
                    (kt == 0 || mbar_test(&bars->sfree, (uint32_t)(kt - 1) & 1u))) {
                    issue_scores(c, kt);
                    ++nq;
                    if (nq == nt) umma_commit(&bars->qempty);   // the piece's last score MMAs
                    progressed = true;
                }
            }
            if (progressed) {
                idle_since = clock64();
            } else {
                if (*c.abort_flag) return;
                if (clock64() - idle_since > kWaitLimitCycles) {
                    atomicOr(&g_device_flags, FLAG_MMA_WAIT);
                    *c.abort_flag = 1;
                    return;
                }
            }
        }
        k += nt;
    }
}

// Monotone count of tiles whose send buffer the bulk copy has read (a counter, not an
// mbarrier: the two groups wait on it for alternate tiles, so a phase parity could be
// two phases behind one of them).
__device__ __forceinline__ void publish_count(int *cnt, int v) {
    asm volatile("st.release.cta.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(cnt)), "r"(v) : "memory");
}
__device__ __forceinline__ int read_count(const int *cnt) {
    int v;
    asm volatile("ld.acquire.cta.shared::cta.b32 %0, [%1];" : "=r"(v) : "r"(smem_u32(cnt)) : "memory");
    return v;
}
// Bounded wait until the count reaches `target`.
__device__ __forceinline__ bool wait_count(const int *cnt, int target, unsigned int flag, volatile int *abort) {
    if (read_count(cnt) >= target) return true;
    const long long t0 = clock64();
    while (true) {
        if (read_count(cnt) >= target) return true;
        if (abort != nullptr && *abort) return false;
        if (clock64() - t0 > kWaitLimitCycles) {
            atomicOr(&g_device_flags, flag);
            if (abort != nullptr) *abort = 1;
            return false;
        }
    }
}

// ------------------------------------------------------------------ sender (warp 2, lane 0)
// Ships each tile's partial scores to the peer: once the tile's group has staged them in
// the send buffer and the peer has consumed the previous tile, one bulk copy moves the
// 32 KB into the peer's receive buffer and completes the transaction count of the
// peer's recv_full barrier of the tile's group; the send buffer is released (the count)
// as soon as the copy has read it.  (Per-thread remote stores of the same bytes took
// ~2.8 us per tile.)
__device__ __forceinline__ void sender(const MlaParams &p, const Ctx &c) {
    Bars *bars = c.bars;
    const uint32_t src = smem_u32(c.smem + OFF_SEND);
    const uint32_t dst = map_to_rank(smem_u32(c.smem + OFF_RECV), c.peer);
    const uint32_t dst_bar0 = map_to_rank(smem_u32(&bars->recv_full[0]), c.peer);
    const uint32_t dst_bar1 = map_to_rank(smem_u32(&bars->recv_full[1]), c.peer);
    int *sent = reinterpret_cast<int *>(c.smem + OFF_ABORT + 8);
    int k = 0;
    for (long long pos = c.p0; pos < c.p1;) {
        const Piece pc = piece_at(c.s_prefix, p.B, 1, pos, c.p1, c.p0);
        pos = pc.ustart + pc.lt1;
        for (int t = 0; t < pc.lt1 - pc.lt0; ++t, ++k) {
            if (!mbar_wait(&bars->staged, (uint32_t)k & 1u, FLAG_FULL_WAIT, c.abort_flag)) return;
            if (k > 0 && !mbar_wait_cluster(&bars->peer_rfree, (uint32_t)(k - 1) & 1u, FLAG_PEER_WAIT, c.abort_flag))
                return;
            bulk_copy_to_peer(dst, src, RECV_BYTES, (k & 1) ? dst_bar1 : dst_bar0);
            bulk_commit_group();
            bulk_wait_read_all();
            publish_count(sent, k + 1);
        }
    }
}

// 16-byte chunk slot of chunk j (columns 4j..4j+3) in row h of a receive buffer.
__device__ __forceinline__ int recv_chunk(int j, int h) { return j ^ (h & 7); }

// ------------------------------------------------------------------ softmax (warps 4-11)
__device__ __forceinline__ void softmax_warps(const MlaParams &p, const Ctx &c, int warp, int lane) {
    Bars *bars = c.bars;
    const int g = (warp - 4) >> 2;              // group: takes the tiles k with k % 2 == g
    const int q = warp & 3;                     // TMEM lane quadrant
    const int h = 32 * q + lane;                // head row
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    const float *recv = reinterpret_cast<const float *>(c.smem + OFF_RECV) + h * TILE;
    uint8_t *send = c.smem + OFF_SEND + h * TILE * 4;
    const uint32_t peer_rfree = map_to_rank(smem_u32(&bars->peer_rfree), c.peer);
    float *mref = reinterpret_cast<float *>(c.smem + OFF_MREF);
    float *lx = reinterpret_cast<float *>(c.smem + OFF_LX);

    int k = 0, pi = 0;
    for (long long pos = c.p0; pos < c.p1; ++pi) {
        const Piece pc = piece_at(c.s_prefix, p.B, 1, pos, c.p1, c.p0);
        pos = pc.ustart + pc.lt1;
        const int len = clamp_len(__ldg(p.seq_lens + pc.b), p.T_max);
        const int nt = pc.lt1 - pc.lt0;
        // ---- latent part of Q_r into TMEM (lane h = head h; bf16 pairs per column):
        //      128 words per row, group g writes words [64g, 64g + 64)
        if (pi > 0 && !warp_all(mbar_spin<false>(&bars->qempty, (uint32_t)(pi - 1) & 1u, FLAG_MMA_WAIT, c.abort_flag)))
            return;
        {
            const bool real = h < p.H;
            const uint32_t *ql = reinterpret_cast<const uint32_t *>(p.q_latent) +
                                 ((size_t)pc.b * p.H + (real ? h : 0)) * 256 + 128 * c.r + 64 * g;
            tc_fence_after();
#pragma unroll
            for (int w = 0; w < 64; w += 32) {
                uint32_t v[32];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    uint4 x = make_uint4(0, 0, 0, 0);
                    if (real) x = __ldg(reinterpret_cast<const uint4 *>(ql + w + 4 * j));
                    v[4 * j] = x.x; v[4 * j + 1] = x.y; v[4 * j + 2] = x.z; v[4 * j + 3] = x.w;
                }
                tmem_st32(c.tmem + lane_base + TM_Q + 64 * g + w, v);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bars->qready);
        }
        float m_last = -INFINITY;     // reference of this group's row sum
        float l_g = 0.f;              // this group's row sum (tiles of the piece it took)
        const int k0 = k;
        for (int t = (g - k0) & 1; t < nt; t += 2) {
            const int kt = k0 + t;
            const int lt = pc.lt0 + t;
            const int y = min(lt * TILE, len - TILE);
            const int tok_lo = lt * TILE - y, tok_hi = min((lt + 1) * TILE, len) - y;
            // ---- this CTA's partial scores of the row
            // (one barrier per group: the group of tile kt + 1 may start waiting while the
            // scores of tile kt are still being computed)
            if (!warp_all(mbar_spin<false>(&bars->sready[g], (uint32_t)(kt >> 1) & 1u, FLAG_MMA_WAIT, c.abort_flag))) return;
            tc_fence_after();
            uint32_t sv[64];
            {
                uint32_t a[32], b[32];
                tmem_ld32(c.tmem + lane_base + TM_S, a);
                tmem_ld32(c.tmem + lane_base + TM_S + 32, b);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) { sv[j] = a[j]; sv[32 + j] = b[j]; }
            }
            tc_fence_before();
            mbar_arrive(&bars->sfree);
            // ---- to the peer: into the send buffer (free once the previous tile's copy has
            //      read it), same row layout as the peer's receive buffer; the sender thread
            //      ships it
            if (kt >= 1 && !warp_all(wait_count(reinterpret_cast<const int *>(c.smem + OFF_ABORT + 8), kt,
                                                  FLAG_PEER_WAIT, c.abort_flag)))
                return;
#pragma unroll
            for (int j = 0; j < 16; ++j)
                *reinterpret_cast<uint4 *>(send + recv_chunk(j, h) * 16) =
                    make_uint4(sv[4 * j], sv[4 * j + 1], sv[4 * j + 2], sv[4 * j + 3]);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->staged);
            // ---- the peer's partial scores; both CTAs add (own + peer) in the same order
            if (!warp_all(mbar_spin<true>(&bars->recv_full[g], (uint32_t)(kt >> 1) & 1u, FLAG_PEER_WAIT,
                                            c.abort_flag)))
                return;
            // arm this group's next tile (kt + 2): its phase of recv_full[g] is the next one
            if (h == 0) mbar_arrive_expect_tx(&bars->recv_full[g], RECV_BYTES);
            // raw scores (own + peer, unscaled) in place from here on
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const float4 v = reinterpret_cast<const float4 *>(recv)[recv_chunk(j, h)];
                sv[4 * j] = __float_as_uint(__uint_as_float(sv[4 * j]) + v.x);
                sv[4 * j + 1] = __float_as_uint(__uint_as_float(sv[4 * j + 1]) + v.y);
                sv[4 * j + 2] = __float_as_uint(__uint_as_float(sv[4 * j + 2]) + v.z);
                sv[4 * j + 3] = __float_as_uint(__uint_as_float(sv[4 * j + 3]) + v.w);
            }
            // the received values are in registers (the adds above consumed them, and
            // instructions issue in order): the peer may send the next tile at once
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster_relaxed(peer_rfree);
            // only a tile with rows outside the sequence needs the mask
            float mx = -INFINITY;
            if (tok_lo == 0 && tok_hi == TILE) {
#pragma unroll
                for (int i = 0; i < 64; ++i) mx = fmaxf(mx, __uint_as_float(sv[i]));
            } else {
#pragma unroll
                for (int i = 0; i < 64; ++i) {
                    const float x = (i >= tok_lo && i < tok_hi) ? __uint_as_float(sv[i]) : -INFINITY;
                    sv[i] = __float_as_uint(x);
                    mx = fmaxf(mx, x);
                }
            }
            mx *= p.scale_log2;     // the scale is positive: max of the scaled scores
            // ---- running max, handed on from the previous tile's group
            float m_prev = -INFINITY;
            if (kt > 0) {
                if (!warp_all(mbar_spin<false>(&bars->hand[(kt - 1) & 1], (uint32_t)((kt - 1) >> 1) & 1u, FLAG_FULL_WAIT,
                                        c.abort_flag)))
                    return;
                if (t > 0) m_prev = mref[((kt - 1) & 1) * HR + h];
            }
            const float m_new = (t == 0 || mx > m_prev + RESCALE_LOG2) ? mx : m_prev;
            mref[(kt & 1) * HR + h] = m_new;
            mbar_arrive(&bars->hand[kt & 1]);
            const bool rescale = t > 0 && m_new != m_prev;
            const float alpha = rescale ? fast_exp2(m_prev - m_new) : 1.f;
            // ---- weights, in two halves of 32 tokens; P goes into TMEM once the previous
            //      value product is done with it (and with O)
            l_g *= fast_exp2(m_last - m_new);      // 0 while this group has no tile yet
            m_last = m_new;
            float ls = 0.f;
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                uint32_t hw[16], lw[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const float a = fast_exp2(fmaf(__uint_as_float(sv[32 * hf + 2 * j]), p.scale_log2, -m_new));
                    const float b = fast_exp2(fmaf(__uint_as_float(sv[32 * hf + 2 * j + 1]), p.scale_log2, -m_new));
                    ls += a + b;
                    split_bf16x2(a, b, hw[j], lw[j]);
                }
                if (hf == 0) {
                    if (kt > 0 && !warp_all(mbar_spin<false>(&bars->odone[(kt - 1) & 1], (uint32_t)((kt - 1) >> 1) & 1u,
                                                      FLAG_MMA_WAIT, c.abort_flag)))
                        return;
                    tc_fence_after();
                }
                tmem_st16(c.tmem + lane_base + TM_P + 16 * hf, hw);
                tmem_st16(c.tmem + lane_base + TM_P + 32 + 16 * hf, lw);
            }
            l_g += ls;
            // rescale this row of O_r (tcgen05.ld/st are warp-collective: the whole warp
            // takes the branch when any row needs it, with factor 1 for the others)
            if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
                for (int cc = 0; cc < 8; ++cc) {
                    const uint32_t addr = c.tmem + lane_base + TM_O + 32 * cc;
                    uint32_t ov[32];
                    tmem_ld32(addr, ov);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j) ov[j] = __float_as_uint(__uint_as_float(ov[j]) * alpha);
                    tmem_st32(addr, ov);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bars->pready);
        }
        k = k0 + nt;
        // ---- end of the piece: merge the groups' row sums, normalise, write
        const int klast = k - 1;
        if (!warp_all(mbar_spin<false>(&bars->hand[klast & 1], (uint32_t)(klast >> 1) & 1u, FLAG_FULL_WAIT, c.abort_flag)))
            return;
        const float m_fin = mref[(klast & 1) * HR + h];
        lx[g * HR + h] = l_g * fast_exp2(m_last - m_fin);
        mbar_arrive(&bars->lx);
        if (!warp_all(mbar_spin<false>(&bars->lx, (uint32_t)pi & 1u, FLAG_FULL_WAIT, c.abort_flag))) return;
        const float l = lx[h] + lx[HR + h];
        const float lse_v = l > 0.f ? (m_fin + __log2f(l)) * 0.69314718055994531f : -INFINITY;
        const float inv = l > 0.f ? 1.f / l : 0.f;
        if (!warp_all(mbar_spin<false>(&bars->odone[klast & 1], (uint32_t)(klast >> 1) & 1u, FLAG_MMA_WAIT, c.abort_flag)))
            return;
        tc_fence_after();
        // The TMEM reads are warp-collective (every lane, padded head rows included);
        // only the stores are limited to the real heads.
        const bool real = h < p.H;
        float *dst;
        if (pc.whole)
            dst = p.out + ((size_t)pc.b * p.H + (real ? h : 0)) * 512;
        else
            dst = p.ws_o + (((size_t)c.worker * 2 + pc.slot) * HR + h) * 512;
        dst += 256 * c.r + 128 * g;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
            uint32_t ov[32];
            tmem_ld32(c.tmem + lane_base + TM_O + 128 * g + 32 * cc, ov);
            tmem_wait_ld();
            if (real) {
                float4 *d4 = reinterpret_cast<float4 *>(dst + 32 * cc);
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    d4[j] = make_float4(__uint_as_float(ov[4 * j]) * inv, __uint_as_float(ov[4 * j + 1]) * inv,
                                        __uint_as_float(ov[4 * j + 2]) * inv, __uint_as_float(ov[4 * j + 3]) * inv);
            }
        }
        if (real && c.r == 0 && g == 0) {
            if (pc.whole)
                p.lse[(size_t)pc.b * p.H + h] = lse_v;
            else
                p.ws_lse[((size_t)c.worker * 2 + pc.slot) * HR + h] = lse_v;
        }
        tc_fence_before();
        mbar_arrive(&bars->ofree);
    }
}

}  // namespace mla

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(mla::NTHREADS, 1)
mla_decode_kernel(const MlaParams p, const __grid_constant__ MlaMaps maps) {
    using namespace mla;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Bars *bars = reinterpret_cast<Bars *>(smem + OFF_BARS);
    uint32_t *tmem_ptr = reinterpret_cast<uint32_t *>(smem + OFF_TMEMPTR);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + OFF_ABORT);
    int *s_prefix = reinterpret_cast<int *>(smem + OFF_PREFIX);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (tid == 0) {
        for (int s = 0; s < NST; ++s) {
            mbar_init(&bars->full[s], 1);
            mbar_init(&bars->empty[s], 1);
        }
        mbar_init(&bars->qready, 2 * NGROUP);
        mbar_init(&bars->qrope_full, 1);
        mbar_init(&bars->qempty, 1);
        mbar_init(&bars->sfree, NGROUP);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars->sready[i], 1);
            mbar_init(&bars->hand[i], NGROUP);
            mbar_init(&bars->odone[i], 1);
        }
        mbar_init(&bars->recv_full[0], 1);
        mbar_init(&bars->recv_full[1], 1);
        mbar_init(&bars->peer_rfree, 4);
        mbar_init(&bars->staged, 4);
        mbar_init(&bars->pready, NGROUP);
        mbar_init(&bars->ofree, 2 * NGROUP);
        mbar_init(&bars->lx, 2 * NGROUP);
        *abort_flag = 0;
        *reinterpret_cast<int *>(smem + OFF_ABORT + 8) = 0;
        fence_mbar_init();
        mbar_arrive_expect_tx(&bars->recv_full[0], RECV_BYTES);   // the phases of tiles 0 and 1
        mbar_arrive_expect_tx(&bars->recv_full[1], RECV_BYTES);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_ptr), TM_COLS);
        tmem_relinquish();
    }
    if (warp == 2) build_tile_prefix(p.seq_lens, p.B, p.T_max, TILE, s_prefix, lane);
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&maps.lat);
        prefetch_tensormap(&maps.rope);
        prefetch_tensormap(&maps.qrope);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    cluster_sync_all();   // the peer's barriers are initialised before any remote arrival

    Ctx c;
    c.smem = smem;
    c.bars = bars;
    c.abort_flag = abort_flag;
    c.s_prefix = s_prefix;
    c.tmem = *tmem_ptr;
    c.r = cluster_ctarank();
    c.peer = c.r ^ 1u;
    c.worker = blockIdx.x >> 1;
    const long long total = s_prefix[p.B];
    const long long W = tiles_per_worker(total, p.workers, p.min_tiles);
    if (blockIdx.x == 0) {
        MetaView mv = meta_view(p.ws_meta);
        if (tid == 0) { mv.w_total[0] = W; mv.w_total[1] = total; }
        for (int i = tid; i <= p.B; i += NTHREADS) mv.prefix[i] = s_prefix[i];
    }
    pdl_launch_dependents();
    c.p0 = (long long)c.worker * W;
    c.p1 = (c.p0 + W < total) ? c.p0 + W : total;

    if (warp < 4) {
        regs_dec<REGS_WG0>();
        if (c.p0 < total) {
            if (warp == 0 && lane == 0) producer(p, maps, c);
            if (warp == 1 && lane == 0) mma_issuer(p, c);
            if (warp == 2 && lane == 0) sender(p, c);
        }
    } else {
        regs_inc<REGS_SOFTMAX>();
        if (c.p0 < total) softmax_warps(p, c, warp, lane);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(c.tmem, TM_COLS);
    }
    cluster_sync_all();   // no CTA leaves while its peer may still write into it
}

}  // namespace kvattn
