// mla_decode.cuh -- absorbed multi-head latent attention decode (latent 512 + RoPE 64)
// on sm_100a tensor cores (tcgen05, accumulators in tensor memory).
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
// all of one SM's tensor memory, and the 128 x 576 query alone is 144 KB of shared
// memory.  A 2-CTA cluster therefore splits the latent columns: CTA r holds columns
// [256r, 256r + 256) of every cached row (CTA 0 also the 64 RoPE columns), the matching
// query columns, and the output accumulator O_r = P * C[:, 256r..] (128 x 256 fp32,
// 256 TMEM columns).  Each CTA computes partial scores over its part of the 576-wide
// contraction and ships them to the other CTA with st.async (distributed shared memory,
// completion counted on the receiver's mbarrier); both CTAs then add the two partials
// in the same order and run the identical online softmax for all 128 heads, so P, the
// rescale factors and the row sums never have to cross the pair.  Every cached byte is
// loaded from HBM once and every MMA is a full-rate M = 128 tcgen05.mma.
//
// Per 64-token tile and CTA:
//   TMA (warp 0)       4 (CTA 0: 5) 128-byte-swizzled boxes [64 tokens x 64 columns]
//                      into a 2-stage ring; the query block once per piece.
//   MMA (warp 1)       S_r = Q_r C_r^T: 16 (20) kind::f16 bf16 MMAs 128x64x16 into TMEM;
//                      later O_r += P C_r: 4 kind::f16 fp16 MMAs 128x256x16 (C_r read
//                      MN-major from the same tile).  Completion via tcgen05.commit.
//   convert (warps 2-3) once the score MMAs have read the tile, the 256 latent columns
//                      are converted in place from bf16 to fp16 for the value product.
//   softmax (warps 4-11) 8 warps = 2 per TMEM lane quadrant, each thread one head row
//                      and 32 of the 64 token columns: send the partial scores, add the
//                      peer's, mask, take the running max (rescaling O only when the max
//                      grows by more than 2^8), write P = 2^(s - m) in fp16, keep the
//                      row sum.
// P and the value tile are fp16 (11 significant bits) so that the weights of a sharp
// softmax over a few tokens stay within the library's tolerance; this is why the latent
// values must lie in the fp16 range.  At the end of a piece every thread normalises its
// 128 output columns from TMEM and writes the final result or the worker's partial for
// the split combine.
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
constexpr int CHUNK_Q = HR * 128;        // one [128 heads x 64 cols] box: 16 KB
constexpr int STAGE = NCH * CHUNK_T;     // 40 KB
constexpr int PBUF = HR * 128;           // P: [128 heads x 64 tokens] fp16: 16 KB
constexpr int NTHREADS = 384;
constexpr int MAX_BATCH = 1024;
constexpr uint32_t TM_O = 0;             // TMEM columns [0, 256): O_r
constexpr uint32_t TM_S = 256;           // TMEM columns [256, 320): partial scores
constexpr uint32_t TM_Q = 320;           // TMEM columns [320, 480): Q_r (bf16 pairs)
constexpr uint32_t TM_COLS = 512;
constexpr float RESCALE_LOG2 = 8.f;      // rescale O only when the row max grows by > 2^8
constexpr uint32_t RECV_BYTES = HR * TILE * 4;   // the peer's partial scores of one tile

constexpr int OFF_ST = 0;
constexpr int OFF_P = OFF_ST + NST * STAGE;              // 163840
constexpr int OFF_RECV = OFF_P + PBUF;                   // the peer's partials: [128 heads][64] fp32
constexpr int OFF_SEND = OFF_RECV + (int)RECV_BYTES;     // this CTA's partials, same layout
constexpr int OFF_XCH = OFF_SEND + (int)RECV_BYTES;      // [2][128][2] fp32
constexpr int OFF_BARS = OFF_XCH + 2 * HR * 2 * 4;       // 215040
constexpr int OFF_TMEMPTR = OFF_BARS + 256;              // 215296
constexpr int OFF_ABORT = OFF_TMEMPTR + 16;
constexpr int OFF_PREFIX = OFF_ABORT + 16;               // 215328
constexpr int smem_bytes(int B) { return 1024 + OFF_PREFIX + (B + 1) * 4; }

struct Bars {
    uint64_t full[NST], empty[NST], qkdone[NST], cvt[NST];
    uint64_t qready;      // Q_r written into TMEM (softmax warps)
    uint64_t qempty;      // every score MMA of the piece has read Q_r
    uint64_t sready, sfree;
    uint64_t recv_full;   // the peer's partial scores landed (tx-counted)
    uint64_t recv_free;   // the peer has read the partial scores this CTA sent it
    uint64_t send_ready;  // this CTA's partial scores are in the send buffer
    uint64_t send_free;   // the bulk copy has finished reading the send buffer
    uint64_t oready[2];   // P written and O rescaled; PV may run
    uint64_t odone;       // PV done (also: P buffer free)
    uint64_t ofree;       // epilogue read O
    uint64_t pair[4];     // the two threads of a head row, per lane quadrant
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
        for (int lt = pc.lt0; lt < pc.lt1; ++lt, ++k) {
            const int s = k % NST;
            const uint32_t ph = (uint32_t)(k / NST) & 1u;
            if (!mbar_wait_sleep(&bars->empty[s], ph ^ 1u, FLAG_EMPTY_WAIT, c.abort_flag)) { ok = false; break; }
            mbar_arrive_expect_tx(&bars->full[s], nch * CHUNK_T);
            const int y = min(lt * TILE, len - TILE);
            uint8_t *st = c.smem + OFF_ST + s * STAGE;
            for (int ch = 0; ch < 4; ++ch)
                tma_load_3d(st + ch * CHUNK_T, &m.lat, &bars->full[s], 256 * (int)c.r + 64 * ch, y, pc.b, pol);
            if (c.r == 0) tma_load_3d(st + 4 * CHUNK_T, &m.rope, &bars->full[s], 0, y, pc.b, pol);
        }
    }
    if (!ok) {
        // Let every copy already issued land before the CTA can exit.
        for (int kk = (k > NST ? k - NST : 0); kk < k; ++kk)
            mbar_wait_sleep(&bars->full[kk % NST], (uint32_t)(kk / NST) & 1u, FLAG_FULL_WAIT, nullptr);
    }
}

// ------------------------------------------------------------------ MMA issuer (warp 1, lane 0)
__device__ __forceinline__ bool issue_scores(const Ctx &c, int kt, int nch, uint32_t st_base) {
    Bars *bars = c.bars;
    const int s = kt % NST;
    if (!mbar_wait_sleep(&bars->full[s], (uint32_t)(kt / NST) & 1u, FLAG_FULL_WAIT, c.abort_flag)) return false;
    if (kt > 0 && !mbar_wait_sleep(&bars->sfree, (uint32_t)(kt - 1) & 1u, FLAG_MMA_WAIT, c.abort_flag)) return false;
    tc_fence_after();
    constexpr uint32_t idesc = idesc_f16(128, TILE, 1, 1, 0);
    for (int ch = 0; ch < nch; ++ch)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            const uint64_t b = smem_desc_sw128(st_base + s * STAGE + ch * CHUNK_T + kk * 32, 16, 1024);
            umma_ts(c.tmem + TM_S, c.tmem + TM_Q + ch * 32 + kk * 8, b, idesc, (ch | kk) != 0);
        }
    umma_commit(&bars->sready);
    umma_commit(&bars->qkdone[s]);
    return true;
}

__device__ __forceinline__ void mma_issuer(const MlaParams &p, const Ctx &c) {
    Bars *bars = c.bars;
    const int nch = c.r == 0 ? 5 : 4;
    const uint32_t st_base = smem_u32(c.smem + OFF_ST);
    const uint32_t p_base = smem_u32(c.smem + OFF_P);
    constexpr uint32_t idesc_pv = idesc_f16(128, 256, 0, 0, 1);
    int k = 0, pi = 0;
    for (long long pos = c.p0; pos < c.p1; ++pi) {
        const Piece pc = piece_at(c.s_prefix, p.B, 1, pos, c.p1, c.p0);
        pos = pc.ustart + pc.lt1;
        const int nt = pc.lt1 - pc.lt0;
        if (!mbar_wait_sleep(&bars->qready, (uint32_t)pi & 1u, FLAG_FULL_WAIT, c.abort_flag)) return;
        tc_fence_after();
        if (!issue_scores(c, k, nch, st_base)) return;
        for (int t = 0; t < nt; ++t) {
            const int kt = k + t;
            if (t + 1 < nt) {
                if (!issue_scores(c, kt + 1, nch, st_base)) return;
            } else {
                umma_commit(&bars->qempty);      // every score MMA of this piece has read Q
            }
            const int s = kt % NST, pb = kt & 1;
            if (!mbar_wait_sleep(&bars->cvt[s], (uint32_t)(kt / NST) & 1u, FLAG_MMA_WAIT, c.abort_flag)) return;
            if (!mbar_wait_sleep(&bars->oready[pb], (uint32_t)(kt >> 1) & 1u, FLAG_MMA_WAIT, c.abort_flag)) return;
            if (t == 0 && pi > 0 &&
                !mbar_wait_sleep(&bars->ofree, (uint32_t)(pi - 1) & 1u, FLAG_MMA_WAIT, c.abort_flag))
                return;
            tc_fence_after();
            fence_proxy_async_smem();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint64_t a = smem_desc_sw128(p_base + kk * 32, 16, 1024);
                const uint64_t b = smem_desc_sw128(st_base + s * STAGE + kk * 2048, CHUNK_T, 1024);
                umma_ss(c.tmem + TM_O, a, b, idesc_pv, (t > 0 || kk > 0) ? 1u : 0u);
            }
            umma_commit(&bars->empty[s]);
            umma_commit(&bars->odone);
        }
        k += nt;
    }
}

// ------------------------------------------------------------------ converters (warps 2-3)
__device__ __forceinline__ void converter(const MlaParams &p, const Ctx &c, int ctid) {
    Bars *bars = c.bars;
    int k = 0;
    for (long long pos = c.p0; pos < c.p1;) {
        const Piece pc = piece_at(c.s_prefix, p.B, 1, pos, c.p1, c.p0);
        pos = pc.ustart + pc.lt1;
        for (int lt = pc.lt0; lt < pc.lt1; ++lt, ++k) {
            const int s = k % NST;
            if (!mbar_wait_sleep(&bars->qkdone[s], (uint32_t)(k / NST) & 1u, FLAG_MMA_WAIT, c.abort_flag)) return;
            uint4 *base = reinterpret_cast<uint4 *>(c.smem + OFF_ST + s * STAGE);
            // the four latent chunks (the value columns): 4 x 8 KB = 2048 16-byte units,
            // four independent loads in flight per thread
            for (int u0 = ctid; u0 < 4 * CHUNK_T / 16; u0 += 4 * 64) {
                uint4 v[4];
#pragma unroll
                for (int r = 0; r < 4; ++r) v[r] = base[u0 + 64 * r];
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    uint32_t w[4] = {v[r].x, v[r].y, v[r].z, v[r].w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float lo = __uint_as_float(w[i] << 16);
                        const float hi = __uint_as_float(w[i] & 0xffff0000u);
                        __half2 h2 = __floats2half2_rn(lo, hi);
                        w[i] = *reinterpret_cast<uint32_t *>(&h2);
                    }
                    base[u0 + 64 * r] = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
            fence_proxy_async_smem();
            mbar_arrive(&bars->cvt[s]);
        }
    }
}

// 16-byte chunk slot of chunk j (columns 4j..4j+3) in row h of a receive buffer.
__device__ __forceinline__ int recv_chunk(int j, int h) { return j ^ (h & 7); }

// ------------------------------------------------------------------ softmax (warps 4-11)
__device__ __forceinline__ void softmax_warps(const MlaParams &p, const Ctx &c, int warp, int lane) {
    Bars *bars = c.bars;
    const int q = warp & 3;
    const int half = (warp - 4) >> 2;
    const int h = 32 * q + lane;
    const bool armer = (warp == 4 && lane == 0);
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    const float *recv = reinterpret_cast<const float *>(c.smem + OFF_RECV);
    float *xch = reinterpret_cast<float *>(c.smem + OFF_XCH);
    // Send / receive buffers: row h holds 16 chunks of 16 bytes (64 fp32 scores), chunk
    // index XOR (row % 8), so a warp's 32 rows spread over all banks.  The whole send
    // buffer travels to the peer's receive buffer in one bulk copy per tile.
    uint8_t *send_row = c.smem + OFF_SEND + h * TILE * 4;
    const uint32_t peer_recv_buf = map_to_rank(smem_u32(c.smem + OFF_RECV), c.peer);
    const uint32_t send_buf = smem_u32(c.smem + OFF_SEND);
    const uint32_t peer_recv_full = map_to_rank(smem_u32(&bars->recv_full), c.peer);
    (void)peer_recv_full;
    const uint32_t peer_recv_free = map_to_rank(smem_u32(&bars->recv_free), c.peer);
    uint8_t *prow = c.smem + OFF_P + h * 128;
    uint32_t pair_uses = 0;

    int k = 0, pi = 0;
    for (long long pos = c.p0; pos < c.p1; ++pi) {
        const Piece pc = piece_at(c.s_prefix, p.B, 1, pos, c.p1, c.p0);
        pos = pc.ustart + pc.lt1;
        const int len = clamp_len(__ldg(p.seq_lens + pc.b), p.T_max);
        const int nt = pc.lt1 - pc.lt0;
        // ---- Q_r of this sequence into TMEM (lane h = head h; bf16 pairs per column):
        //      CTA 0 holds latent columns 0..255 and the 64 RoPE columns (160 words),
        //      CTA 1 latent columns 256..511 (128 words).  Half 0 writes words [0, 96),
        //      half 1 the rest, 32 words per tcgen05.st.
        if (pi > 0 && !warp_all(mbar_wait_sleep(&bars->qempty, (uint32_t)(pi - 1) & 1u, FLAG_MMA_WAIT, c.abort_flag)))
            return;
        {
            const int nwords = c.r == 0 ? 160 : 128;
            const int w0 = half == 0 ? 0 : 96, w1 = half == 0 ? 96 : nwords;
            const bool real = h < p.H;
            const uint32_t *ql = reinterpret_cast<const uint32_t *>(p.q_latent) +
                                 ((size_t)pc.b * p.H + (real ? h : 0)) * 256 + 128 * c.r;
            const uint32_t *qr = reinterpret_cast<const uint32_t *>(p.q_rope) +
                                 ((size_t)pc.b * p.H + (real ? h : 0)) * 32;
            tc_fence_after();
            for (int w = w0; w < w1; w += 32) {
                uint32_t v[32];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int word = w + 4 * j;
                    uint4 x = make_uint4(0, 0, 0, 0);
                    if (real) x = word < 128 ? __ldg(reinterpret_cast<const uint4 *>(ql + word))
                                             : __ldg(reinterpret_cast<const uint4 *>(qr + (word - 128)));
                    v[4 * j] = x.x; v[4 * j + 1] = x.y; v[4 * j + 2] = x.z; v[4 * j + 3] = x.w;
                }
                tmem_st32(c.tmem + lane_base + TM_Q + w, v);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bars->qready);
        }
        float m_ref = -INFINITY;
        float l_part = 0.f;
        for (int t = 0; t < nt; ++t, ++k) {
            const int lt = pc.lt0 + t;
            const int y = min(lt * TILE, len - TILE);
            const int tok_lo = lt * TILE - y, tok_hi = min((lt + 1) * TILE, len) - y;
            // ---- this CTA's partial scores
            if (!warp_all(mbar_wait_sleep(&bars->sready, (uint32_t)k & 1u, FLAG_MMA_WAIT, c.abort_flag))) return;
            tc_fence_after();
            uint32_t sv[32];
            tmem_ld32(c.tmem + lane_base + TM_S + 32 * half, sv);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&bars->sfree);
            // ---- stage them in the send buffer (free once the previous bulk copy has read it;
            //      the issuing thread checks that here, off the previous tile's critical path)
            if (armer && k > 0) {
                bulk_wait_read_all();
                mbar_arrive(&bars->send_free);
            }
            if (k > 0 && !warp_all(mbar_wait_sleep(&bars->send_free, (uint32_t)(k - 1) & 1u, FLAG_PEER_WAIT,
                                                   c.abort_flag)))
                return;
#pragma unroll
            for (int j = 0; j < 8; ++j)
                *reinterpret_cast<uint4 *>(send_row + recv_chunk(8 * half + j, h) * 16) =
                    make_uint4(sv[4 * j], sv[4 * j + 1], sv[4 * j + 2], sv[4 * j + 3]);
            fence_proxy_async_smem();
            mbar_arrive(&bars->send_ready);
            if (armer) {
                // one bulk copy of all 128 rows into the peer, once the peer has read the last one
                bool ok = mbar_wait_sleep(&bars->send_ready, (uint32_t)k & 1u, FLAG_FULL_WAIT, c.abort_flag);
                if (ok && k > 0)
                    ok = mbar_wait_cluster(&bars->recv_free, (uint32_t)(k - 1) & 1u, FLAG_PEER_WAIT, c.abort_flag);
                if (ok) {
                    bulk_copy_to_peer(peer_recv_buf, send_buf, RECV_BYTES, peer_recv_full);
                    bulk_commit_group();
                }
            }
            // ---- the peer's partial scores of this tile (one arrival + RECV_BYTES per phase)
            if (armer) mbar_arrive_expect_tx(&bars->recv_full, RECV_BYTES);
            if (!warp_all(mbar_wait_cluster(&bars->recv_full, (uint32_t)k & 1u, FLAG_PEER_WAIT, c.abort_flag)))
                return;
            float s[32];
            const float4 *src = reinterpret_cast<const float4 *>(recv + h * TILE);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float4 v = src[recv_chunk(8 * half + j, h)];
                // both CTAs add (own + peer); fp32 addition commutes, so the sums match
                s[4 * j + 0] = __uint_as_float(sv[4 * j + 0]) + v.x;
                s[4 * j + 1] = __uint_as_float(sv[4 * j + 1]) + v.y;
                s[4 * j + 2] = __uint_as_float(sv[4 * j + 2]) + v.z;
                s[4 * j + 3] = __uint_as_float(sv[4 * j + 3]) + v.w;
            }
            float mx = -INFINITY;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const int row = 32 * half + j;
                s[j] = (row >= tok_lo && row < tok_hi) ? s[j] * p.scale_log2 : -INFINITY;
                mx = fmaxf(mx, s[j]);
            }
            // the received values are consumed (mx depends on all of them): the peer may
            // overwrite its slice of this buffer now
            mbar_arrive_cluster_relaxed(peer_recv_free);
            // row max over both halves of the tile (the other half lives in warp q +/- 4)
            float *slot = xch + (pair_uses & 1u) * (HR * 2);
            slot[h * 2 + half] = mx;
            mbar_arrive(&bars->pair[q]);
            if (!warp_all(mbar_wait_sleep(&bars->pair[q], pair_uses & 1u, FLAG_FULL_WAIT, c.abort_flag))) return;
            ++pair_uses;
            mx = fmaxf(mx, slot[h * 2 + (half ^ 1)]);
            float alpha = 1.f;
            bool rescale = false;
            if (t == 0) {
                m_ref = mx;
            } else if (mx > m_ref + RESCALE_LOG2) {
                alpha = fast_exp2(m_ref - mx);
                m_ref = mx;
                rescale = true;
            }
            float ls = 0.f;
            uint32_t ph[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const float a = fast_exp2(s[2 * j] - m_ref);
                const float b = fast_exp2(s[2 * j + 1] - m_ref);
                __half2 h2 = __floats2half2_rn(a, b);
                ph[j] = *reinterpret_cast<uint32_t *>(&h2);
                ls += a + b;
            }
            l_part = (t == 0) ? ls : (rescale ? l_part * alpha + ls : l_part + ls);
            // ---- the previous value product has finished with P and with O
            const bool need = rescale;
            if (k > 0 && !warp_all(mbar_wait_sleep(&bars->odone, (uint32_t)(k - 1) & 1u, FLAG_MMA_WAIT, c.abort_flag)))
                return;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int chunk = 4 * half + j;                  // tokens 8*chunk .. +7
                *reinterpret_cast<uint4 *>(prow + ((chunk ^ (h & 7)) << 4)) =
                    make_uint4(ph[4 * j], ph[4 * j + 1], ph[4 * j + 2], ph[4 * j + 3]);
            }
            fence_proxy_async_smem();
            // ---- rescale this row of O_r (tcgen05.ld/st are warp-collective: the whole warp
            //      takes the branch when any row needs it, with factor 1 for the others)
            if (__any_sync(0xffffffffu, need)) {
                tc_fence_after();
                const float f = need ? alpha : 1.f;
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    const uint32_t addr = c.tmem + lane_base + TM_O + 128 * half + 32 * cc;
                    uint32_t ov[32];
                    tmem_ld32(addr, ov);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j) ov[j] = __float_as_uint(__uint_as_float(ov[j]) * f);
                    tmem_st32(addr, ov);
                }
                tmem_wait_st();
            }
            tc_fence_before();
            mbar_arrive(&bars->oready[k & 1]);
        }
        // ---- end of the piece: normaliser, lse, output
        if (!warp_all(mbar_wait_sleep(&bars->odone, (uint32_t)(k - 1) & 1u, FLAG_MMA_WAIT, c.abort_flag))) return;
        tc_fence_after();
        float *slot = xch + (pair_uses & 1u) * (HR * 2);
        slot[h * 2 + half] = l_part;
        mbar_arrive(&bars->pair[q]);
        if (!warp_all(mbar_wait_sleep(&bars->pair[q], pair_uses & 1u, FLAG_FULL_WAIT, c.abort_flag))) return;
        ++pair_uses;
        const float l = l_part + slot[h * 2 + (half ^ 1)];
        const float lse_v = l > 0.f ? (m_ref + __log2f(l)) * 0.69314718055994531f : -INFINITY;
        const float inv = l > 0.f ? 1.f / l : 0.f;
        // The TMEM reads are warp-collective (every lane, padded head rows included);
        // only the stores are limited to the real heads.
        const bool real = h < p.H;
        float *dst;
        if (pc.whole)
            dst = p.out + ((size_t)pc.b * p.H + (real ? h : 0)) * 512;
        else
            dst = p.ws_o + (((size_t)c.worker * 2 + pc.slot) * HR + h) * 512;
        dst += 256 * c.r + 128 * half;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
            uint32_t ov[32];
            tmem_ld32(c.tmem + lane_base + TM_O + 128 * half + 32 * cc, ov);
            tmem_wait_ld();
            if (real) {
                float4 *d4 = reinterpret_cast<float4 *>(dst + 32 * cc);
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    d4[j] = make_float4(__uint_as_float(ov[4 * j]) * inv, __uint_as_float(ov[4 * j + 1]) * inv,
                                        __uint_as_float(ov[4 * j + 2]) * inv, __uint_as_float(ov[4 * j + 3]) * inv);
            }
        }
        if (real && c.r == 0 && half == 0) {
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
            mbar_init(&bars->qkdone[s], 1);
            mbar_init(&bars->cvt[s], 64);
        }
        mbar_init(&bars->qready, 256);
        mbar_init(&bars->qempty, 1);
        mbar_init(&bars->sready, 1);
        mbar_init(&bars->sfree, 256);
        mbar_init(&bars->recv_full, 1);
        mbar_init(&bars->recv_free, 256);
        mbar_init(&bars->send_ready, 256);
        mbar_init(&bars->send_free, 1);
        mbar_init(&bars->oready[0], 256);
        mbar_init(&bars->oready[1], 256);
        mbar_init(&bars->odone, 1);
        mbar_init(&bars->ofree, 256);
        for (int i = 0; i < 4; ++i) mbar_init(&bars->pair[i], 64);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_ptr), TM_COLS);
        tmem_relinquish();
    }
    if (warp == 2) build_tile_prefix(p.seq_lens, p.B, p.T_max, TILE, s_prefix, lane);
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&maps.lat);
        prefetch_tensormap(&maps.rope);
        prefetch_tensormap(&maps.qlat);
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

    if (c.p0 < total) {
        if (warp == 0) {
            if (lane == 0) producer(p, maps, c);
        } else if (warp == 1) {
            if (lane == 0) mma_issuer(p, c);
        } else if (warp < 4) {
            converter(p, c, tid - 64);
        } else {
            softmax_warps(p, c, warp, lane);
        }
    }

    if (warp == 4 && lane == 0) bulk_wait_read_all();   // the last send has left this CTA
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(c.tmem, TM_COLS);
    }
    cluster_sync_all();   // no CTA leaves while its peer may still write into it
}

}  // namespace kvattn
