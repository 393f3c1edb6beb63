// mla_decode.cuh -- absorbed multi-head latent attention decode (latent 512 + RoPE 64)
// on sm_100a tensor cores, each tile computed by a CTA pair with cta_group::2 MMAs.
//
// What it computes ("Attention variants: MQA, GQA, and MLA", section "MLA: cache a
// latent, not the keys and values"): with the key up-projection folded into the query,
// head h of sequence b scores every cached token t as
//     s[h,t] = scale * (q_lat[h] . c_t + q_rope[h] . r_t)
// and returns out[h] = sum_t softmax(s[h])_t * c_t, a 512-wide latent (the value
// up-projection is applied by the caller) -- one shared 576-wide key row per token,
// whose first 512 elements are also the value.
//
// Why a CTA pair.  The fp32 accumulator of 128 heads x 512 latent columns is 256 KB, all
// of one SM's tensor memory.  So the 128 heads are split over the two CTAs of a cluster:
// CTA r owns heads [64r, 64r + 64), and every product is a pair MMA (cta_group::2, M =
// 128: each CTA supplies its 64 rows of A, and half of the B columns, which the pair
// shares through the tensor cores).  Each CTA's tensor memory then holds its 64 heads x
// N result in the "2x2" layout: lane m (m < 64) holds columns [0, N/2) of row m and lane
// 64 + m columns [N/2, N).  Nothing is exchanged between the CTAs by threads: no score,
// weight or row sum crosses the pair, and each head's softmax runs once.
//
// Per 128-token tile t0 .. t0+127 (tokens of half h: t0 + 64h ..):
//   score product S = Q K^T (M = 128 heads, N = 128 tokens, K = 576): A = this CTA's 64
//     query rows (shared memory, loaded once per sequence: 8 latent chunks + 1 RoPE
//     chunk of 64 columns), B = the 576-wide key rows of tile half r (CTA r loads the
//     half its B columns are).  9 chunks x 4 MMAs of K = 16.  In tensor memory, lane m
//     holds head 64r + m's scores of half 0's tokens, lane 64 + m those of half 1's.
//   value product O += P C (M = 128 heads, N = 256 latent columns per MMA, two MMAs for
//     the 512 columns, K = 128 tokens): A = this CTA's weights P (shared memory, K-major),
//     B = the latent columns [256j + 128r, 256j + 128r + 128) of all 128 tokens (MN-major,
//     loaded by CTA r for both halves: the B columns it supplies).  Lane m holds head
//     64r + m's output columns 256j + [0, 128), lane 64 + m columns 256j + [128, 256).
//   The weights enter as a bf16 high part (the top 16 bits of each fp32 weight) plus a
//     bf16 remainder, two MMAs per K step, so they keep ~16 significant bits (a plain
//     bf16 weight, 8 bits, misses the 2e-3 relative tolerance on sharp softmaxes).
// Latent columns are thus read twice per pair (once as keys by the half's owner, once as
// values by each CTA for its columns), the second time from L2.
//
// Warp roles (256 threads per CTA):
//   warp 0, one thread   TMA producer (both CTAs): the query block once per sequence, a
//                        6-slot ring of key chunks (8 KB) and a 4-slot ring of value
//                        chunk pairs (16 KB); completions signal rank 0's barriers.
//   warp 1, one thread   MMA issuer (rank 0 only): S of tile k + 1 before O += P C of
//                        tile k, so the softmax of tile k overlaps the next score product.
//   warps 4-7            softmax, one thread per tensor-memory lane (head 64r + m, tile
//                        half h): masks, tile maximum (the two halves of a head meet in
//                        shared memory), lazy running max (moves only when a tile's
//                        maximum exceeds it by more than 2^8; then this CTA's rows of O
//                        are rescaled in tensor memory), weights into shared memory,
//                        row sums; at the end of a piece the normalised result.
// Every wait is bounded; every wait ahead of a warp-collective instruction is made
// warp-uniform.  No TMA load uses multicast.
#pragma once
#include "common.cuh"
#include "schedule.cuh"
#include "tc05.cuh"

namespace kvattn {
namespace mla {

constexpr int TILE = 128;                // tokens per tile of a CTA pair (N of the score product)
constexpr int SUB = 64;                  // tokens of a tile half (one CTA's B columns of the score product)
constexpr int HR = 128;                  // head rows of the pair (M)
constexpr int HC = 64;                   // head rows of one CTA
constexpr int CHUNK = SUB * 128;         // one TMA box [64 rows x 64 bf16 columns], 128-byte swizzled: 8 KB
constexpr int NQC = 9;                   // query chunks: 8 latent + 1 RoPE
constexpr int NSS = 6;                   // key ring slots (one chunk each)
constexpr int NPV = 4;                   // value ring slots (two chunks each: 128 latent columns)
constexpr int NTHREADS = 256;
constexpr int MAX_BATCH = 1024;
constexpr float RESCALE_LOG2 = 8.f;      // rescale O only when the row max grows by > 2^8
constexpr uint32_t TM_O = 0;             // tensor memory columns [0, 256): O (two blocks of 128)
constexpr uint32_t TM_S = 256;           // [256, 384): the scores of two tiles (64 columns each)
constexpr uint32_t TM_COLS = 512;

constexpr int OFF_Q = 0;                               // query chunks [9][64 heads x 128 B]
constexpr int OFF_P = OFF_Q + NQC * CHUNK;             // weights: high [2 halves], remainder [2 halves]
constexpr int OFF_SR = OFF_P + 4 * CHUNK;              // key ring
constexpr int OFF_PV = OFF_SR + NSS * CHUNK;           // value ring
constexpr int OFF_MX = OFF_PV + NPV * 2 * CHUNK;       // [2 tiles][2 halves][64] tile maxima
constexpr int OFF_LX = OFF_MX + 2 * 2 * HC * 4;        // [2 halves][64] row sums
constexpr int OFF_BARS = OFF_LX + 2 * HC * 4;
constexpr int OFF_TMEMPTR = OFF_BARS + 512;
constexpr int OFF_ABORT = OFF_TMEMPTR + 16;
constexpr int OFF_PREFIX = OFF_ABORT + 16;
constexpr int smem_bytes(int B) { return 1024 + OFF_PREFIX + (B + 1) * 4; }
static_assert(smem_bytes(MAX_BATCH) <= 232448, "shared memory of the MLA kernel exceeds 227 KB");

struct Bars {
    uint64_t sfull[NSS], sempty[NSS];   // key ring (full: rank 0, both CTAs' bytes; empty: both CTAs)
    uint64_t vfull[NPV], vempty[NPV];   // value ring
    uint64_t qfull;                     // query block of both CTAs landed (rank 0)
    uint64_t qempty;                    // every score product of the piece has read Q (both CTAs)
    uint64_t sready[2];                 // scores of a tile (parity) in tensor memory (both CTAs)
    uint64_t sfree[2];                  // both CTAs have read them (rank 0: 4 warps x 2 CTAs)
    uint64_t pready;                    // weights written, O rescaled, in both CTAs (rank 0)
    uint64_t odone;                     // value product of a tile finished (both CTAs)
    uint64_t ofree;                     // both CTAs' epilogues have read O (rank 0)
    uint64_t mxbar[2];                  // the four softmax warps' tile maxima written (tile parity)
    uint64_t lxbar;                     // the four softmax warps' row sums written (end of a piece)
};
static_assert(sizeof(Bars) <= 512, "barrier block overflows its slot");

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
    int workers;       // CTA pairs
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
    uint32_t r;        // rank in the pair
    int worker;
    long long p0, p1;
};

// Where half h of tile lt of a sequence of length len is loaded from, and which of its 64
// rows are tokens of that half.  A half is a 64-token sub-tile (pages hold whole
// sub-tiles); the last sub-tile of the sequence is loaded shifted back so that it ends
// at the last token (tile_source), its first rows then repeat tokens of the sub-tile
// before it (or lie before its page and are zero-filled); a half past the sequence's end
// loads the last sub-tile again.  Rows below `lo` are masked.
struct HalfSrc {
    int y, page, lo;
};
__device__ __forceinline__ HalfSrc half_source(const MlaParams &p, int b, int len, int lt, int h) {
    const int n_sub = (len + SUB - 1) / SUB;
    int st = 2 * lt + h;
    HalfSrc s;
    if (st >= n_sub) {
        st = n_sub - 1;
        s.lo = SUB;
    } else {
        s.lo = SUB * st + SUB - len > 0 ? SUB * st + SUB - len : 0;
    }
    const TileSrc t = tile_source(p.block_table, p.max_pages, p.page_size, b, st, SUB, len);
    s.y = t.y;
    s.page = t.page;
    return s;
}

// ------------------------------------------------------------------ producer (warp 0, lane 0)
// Both CTAs load, in the order the MMAs consume: the query block of a sequence, then the
// key chunks of tile k0, and for every tile k of the piece the key chunks of tile k + 1
// followed by the value chunks of tile k.  Completions go to rank 0's barriers, which
// rank 0 arms with the bytes of both CTAs.
__device__ __forceinline__ void producer(const MlaParams &p, const MlaMaps &m, const Ctx &c) {
    Bars *bars = c.bars;
    const uint64_t pol_keep = l2_policy_evict_normal();   // keys: the latent columns are read again
    const uint64_t pol_last = l2_policy_evict_first();    // values: last read
    const bool lead = c.r == 0;
    const uint32_t qfull0 = map_to_rank(smem_u32(&bars->qfull), 0);
    int sidx = 0, vidx = 0, pi = 0;
    bool ok = true;
    for (long long pos = c.p0; pos < c.p1 && ok; ++pi) {
        const Piece pc = piece_at(c.s_prefix, p.B, 1, pos, c.p1, c.p0);
        pos = pc.ustart + pc.lt1;
        const int len = clamp_len(__ldg(p.seq_lens + pc.b), p.T_max);
        const int nt = pc.lt1 - pc.lt0;
        // this CTA's 64 query rows: 8 latent chunks and the RoPE chunk
        if (pi > 0 && !mbar_wait(&bars->qempty, (uint32_t)(pi - 1) & 1u, FLAG_EMPTY_WAIT, c.abort_flag)) {
            ok = false;
            break;
        }
        if (lead) mbar_arrive_expect_tx(&bars->qfull, 2 * NQC * CHUNK);
        for (int ch = 0; ch < 8; ++ch)
            tma_load_3d_pair(c.smem + OFF_Q + ch * CHUNK, &m.qlat, qfull0, 64 * ch, HC * (int)c.r, pc.b, pol_keep);
        tma_load_3d_pair(c.smem + OFF_Q + 8 * CHUNK, &m.qrope, qfull0, 0, HC * (int)c.r, pc.b, pol_keep);

        auto load_keys = [&](int lt) -> bool {
            const HalfSrc hs = half_source(p, pc.b, len, lt, (int)c.r);
            for (int ch = 0; ch < NQC; ++ch, ++sidx) {
                const int s = sidx % NSS;
                if (!mbar_wait(&bars->sempty[s], ((uint32_t)(sidx / NSS) & 1u) ^ 1u, FLAG_EMPTY_WAIT, c.abort_flag))
                    return false;
                if (lead) mbar_arrive_expect_tx(&bars->sfull[s], 2 * CHUNK);
                const uint32_t bar = map_to_rank(smem_u32(&bars->sfull[s]), 0);
                if (ch < 8)
                    tma_load_3d_pair(c.smem + OFF_SR + s * CHUNK, &m.lat, bar, 64 * ch, hs.y, hs.page, pol_keep);
                else
                    tma_load_3d_pair(c.smem + OFF_SR + s * CHUNK, &m.rope, bar, 0, hs.y, hs.page, pol_keep);
            }
            return true;
        };
        auto load_values = [&](int lt) -> bool {
            for (int j = 0; j < 2; ++j)
                for (int h = 0; h < 2; ++h, ++vidx) {
                    const HalfSrc hs = half_source(p, pc.b, len, lt, h);
                    const int s = vidx % NPV;
                    if (!mbar_wait(&bars->vempty[s], ((uint32_t)(vidx / NPV) & 1u) ^ 1u, FLAG_EMPTY_WAIT,
                                   c.abort_flag))
                        return false;
                    if (lead) mbar_arrive_expect_tx(&bars->vfull[s], 4 * CHUNK);
                    const uint32_t bar = map_to_rank(smem_u32(&bars->vfull[s]), 0);
                    uint8_t *dst = c.smem + OFF_PV + s * 2 * CHUNK;
                    const int x = 256 * j + 128 * (int)c.r;
                    tma_load_3d_pair(dst, &m.lat, bar, x, hs.y, hs.page, pol_last);
                    tma_load_3d_pair(dst + CHUNK, &m.lat, bar, x + 64, hs.y, hs.page, pol_last);
                }
            return true;
        };
        if (!load_keys(pc.lt0)) { ok = false; break; }
        for (int t = 0; t < nt; ++t) {
            if (t + 1 < nt && !load_keys(pc.lt0 + t + 1)) { ok = false; break; }
            if (!load_values(pc.lt0 + t)) { ok = false; break; }
        }
    }
    if (!ok && lead) {
        // Let the copies already issued land before the CTAs can exit.
        for (int i = (sidx > NSS ? sidx - NSS : 0); i < sidx; ++i)
            mbar_wait_sleep(&bars->sfull[i % NSS], (uint32_t)(i / NSS) & 1u, FLAG_FULL_WAIT, nullptr);
        for (int i = (vidx > NPV ? vidx - NPV : 0); i < vidx; ++i)
            mbar_wait_sleep(&bars->vfull[i % NPV], (uint32_t)(i / NPV) & 1u, FLAG_FULL_WAIT, nullptr);
    }
}

// ------------------------------------------------------------------ MMA issuer (rank 0, warp 1, lane 0)
__device__ __forceinline__ bool wait_remote(uint64_t *bar, uint32_t parity, const Ctx &c) {
    return mbar_spin<true>(bar, parity, FLAG_PEER_WAIT, c.abort_flag);
}

__device__ __forceinline__ void mma_issuer(const MlaParams &p, const Ctx &c) {
    Bars *bars = c.bars;
    constexpr uint32_t id_s = idesc_f16(128, TILE, 1, 1, 0);   // K-major A and B
    constexpr uint32_t id_v = idesc_f16(128, 256, 1, 1, 1);    // B (the latents) MN-major
    const uint32_t q_base = smem_u32(c.smem + OFF_Q);
    const uint32_t p_base = smem_u32(c.smem + OFF_P);
    int sidx = 0, vidx = 0;

    // S of tile kt into score buffer kt & 1: 9 chunks x 4 K-steps of 16.
    auto issue_scores = [&](int kt) -> bool {
        const int sb = kt & 1;
        if (kt >= 2 && !wait_remote(&bars->sfree[sb], (uint32_t)((kt >> 1) - 1) & 1u, c)) return false;
        for (int ch = 0; ch < NQC; ++ch, ++sidx) {
            const int s = sidx % NSS;
            if (!mbar_wait(&bars->sfull[s], (uint32_t)(sidx / NSS) & 1u, FLAG_FULL_WAIT, c.abort_flag)) return false;
            tc_fence_after();
            const uint32_t kb = smem_u32(c.smem + OFF_SR + s * CHUNK);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                umma_pair_ss(c.tmem + TM_S + 64 * sb, smem_desc_sw128(q_base + ch * CHUNK + kk * 32, 16, 1024),
                             smem_desc_sw128(kb + kk * 32, 16, 1024), id_s, (ch | kk) != 0);
            umma_pair_commit_both(&bars->sempty[s]);
        }
        umma_pair_commit_both(&bars->sready[sb]);
        return true;
    };
    // O += P_hi C + P_lo C for tile kt: latent blocks j, token halves h, K-steps of 16.
    auto issue_values = [&](int kt, bool first) -> bool {
        if (!wait_remote(&bars->pready, (uint32_t)kt & 1u, c)) return false;
        for (int j = 0; j < 2; ++j)
            for (int h = 0; h < 2; ++h, ++vidx) {
                const int s = vidx % NPV;
                if (!mbar_wait(&bars->vfull[s], (uint32_t)(vidx / NPV) & 1u, FLAG_FULL_WAIT, c.abort_flag))
                    return false;
                tc_fence_after();
                const uint32_t vb = smem_u32(c.smem + OFF_PV + s * 2 * CHUNK);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t bd = smem_desc_sw128(vb + kk * 2048, CHUNK, 1024);
                    const uint32_t pa = p_base + h * CHUNK + kk * 32;
                    umma_pair_ss(c.tmem + TM_O + 128 * j, smem_desc_sw128(pa, 16, 1024), bd, id_v,
                                 (!first || h > 0 || kk > 0) ? 1u : 0u);
                    umma_pair_ss(c.tmem + TM_O + 128 * j, smem_desc_sw128(pa + 2 * CHUNK, 16, 1024), bd, id_v, 1u);
                }
                umma_pair_commit_both(&bars->vempty[s]);
            }
        umma_pair_commit_both(&bars->odone);
        return true;
    };

    int k = 0, pi = 0;
    for (long long pos = c.p0; pos < c.p1; ++pi) {
        const Piece pc = piece_at(c.s_prefix, p.B, 1, pos, c.p1, c.p0);
        pos = pc.ustart + pc.lt1;
        const int nt = pc.lt1 - pc.lt0;
        if (!mbar_wait(&bars->qfull, (uint32_t)pi & 1u, FLAG_FULL_WAIT, c.abort_flag)) return;
        if (!issue_scores(k)) return;
        if (nt == 1) umma_pair_commit_both(&bars->qempty);
        for (int t = 0; t < nt; ++t) {
            const int kt = k + t;
            if (t + 1 < nt) {
                if (!issue_scores(kt + 1)) return;
                if (t + 2 == nt) umma_pair_commit_both(&bars->qempty);   // the piece's last score product
            }
            // the previous piece's epilogue must have read O before the first product overwrites it
            if (t == 0 && pi > 0 && !wait_remote(&bars->ofree, (uint32_t)(pi - 1) & 1u, c)) return;
            if (!issue_values(kt, t == 0)) return;
        }
        k += nt;
    }
}

// ------------------------------------------------------------------ softmax (warps 4-7)
__device__ __forceinline__ void softmax_warps(const MlaParams &p, const Ctx &c, int warp, int lane) {
    Bars *bars = c.bars;
    const int q = warp & 3;                     // tensor-memory lane quadrant
    const int L = 32 * q + lane;                // tensor-memory lane
    const int hh = L & (HC - 1);                // head row of this CTA
    const int half = L >> 6;                    // tile half whose scores the lane holds
    const int head = HC * (int)c.r + hh;
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    float *mx_buf = reinterpret_cast<float *>(c.smem + OFF_MX);
    float *lx_buf = reinterpret_cast<float *>(c.smem + OFF_LX);
    const uint32_t sfree0 = map_to_rank(smem_u32(&bars->sfree[0]), 0);
    const uint32_t sfree1 = map_to_rank(smem_u32(&bars->sfree[1]), 0);
    const uint32_t pready0 = map_to_rank(smem_u32(&bars->pready), 0);
    const uint32_t ofree0 = map_to_rank(smem_u32(&bars->ofree), 0);
    uint8_t *row_hi = c.smem + OFF_P + half * CHUNK + hh * 128;   // this row of the weights (K-major, swizzled)
    uint8_t *row_lo = row_hi + 2 * CHUNK;
    const float sl2 = p.scale_log2;

    int k = 0, pi = 0;
    for (long long pos = c.p0; pos < c.p1; ++pi) {
        const Piece pc = piece_at(c.s_prefix, p.B, 1, pos, c.p1, c.p0);
        pos = pc.ustart + pc.lt1;
        const int len = clamp_len(__ldg(p.seq_lens + pc.b), p.T_max);
        const int nt = pc.lt1 - pc.lt0;
        float m_ref = -INFINITY;      // running max (log2 units), shared by the two halves of the head
        float l = 0.f;                // row sum of this half's weights, relative to m_ref
        for (int t = 0; t < nt; ++t) {
            const int kt = k + t;
            const int sb = kt & 1;
            const int lo = half_source(p, pc.b, len, pc.lt0 + t, half).lo;
            // ---- scores of this lane (64 tokens of its half)
            if (!warp_all(mbar_spin<false>(&bars->sready[sb], (uint32_t)(kt >> 1) & 1u, FLAG_MMA_WAIT, c.abort_flag)))
                return;
            tc_fence_after();
            float sv[64];
            {
                uint32_t a[32], b[32];
                tmem_ld32(c.tmem + lane_base + TM_S + 64 * sb, a);
                tmem_ld32(c.tmem + lane_base + TM_S + 64 * sb + 32, b);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    sv[j] = __uint_as_float(a[j]);
                    sv[32 + j] = __uint_as_float(b[j]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(sb ? sfree1 : sfree0);
            // ---- scaled (log2 units), masked, tile maximum of this half
            float mx = -INFINITY;
            if (lo == 0) {
#pragma unroll
                for (int i = 0; i < 64; ++i) {
                    sv[i] *= sl2;
                    mx = fmaxf(mx, sv[i]);
                }
            } else {
#pragma unroll
                for (int i = 0; i < 64; ++i) {
                    sv[i] = i >= lo ? sv[i] * sl2 : -INFINITY;
                    mx = fmaxf(mx, sv[i]);
                }
            }
            // ---- the head's tile maximum over both halves, then the running max
            mx_buf[(sb * 2 + half) * HC + hh] = mx;
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->mxbar[sb]);
            if (!warp_all(mbar_spin<false>(&bars->mxbar[sb], (uint32_t)(kt >> 1) & 1u, FLAG_FULL_WAIT, c.abort_flag)))
                return;
            const float M = fmaxf(mx, mx_buf[(sb * 2 + (half ^ 1)) * HC + hh]);
            const float m_new = (t == 0 || M > m_ref + RESCALE_LOG2) ? M : m_ref;
            const bool rescale = t > 0 && m_new != m_ref;
            const float alpha = rescale ? fast_exp2(m_ref - m_new) : 1.f;
            m_ref = m_new;
            // ---- weights 2^(s - m): a bf16 high part and a bf16 remainder
            uint32_t whi[32], wlo[32];
            float ls = 0.f;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const float a = fast_exp2(sv[2 * j] - m_new);
                const float b = fast_exp2(sv[2 * j + 1] - m_new);
                ls += a + b;
                split_bf16x2(a, b, whi[j], wlo[j]);
            }
            l = l * alpha + ls;
            // ---- the previous value product must be done with the weights and with O
            if (kt > 0 && !warp_all(mbar_spin<false>(&bars->odone, (uint32_t)(kt - 1) & 1u, FLAG_MMA_WAIT, c.abort_flag)))
                return;
            tc_fence_after();
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int slot = (u ^ (hh & 7)) * 16;
                *reinterpret_cast<uint4 *>(row_hi + slot) =
                    make_uint4(whi[4 * u], whi[4 * u + 1], whi[4 * u + 2], whi[4 * u + 3]);
                *reinterpret_cast<uint4 *>(row_lo + slot) =
                    make_uint4(wlo[4 * u], wlo[4 * u + 1], wlo[4 * u + 2], wlo[4 * u + 3]);
            }
            // rescale this lane's 256 columns of O (warp-collective: the whole warp takes
            // the branch when any of its rows needs it, with factor 1 for the others)
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
                tmem_wait_st();
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(pready0);
        }
        // ---- end of the piece: the head's row sum, normalise, write
        const int klast = k + nt - 1;
        k += nt;
        lx_buf[half * HC + hh] = l;
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->lxbar);
        if (!warp_all(mbar_spin<false>(&bars->lxbar, (uint32_t)pi & 1u, FLAG_FULL_WAIT, c.abort_flag))) return;
        const float ltot = l + lx_buf[(half ^ 1) * HC + hh];
        const float lse_v = ltot > 0.f ? (m_ref + __log2f(ltot)) * 0.69314718055994531f : -INFINITY;
        const float inv = ltot > 0.f ? 1.f / ltot : 0.f;
        if (!warp_all(mbar_spin<false>(&bars->odone, (uint32_t)klast & 1u, FLAG_MMA_WAIT, c.abort_flag))) return;
        tc_fence_after();
        const bool real = head < p.H;
        float *dst = pc.whole ? p.out + ((size_t)pc.b * p.H + (real ? head : 0)) * 512
                              : p.ws_o + (((size_t)c.worker * 2 + pc.slot) * HR + head) * 512;
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                uint32_t ov[32];
                tmem_ld32(c.tmem + lane_base + TM_O + 128 * j + 32 * cc, ov);
                tmem_wait_ld();
                if (real) {
                    float4 *d4 = reinterpret_cast<float4 *>(dst + 256 * j + 128 * half + 32 * cc);
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        d4[e] = make_float4(__uint_as_float(ov[4 * e]) * inv, __uint_as_float(ov[4 * e + 1]) * inv,
                                            __uint_as_float(ov[4 * e + 2]) * inv, __uint_as_float(ov[4 * e + 3]) * inv);
                }
            }
        if (real && half == 0) {
            if (pc.whole)
                p.lse[(size_t)pc.b * p.H + head] = lse_v;
            else
                p.ws_lse[((size_t)c.worker * 2 + pc.slot) * HR + head] = lse_v;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(ofree0);
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
        for (int s = 0; s < NSS; ++s) {
            mbar_init(&bars->sfull[s], 1);
            mbar_init(&bars->sempty[s], 1);
        }
        for (int s = 0; s < NPV; ++s) {
            mbar_init(&bars->vfull[s], 1);
            mbar_init(&bars->vempty[s], 1);
        }
        mbar_init(&bars->qfull, 1);
        mbar_init(&bars->qempty, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars->sready[i], 1);
            mbar_init(&bars->sfree[i], 8);   // one arrival per softmax warp of either CTA
        }
        mbar_init(&bars->pready, 8);
        mbar_init(&bars->odone, 1);
        mbar_init(&bars->ofree, 8);
        mbar_init(&bars->mxbar[0], 4);
        mbar_init(&bars->mxbar[1], 4);
        mbar_init(&bars->lxbar, 4);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(tmem_ptr), TM_COLS);
        tmem_relinquish_pair();
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
    cluster_sync_all();   // both CTAs' barriers are initialised before any remote arrival

    Ctx c;
    c.smem = smem;
    c.bars = bars;
    c.abort_flag = abort_flag;
    c.s_prefix = s_prefix;
    c.tmem = *tmem_ptr;
    c.r = cluster_ctarank();
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
        if (warp == 0 && lane == 0) producer(p, maps, c);
        if (warp == 1 && lane == 0 && c.r == 0) mma_issuer(p, c);
        if (warp >= 4) softmax_warps(p, c, warp, lane);
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync_all();   // every pair MMA and remote arrival of both CTAs is done
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(c.tmem, TM_COLS);
    }
    cluster_sync_all();   // no CTA leaves before its peer has released the columns
}

}  // namespace kvattn
