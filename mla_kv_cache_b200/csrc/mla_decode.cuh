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
//     query rows, once per sequence -- latent columns [0, 256) in tensor memory (written
//     by the softmax threads, each row in lanes m and 64 + m), latent columns [256, 512)
//     and the RoPE part in shared memory (TMA) --, B = the 576-wide key rows of tile half
//     r (CTA r loads the half its B columns are).  9 chunks of 64 columns x 4 MMAs of
//     K = 16.  In tensor memory, lane m holds head 64r + m's scores of half 0's tokens,
//     lane 64 + m those of half 1's.
//   value product O += P C (M = 128 heads, N = 256 latent columns per MMA, two MMAs for
//     the 512 columns, K = 128 tokens): A = this CTA's weights P (shared memory, K-major),
//     B = the latent columns [256j + 128r, 256j + 128r + 128) of all 128 tokens (MN-major,
//     loaded by CTA r for both halves: the B columns it supplies).  Lane m holds head
//     64r + m's output columns 256j + [0, 128), lane 64 + m columns 256j + [128, 256).
//     It runs in two steps, token half 0 then token half 1, each committed on its own
//     barrier: the weights and the value slot of half 0 are free as soon as the first
//     step is done, so the next tile's half-0 weights are written while the second step
//     still runs, and the next tile's first step can follow this tile's second one
//     without a gap.
// Latent columns are thus read twice per pair (once as keys by the half's owner, once as
// values by each CTA for its columns), the second time from L2.
//
// Warp roles (384 threads per CTA):
//   warp 0, one thread   key producer (both CTAs): the shared-memory part of the query
//                        block once per sequence and a ring of three 24 KB key slots (one
//                        tile, one multi-chunk copy a slot); completions to rank 0.
//   warp 2, one thread   value producer (both CTAs): two 32 KB value slots (one copy each), one per token
//                        half of a tile, independent of the key stream; its loads hit L2
//                        (the keys' latent columns, loaded by the pair moments before).
// Each slot release is one tcgen05.commit, which costs the issuing thread ~300 cycles
// (measured, against ~56 for an MMA), so the slots are a few chunks each.
//   warp 1, one thread   score MMA issuer (rank 0 only), running ahead of the softmax by
//                        one tile (two score buffers).
//   warp 3, one thread   value MMA issuer (rank 0 only).
//   warps 4-11           softmax, two threads per tensor-memory lane (head 64r + m, tile
//                        half h; 32 score columns each): masks, partial tile maxima (the
//                        four parts of a head meet in shared memory), lazy running max
//                        (moves only when a tile's maximum exceeds it by more than 2^8;
//                        then this CTA's rows of O are rescaled in tensor memory), weights
//                        into shared memory, row sums; at the end of a piece the
//                        normalised result.  The warps of token half 0 (lanes 0-63) write
//                        the half-0 weights, those of half 1 the half-1 weights.
// End of a piece.  Each softmax warp owns a 32-head x 128-column block of O; it normalises
// the block and writes it row-contiguously (transposed through its own 4 KB of the
// weights buffer, so that eight lanes store one row's 128 bytes).  A sequence cut by a
// worker boundary leaves one partial block (and log-sum-exp) per worker in the
// workspace; the warp then counts itself in at a per-(sequence, rank, warp) counter, and
// the last of the sequence's workers to arrive merges that block's partials by
// log-sum-exp into the output (a sequence cut in two, after the worker's last piece:
// its own block again from tensor memory, only the other part's from the workspace).  No worker waits for another, and there is no second
// kernel.  Empty sequences (no worker) get out = 0, lse = -inf, spread over the workers.
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
constexpr int NQC = 9;                   // query / key chunks of 64 columns: 8 latent + 1 RoPE
constexpr int NQT = 4;                   // query chunks held in tensor memory (latent columns [0, 256))
constexpr int NQS = NQC - NQT;           // query chunks in shared memory (latent [256, 512) + RoPE)
constexpr int NKS = 3;                   // key ring: 3 slots of 3 chunks (192 columns), one tile
constexpr int NVS = 2;                   // value slots: one per token half (this CTA's 256 latent columns)
constexpr int KSLOT = 3 * CHUNK;         // 24 KB
constexpr int VSLOT = 4 * CHUNK;         // 32 KB
constexpr int NTHREADS = 384;            // warps 0-3: producers and MMA issuers, 4-11: softmax
constexpr int NSOFT = 8;                 // softmax warps
constexpr int MAX_BATCH = 1024;
constexpr float RESCALE_LOG2 = 8.f;      // rescale O only when the row max grows by > 2^8
constexpr uint32_t TM_O = 0;             // tensor memory columns [0, 256): O (two blocks of 128)
constexpr uint32_t TM_S = 256;           // [256, 384): the scores of two tiles (64 columns each)
constexpr uint32_t TM_Q = 384;           // [384, 512): query latent columns [0, 256), bf16 pairs
constexpr uint32_t TM_COLS = 512;

constexpr int OFF_Q = 0;                               // query chunks [5][64 heads x 128 B]
constexpr int OFF_P = OFF_Q + NQS * CHUNK;             // weights of a tile: high h0, h1, remainder h0, h1
constexpr int OFF_SR = OFF_P + 4 * CHUNK;              // key ring
constexpr int OFF_PV = OFF_SR + NKS * KSLOT;           // value ring
constexpr int OFF_END = OFF_PV + NVS * VSLOT;          // 208 KB
constexpr int OFF_MX = OFF_END + 8192;                 // (after the E4M3 layout's 216 KB too)
                                                       // [2 tiles][4 parts][64] partial tile maxima
constexpr int OFF_LX = OFF_MX + 2 * 4 * HC * 4;        // [4 parts][64] partial row sums
constexpr int OFF_QX = OFF_LX + 4 * HC * 4;            // [2][4 parts][64] partial query maxima (E4M3)
constexpr int OFF_BARS = OFF_QX + 2 * 4 * HC * 4;
constexpr int OFF_TMEMPTR = OFF_BARS + 512;
constexpr int OFF_ABORT = OFF_TMEMPTR + 16;
constexpr int OFF_PREFIX = OFF_ABORT + 16;
constexpr int smem_bytes(int B) { return 1024 + OFF_PREFIX + (B + 1) * 4; }
static_assert(smem_bytes(MAX_BATCH) <= 232448, "shared memory of the MLA kernel exceeds 227 KB");

// The E4M3 cache (one byte per code; a box is [64 rows x 128 codes], 128-byte swizzle, 8 KB).
// Shared memory: the query's high parts (5 boxes: latent codes 0-511, then the RoPE part in
// the first 64 codes of a fifth box) and its remainders, the weights' three parts ([64
// heads x 128 tokens] each), a key ring of two tiles (5 boxes per tile; the RoPE box is
// read from a 64-code-wide tensor, its other 64 codes are the TMA's zero fill and are
// never multiplied), and one value slot per token half (this CTA's 256 latent codes of
// the half's 64 tokens: 2 boxes).  216 KB.
namespace e4 {
constexpr int QPART = 5 * CHUNK;               // 40 KB: one part of the query
constexpr int OFF_Q = 0;
constexpr int OFF_P = OFF_Q + 2 * QPART;       // high part, middle part, low part
constexpr int NPP = 3;                         // parts of a weight
constexpr int PPART = CHUNK;                   // 8 KB
constexpr int OFF_SR = OFF_P + NPP * PPART;
constexpr int NKS = 2;                         // key ring: two tiles
constexpr int KSLOT = 5 * CHUNK;               // 40 KB
constexpr int OFF_PV = OFF_SR + NKS * KSLOT;
constexpr int VSLOT = 2 * CHUNK;               // 16 KB
static_assert(OFF_PV + NVS * VSLOT == OFF_MX, "E4M3 layout");
constexpr uint32_t TM_SR = 384;                // [384, 512): the RoPE part of the scores of two tiles
constexpr float RESCALE_LOG2 = 2.f;            // the weights stay below 2^(6 + 2) = 256 < 448
constexpr float P_LOG2 = 6.f;                  // the weights carry 2^6
}  // namespace e4

struct Bars {
    // Every ring slot serves each tile once, so its phase is the tile count.  The release
    // of a tile's last key slot is that tile's sready; a value slot and the weights of its
    // token half are released by that half's odone.
    uint64_t kfull[NKS];                // key ring (rank 0, both CTAs' bytes)
    uint64_t kempty[NKS - 1];           // release of key slots 0 and 1 (both CTAs)
    uint64_t sready[2];                 // the scores of a tile are in tensor memory (score buffer =
                                        // tile parity; both CTAs)
    uint64_t vfull[NVS];                // value slot of token half h (rank 0)
    uint64_t odone[2][2];               // [h][tile parity]: the half-h step of a tile's value product
                                        // is done (both CTAs); h = 1: the whole product
    uint64_t qfull;                     // shared-memory query chunks of both CTAs landed (rank 0)
    uint64_t qtm;                       // tensor-memory query columns written in both CTAs (rank 0)
    uint64_t qempty;                    // every score product of the piece has read Q (both CTAs)
    uint64_t sfree[2];                  // both CTAs have read them (rank 0: 8 warps x 2 CTAs)
    uint64_t pready[2][2];              // [h][tile parity], rank 0: the half-h weights are written
                                        // (h = 0 also: every rescale of O is done; all 16 softmax
                                        // warps arrive) -- h = 1: the 8 warps of half 1
    uint64_t ofree;                     // both CTAs' epilogues have read O (rank 0)
    uint64_t mxbar[2];                  // the softmax warps' tile maxima written (tile parity)
    uint64_t lxbar;                     // the softmax warps' row sums written (end of a piece)
    uint64_t qxbar;                     // the softmax warps' query maxima written (E4M3 cache)
};
static_assert(sizeof(Bars) <= 512, "barrier block overflows its slot");

}  // namespace mla

struct MlaParams {
    const __nv_bfloat16 *q_latent;   // [B, H, 512]
    const __nv_bfloat16 *q_rope;     // [B, H, 64]
    const int32_t *seq_lens;
    float *out;        // [B, H, 512]
    float *lse;        // [B, H]
    float *ws_lse;     // [workers, 2, 128]
    float *ws_o;       // [workers, 2, 128, 512]
    int B, H, T_max;
    int workers;       // CTA pairs
    int min_tiles;
    float scale_log2;
    const int32_t *block_table; // [B, max_pages] physical pages (paged cache); null: contiguous
    int max_pages;              // block-table columns
    int page_size;              // rows per page (T_max when contiguous)
    unsigned int epoch;         // number of this call (never 0), tags the merge counters
    float latent_scale;         // E4M3 cache: a latent code's value is code * latent_scale
    float rope_scale;           // E4M3 cache: a RoPE code's value is code * rope_scale
};

// rope / qrope: [pages][page rows][columns] boxes of [64 rows x 128 bytes]; latk / latk2:
// views [pages][chunk][page rows][64] whose chunk dimension strides 128 bytes inside a row
// (one copy moves a key slot's latent chunks: 3 and 2 of them in bf16, 4 in E4M3); latv: a
// 5-D view that moves a value slot in one copy; qlatc: the query's shared-memory latent
// chunks (bf16) in one copy.
struct MlaMaps {
    CUtensorMap rope, qrope, latk, latk2, latv, qlatc;
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
    long long W;       // tiles per worker
    long long p0, p1;
};

// Merge counters of the split sequences: one per (sequence, CTA rank, softmax warp), each
// counting the workers whose partial block of that warp has been written in the call
// numbered by its high 32 bits.  Zero at load; a call's first arrival re-tags it, and its
// last arrival sets the count back to zero under the same tag, so that a launch replayed
// with the same number (a captured CUDA graph) counts from zero again.  The tag keeps a
// call that stopped early (an error flag set) from corrupting the next call's count.
__device__ unsigned long long g_mla_merge_count[MAX_BATCH * 2 * NSOFT];

// One arrival of this call at a merge counter; true for the last of n arrivals.  The
// compare-and-swap loop retries only when another arrival got in between.
__device__ __forceinline__ bool merge_arrive_last(unsigned long long *cnt, unsigned int epoch, int n) {
    unsigned long long cur = *reinterpret_cast<volatile unsigned long long *>(cnt);
    unsigned long long nxt = 0;
    for (int i = 0; i < (1 << 20); ++i) {
        nxt = (unsigned int)(cur >> 32) == epoch ? cur + 1 : ((unsigned long long)epoch << 32) | 1ull;
        const unsigned long long prev = atomicCAS(cnt, cur, nxt);
        if (prev == cur) {
            const bool last = (unsigned int)(nxt & 0xffffffffull) == (unsigned int)n;
            // every arrival of this launch is in: no one reads the count again before the
            // next launch
            if (last) atomicExch(cnt, (unsigned long long)epoch << 32);
            return last;
        }
        cur = prev;
    }
    atomicOr(&g_device_flags, FLAG_PEER_WAIT);
    return false;
}

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

// ------------------------------------------------------------------ producers
// Two threads per CTA, one per ring, each loading in the order the MMAs consume its
// ring: the key producer (warp 0) the shared-memory query chunks of a sequence, then the
// key chunks of every tile of the piece; the value producer (warp 2) the value chunks of
// every tile.  Completions go to rank 0's barriers, which rank 0 arms with the bytes of
// both CTAs.
template <bool KV8>
__device__ __forceinline__ void key_producer(const MlaParams &p, const MlaMaps &m, const Ctx &c) {
    Bars *bars = c.bars;
    const uint64_t pol_keep = l2_policy_evict_normal();   // the latent columns are read again as values
    const bool lead = c.r == 0;
    const uint32_t qfull0 = map_to_rank(smem_u32(&bars->qfull), 0);
    int nld = 0, pi = 0;
    bool ok = true;
    for (long long pos = c.p0; pos < c.p1 && ok; ++pi) {
        const Piece pc = piece_at(c.s_prefix, p.B, 1, pos, c.p1, c.p0);
        pos = pc.ustart + pc.lt1;
        const int len = clamp_len(__ldg(p.seq_lens + pc.b), p.T_max);
        if constexpr (KV8) {
            // one slot per tile, two slots: tile nld's slot last held tile nld - 2, whose
            // score product's completion (sready of its parity) frees it
            for (int lt = pc.lt0; lt < pc.lt1 && ok; ++lt, ++nld) {
                const int slot = nld % e4::NKS;
                if (nld >= e4::NKS && !mbar_wait(&bars->sready[nld & 1], (uint32_t)((nld - 2) >> 1) & 1u,
                                                 FLAG_EMPTY_WAIT, c.abort_flag)) {
                    ok = false;
                    break;
                }
                const HalfSrc hs = half_source(p, pc.b, len, lt, (int)c.r);
                if (lead) mbar_arrive_expect_tx(&bars->kfull[slot], 2 * e4::KSLOT);
                const uint32_t bar = map_to_rank(smem_u32(&bars->kfull[slot]), 0);
                uint8_t *dst = c.smem + e4::OFF_SR + slot * e4::KSLOT;
                tma_load_4d_pair(dst, &m.latk, bar, 0, hs.y, 0, hs.page, pol_keep);   // latent chunks 0..3
                tma_load_3d_pair(dst + 4 * CHUNK, &m.rope, bar, 0, hs.y, hs.page, pol_keep);
            }
            continue;
        }
        // this CTA's 64 query rows: latent chunks 4..7 and the RoPE chunk
        if (pi > 0 && !mbar_wait(&bars->qempty, (uint32_t)(pi - 1) & 1u, FLAG_EMPTY_WAIT, c.abort_flag)) {
            ok = false;
            break;
        }
        if (lead) mbar_arrive_expect_tx(&bars->qfull, 2 * NQS * CHUNK);
        tma_load_4d_pair(c.smem + OFF_Q, &m.qlatc, qfull0, 0, HC * (int)c.r, NQT, pc.b, pol_keep);   // chunks 4..7
        tma_load_3d_pair(c.smem + OFF_Q + (NQS - 1) * CHUNK, &m.qrope, qfull0, 0, HC * (int)c.r, pc.b, pol_keep);
        for (int lt = pc.lt0; lt < pc.lt1 && ok; ++lt) {
            const HalfSrc hs = half_source(p, pc.b, len, lt, (int)c.r);
            for (int s = 0; s < NKS; ++s, ++nld) {
                // slot s of the previous tile must have been read: slots 0 and 1 have their
                // own release barrier, the last slot's is the previous tile's sready
                const int kt = nld / NKS;
                const bool freed = s < NKS - 1
                    ? mbar_wait(&bars->kempty[s], ((uint32_t)kt & 1u) ^ 1u, FLAG_EMPTY_WAIT, c.abort_flag)
                    : (kt == 0 || mbar_wait(&bars->sready[(kt - 1) & 1], (uint32_t)((kt - 1) >> 1) & 1u,
                                            FLAG_EMPTY_WAIT, c.abort_flag));
                if (!freed) {
                    ok = false;
                    break;
                }
                if (lead) mbar_arrive_expect_tx(&bars->kfull[s], 2 * KSLOT);
                const uint32_t bar = map_to_rank(smem_u32(&bars->kfull[s]), 0);
                uint8_t *dst = c.smem + OFF_SR + s * KSLOT;
                if (s < NKS - 1) {   // latent chunks 3s .. 3s + 2
                    tma_load_4d_pair(dst, &m.latk, bar, 0, hs.y, 3 * s, hs.page, pol_keep);
                } else {             // latent chunks 6, 7 and the RoPE chunk
                    tma_load_4d_pair(dst, &m.latk2, bar, 0, hs.y, 6, hs.page, pol_keep);
                    tma_load_3d_pair(dst + 2 * CHUNK, &m.rope, bar, 0, hs.y, hs.page, pol_keep);
                }
            }
        }
    }
    if (!ok && lead) {
        // Let the copies already issued land before the CTAs can exit.
        constexpr int nks = KV8 ? e4::NKS : NKS;
        for (int i = (nld > nks ? nld - nks : 0); i < nld; ++i)
            mbar_wait_sleep(&bars->kfull[i % nks], (uint32_t)(i / nks) & 1u, FLAG_FULL_WAIT, nullptr);
        if (!KV8 && pi > 0) mbar_wait_sleep(&bars->qfull, (uint32_t)(pi - 1) & 1u, FLAG_FULL_WAIT, nullptr);
    }
}

template <bool KV8>
__device__ __forceinline__ void value_producer(const MlaParams &p, const MlaMaps &m, const Ctx &c) {
    Bars *bars = c.bars;
    const uint64_t pol_last = l2_policy_evict_first();    // the values' read is the last one
    const bool lead = c.r == 0;
    int nld = 0;
    bool ok = true;
    for (long long pos = c.p0; pos < c.p1 && ok;) {
        const Piece pc = piece_at(c.s_prefix, p.B, 1, pos, c.p1, c.p0);
        pos = pc.ustart + pc.lt1;
        const int len = clamp_len(__ldg(p.seq_lens + pc.b), p.T_max);
        for (int lt = pc.lt0; lt < pc.lt1 && ok; ++lt) {
            for (int h = 0; h < NVS; ++h, ++nld) {
                // slot h is free once the previous tile's half-h step is done
                const int kt = nld / NVS;
                if (kt > 0 && !mbar_wait(&bars->odone[h][(kt - 1) & 1], (uint32_t)((kt - 1) >> 1) & 1u,
                                         FLAG_EMPTY_WAIT, c.abort_flag)) {
                    ok = false;
                    break;
                }
                const HalfSrc hs = half_source(p, pc.b, len, lt, h);
                constexpr int vslot = KV8 ? e4::VSLOT : VSLOT;
                if (lead) mbar_arrive_expect_tx(&bars->vfull[h], 2 * vslot);
                const uint32_t bar = map_to_rank(smem_u32(&bars->vfull[h]), 0);
                uint8_t *dst = c.smem + (KV8 ? e4::OFF_PV : OFF_PV) + h * vslot;
                // this CTA's columns of latent blocks j = 0, 1 in one copy: bf16 chunks
                // 4j + 2r + {0, 1}, E4M3 128-code chunks 2j + r; shared memory [j][chunk]
                tma_load_5d_pair(dst, &m.latv, bar, 0, hs.y, (KV8 ? 1 : 2) * (int)c.r, 0, hs.page, pol_last);
            }
        }
    }
    if (!ok && lead)
        for (int i = (nld > NVS ? nld - NVS : 0); i < nld; ++i)
            mbar_wait_sleep(&bars->vfull[i % NVS], (uint32_t)(i / NVS) & 1u, FLAG_FULL_WAIT, nullptr);
}

// ------------------------------------------------------------------ MMA issuer (rank 0, warp 1, lane 0)
// Waits of the issuing threads on barriers that the softmax warps of both CTAs arrive on.
// The issuers share their SM sub-partitions with softmax warps, so they wait with
// try_wait (which suspends the thread for a while between tests) rather than polling.
__device__ __forceinline__ bool wait_remote(uint64_t *bar, uint32_t parity, const Ctx &c) {
    return mbar_wait(bar, parity, FLAG_PEER_WAIT, c.abort_flag);
}

// Two issuing threads: the score products (warp 1) and the value products (warp 3).  A
// thread can issue a tcgen05.mma only every ~60 cycles, about the tensor time of one
// N = 128 pair MMA, so one thread could not keep the tensor pipe busy with both streams;
// the two streams use different accumulators and each thread commits its own MMAs.
// Shared-memory descriptors are formed once; an operand's descriptor is the template
// plus its address in 16-byte units (the start field never carries: shared addresses
// are below 2^18), so the issue loops add constants only.

// S of every tile into score buffer kt & 1: 9 chunks x 4 K-steps of 16 (E4M3: 4 latent
// boxes x 4 K-steps of 32 codes, each times the query's high part and its remainder; the
// RoPE box's 2 K-steps into a score buffer of their own, since the RoPE codes have their
// own scale).
template <bool KV8>
__device__ __forceinline__ void score_issuer(const MlaParams &p, const Ctx &c) {
    Bars *bars = c.bars;
    if constexpr (KV8) {
        constexpr uint32_t id_s = idesc_e4m3(128, TILE, 0, 0);     // K-major A and B
        const uint64_t tmpl = smem_desc_sw128(0, 16, 1024);
        const uint64_t q_desc = tmpl + (smem_u32(c.smem + e4::OFF_Q) >> 4);
        const uint64_t kr_desc = tmpl + (smem_u32(c.smem + e4::OFF_SR) >> 4);
        int k = 0, pi = 0;
        for (long long pos = c.p0; pos < c.p1; ++pi) {
            const Piece pc = piece_at(c.s_prefix, p.B, 1, pos, c.p1, c.p0);
            pos = pc.ustart + pc.lt1;
            const int nt = pc.lt1 - pc.lt0;
            // the query parts are written by the softmax warps of both CTAs
            if (!wait_remote(&bars->qtm, (uint32_t)pi & 1u, c)) return;
            tc_fence_after();
            for (int kt = k; kt < k + nt; ++kt) {
                const int sb = kt & 1, slot = kt % e4::NKS;
                const uint32_t d = c.tmem + TM_S + 64 * sb;
                if (kt >= 2 && !wait_remote(&bars->sfree[sb], (uint32_t)((kt >> 1) - 1) & 1u, c)) return;
                if (!mbar_wait(&bars->kfull[slot], (uint32_t)(kt / e4::NKS) & 1u, FLAG_FULL_WAIT, c.abort_flag))
                    return;
                tc_fence_after();
                const uint64_t kb = kr_desc + (uint64_t)((slot * e4::KSLOT) >> 4);
#pragma unroll
                for (int ch = 0; ch < 5; ++ch) {
                    const uint32_t dd = ch < 4 ? d : c.tmem + e4::TM_SR + 64 * sb;
#pragma unroll
                    for (int kk = 0; kk < (ch < 4 ? 4 : 2); ++kk) {   // +32 bytes per K-step
                        const uint64_t off = (uint64_t)((ch * CHUNK + kk * 32) >> 4);
                        const uint32_t acc = ((ch & 3) | kk) != 0 ? 1u : 0u;   // (ch 4: a new accumulator)
                        umma_pair_ss_f8(dd, q_desc + off, kb + off, id_s, acc);
                        umma_pair_ss_f8(dd, q_desc + off + (uint64_t)(e4::QPART >> 4), kb + off, id_s, 1u);
                    }
                }
                umma_pair_commit_both(&bars->sready[sb]);   // also frees the key slot
            }
            umma_pair_commit_both(&bars->qempty);
            k += nt;
        }
        return;
    }
    constexpr uint32_t id_s = idesc_f16(128, TILE, 1, 1, 0);   // K-major A and B
    const uint64_t k_tmpl = smem_desc_sw128(0, 16, 1024);       // K-major, 128-byte swizzle
    const uint64_t q_desc = k_tmpl + (smem_u32(c.smem + OFF_Q) >> 4);
    const uint64_t kr_desc = k_tmpl + (smem_u32(c.smem + OFF_SR) >> 4);
    const uint32_t tm_q = c.tmem + TM_Q;
    int k = 0, pi = 0;
    for (long long pos = c.p0; pos < c.p1; ++pi) {
        const Piece pc = piece_at(c.s_prefix, p.B, 1, pos, c.p1, c.p0);
        pos = pc.ustart + pc.lt1;
        const int nt = pc.lt1 - pc.lt0;
        if (!mbar_wait(&bars->qfull, (uint32_t)pi & 1u, FLAG_FULL_WAIT, c.abort_flag)) return;
        if (!wait_remote(&bars->qtm, (uint32_t)pi & 1u, c)) return;
        tc_fence_after();
        for (int kt = k; kt < k + nt; ++kt) {
            const int sb = kt & 1;
            const uint32_t d = c.tmem + TM_S + 64 * sb;
            if (kt >= 2 && !wait_remote(&bars->sfree[sb], (uint32_t)((kt >> 1) - 1) & 1u, c)) return;
            for (int s = 0; s < NKS; ++s) {
                if (!mbar_wait(&bars->kfull[s], (uint32_t)kt & 1u, FLAG_FULL_WAIT, c.abort_flag)) return;
                tc_fence_after();
#pragma unroll
                for (int e = 0; e < 3; ++e) {
                    const int ch = 3 * s + e;
                    const uint64_t bd = kr_desc + (uint64_t)((s * KSLOT + e * CHUNK) >> 4);
                    if (ch < NQT) {
                        const uint32_t a = tm_q + 32 * ch;
                        umma_pair_ts(d, a, bd, id_s, ch != 0);
                        umma_pair_ts(d, a + 8, bd + 2, id_s, 1u);
                        umma_pair_ts(d, a + 16, bd + 4, id_s, 1u);
                        umma_pair_ts(d, a + 24, bd + 6, id_s, 1u);
                    } else {
                        const uint64_t ad = q_desc + (uint64_t)((ch - NQT) * (CHUNK >> 4));
                        umma_pair_ss(d, ad, bd, id_s, 1u);
                        umma_pair_ss(d, ad + 2, bd + 2, id_s, 1u);
                        umma_pair_ss(d, ad + 4, bd + 4, id_s, 1u);
                        umma_pair_ss(d, ad + 6, bd + 6, id_s, 1u);
                    }
                }
                if (s < NKS - 1)
                    umma_pair_commit_both(&bars->kempty[s]);
                else
                    umma_pair_commit_both(&bars->sready[sb]);   // releases the last slot too
            }
        }
        umma_pair_commit_both(&bars->qempty);   // the piece's score products are done with Q
        k += nt;
    }
}

// O += P_hi C + P_lo C for every tile kt: token halves h (one commit each), latent
// blocks j, K-steps of 16 tokens (E4M3: 32).
template <bool KV8>
__device__ __forceinline__ void value_issuer(const MlaParams &p, const Ctx &c) {
    Bars *bars = c.bars;
    constexpr uint32_t id_v = idesc_f16(128, 256, 1, 1, 1);    // B (the latents) MN-major
    constexpr uint32_t id_v8 = idesc_e4m3(128, 256, 0, 1);
    const uint64_t k_tmpl = smem_desc_sw128(0, 16, 1024);       // K-major, 128-byte swizzle
    // MN-major: bf16 -- the two 64-column chunks 8 KB apart; E4M3 -- one 128-code row per token
    const uint64_t v_tmpl = smem_desc_sw128(0, CHUNK, 1024);
    const uint64_t p_desc = k_tmpl + (smem_u32(c.smem + (KV8 ? e4::OFF_P : OFF_P)) >> 4);
    const uint64_t vr_desc = v_tmpl + (smem_u32(c.smem + (KV8 ? e4::OFF_PV : OFF_PV)) >> 4);
    int k = 0, pi = 0;
    for (long long pos = c.p0; pos < c.p1; ++pi) {
        const Piece pc = piece_at(c.s_prefix, p.B, 1, pos, c.p1, c.p0);
        pos = pc.ustart + pc.lt1;
        const int nt = pc.lt1 - pc.lt0;
        // the previous piece's epilogue must have read O before the first product overwrites it
        if (pi > 0 && !wait_remote(&bars->ofree, (uint32_t)(pi - 1) & 1u, c)) return;
        for (int kt = k; kt < k + nt; ++kt) {
            const bool first = kt == k;
#pragma unroll 1
            for (int h = 0; h < 2; ++h) {
                if (!wait_remote(&bars->pready[h][kt & 1], (uint32_t)(kt >> 1) & 1u, c)) return;
                if (!mbar_wait(&bars->vfull[h], (uint32_t)kt & 1u, FLAG_FULL_WAIT, c.abort_flag)) return;
                tc_fence_after();
                if constexpr (KV8) {
                    // weights: K-major [64 heads x 128 tokens], half h = bytes [64h, 64h + 64) of
                    // each row; values: MN-major, 32 tokens = 4 KB per K-step
#pragma unroll
                    for (int jb = 0; jb < 2; ++jb) {
                        const uint32_t d = c.tmem + TM_O + 128 * jb;
                        const uint64_t bd = vr_desc + (uint64_t)((h * e4::VSLOT + jb * CHUNK) >> 4);
#pragma unroll
                        for (int kk = 0; kk < 2; ++kk) {
                            const uint64_t pa = p_desc + (uint64_t)(((2 * h + kk) * 32) >> 4);
                            const uint64_t vb = bd + (uint64_t)((kk * 4096) >> 4);
                            umma_pair_ss_f8(d, pa, vb, id_v8, (!first || h > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
                            for (int pp = 1; pp < e4::NPP; ++pp)
                                umma_pair_ss_f8(d, pa + (uint64_t)((pp * e4::PPART) >> 4), vb, id_v8, 1u);
                        }
                    }
                    umma_pair_commit_both(&bars->odone[h][kt & 1]);
                    continue;
                }
                const uint64_t hi = p_desc + (uint64_t)(h * (CHUNK >> 4));
                const uint64_t lo = hi + (uint64_t)(2 * (CHUNK >> 4));
#pragma unroll
                for (int jb = 0; jb < 2; ++jb) {
                    const uint32_t d = c.tmem + TM_O + 128 * jb;
                    const uint64_t bd = vr_desc + (uint64_t)((h * VSLOT + jb * 2 * CHUNK) >> 4);
                    umma_pair_ss(d, hi, bd, id_v, (!first || h > 0) ? 1u : 0u);
                    umma_pair_ss(d, lo, bd, id_v, 1u);
#pragma unroll
                    for (int kk = 1; kk < 4; ++kk) {   // next 16 tokens: +32 B in the weights, +2 KB in the latents
                        umma_pair_ss(d, hi + 2 * kk, bd + 128 * kk, id_v, 1u);
                        umma_pair_ss(d, lo + 2 * kk, bd + 128 * kk, id_v, 1u);
                    }
                }
                umma_pair_commit_both(&bars->odone[h][kt & 1]);   // frees value slot h and the half-h weights
            }
        }
        k += nt;
    }
}

// ------------------------------------------------------------------ softmax (warps 4-11)
// Two warps per tensor-memory lane quadrant: warp 4 + 4cg + q takes score columns
// [32cg, 32cg + 32) of the lanes of quadrant q, i.e. 32 of the 64 tokens of its tile half.
// The four partial tile maxima of a head (two halves x two column groups) meet in shared
// memory, as do its four partial row sums at the end of a piece.  Column group cg also
// owns O's block j = cg in the lane (its rescale, its epilogue) and half of the lane's
// query columns in tensor memory.
// Waits use try_wait (the thread is suspended between tests) so that waiting softmax
// warps leave the issue slots to the producer and MMA threads on the same sub-partition.
__device__ __forceinline__ bool wait_local(uint64_t *bar, uint32_t parity, unsigned int flag, const Ctx &c) {
    return warp_all(mbar_wait(bar, parity, flag, c.abort_flag));
}

template <bool KV8>
__device__ __forceinline__ void softmax_warps(const MlaParams &p, const Ctx &c, int warp, int lane) {
    Bars *bars = c.bars;
    constexpr float RESCALE = KV8 ? e4::RESCALE_LOG2 : RESCALE_LOG2;
    const int q = warp & 3;                     // tensor-memory lane quadrant
    const int cg = (warp - 4) >> 2;             // column group: score columns [32cg, 32cg + 32)
    const int L = 32 * q + lane;                // tensor-memory lane
    const int hh = L & (HC - 1);                // head row of this CTA
    const int half = L >> 6;                    // tile half whose scores the lane holds
    const int part = 2 * half + cg;             // this thread's share of the head's tile
    const int head = HC * (int)c.r + hh;
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    float *mx_buf = reinterpret_cast<float *>(c.smem + OFF_MX);   // [2 tiles][4 parts][64]
    float *lx_buf = reinterpret_cast<float *>(c.smem + OFF_LX);   // [4 parts][64]
    const uint32_t sfree0 = map_to_rank(smem_u32(&bars->sfree[0]), 0);
    const uint32_t sfree1 = map_to_rank(smem_u32(&bars->sfree[1]), 0);
    // the weights-ready barriers this thread arrives on (rank 0), by tile parity: the
    // first step's (every warp) and its own half's
    const uint32_t pready_first0 = map_to_rank(smem_u32(&bars->pready[0][0]), 0);
    const uint32_t pready_first1 = map_to_rank(smem_u32(&bars->pready[0][1]), 0);
    const uint32_t pready_own0 = map_to_rank(smem_u32(&bars->pready[half][0]), 0);
    const uint32_t pready_own1 = map_to_rank(smem_u32(&bars->pready[half][1]), 0);
    const uint32_t ofree0 = map_to_rank(smem_u32(&bars->ofree), 0);
    const uint32_t qtm0 = map_to_rank(smem_u32(&bars->qtm), 0);
    // this thread's 32 tokens of the weights: row hh of the half's K-major chunk, 16-byte
    // units 4cg .. 4cg + 3 (128-byte swizzle)
    uint8_t *row_hi = c.smem + OFF_P + half * CHUNK + hh * 128;
    uint8_t *row_lo = row_hi + 2 * CHUNK;
    // E4M3: row hh of the weights' [64 heads x 128 tokens] parts, units 4 half + 2 cg + {0, 1}
    uint8_t *row8_hi = c.smem + e4::OFF_P + hh * 128;
    // score scale in log2 units (E4M3: the scores arrive scaled, sl2 = 1; sl2_lat / sl2_rope
    // are the scale times the codes' scale and 2^-e of the head's query part)
    const float sl2 = KV8 ? 1.f : p.scale_log2;
    float sl2_lat = 0.f, sl2_rope = 0.f;

    // Query latent columns [64cg, 64cg + 64) (bf16 pairs) of this lane's head of sequence
    // b: loaded into registers, then (once the previous piece's score products are done
    // with the columns) written to tensor memory; both lanes of a head hold the row.
    const bool realq = head < p.H;
    auto q_row = [&](int b) {
        return reinterpret_cast<const uint4 *>(p.q_latent + ((size_t)b * p.H + (realq ? head : 0)) * 512) + 16 * cg;
    };
    auto load_q = [&](int b, uint32_t (&v0)[32], uint32_t (&v1)[32]) {
        const uint4 *qrow = q_row(b);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            uint4 x = make_uint4(0, 0, 0, 0), y = make_uint4(0, 0, 0, 0);
            if (realq) {
                x = __ldg(qrow + e);
                y = __ldg(qrow + 8 + e);
            }
            v0[4 * e] = x.x; v0[4 * e + 1] = x.y; v0[4 * e + 2] = x.z; v0[4 * e + 3] = x.w;
            v1[4 * e] = y.x; v1[4 * e + 1] = y.y; v1[4 * e + 2] = y.z; v1[4 * e + 3] = y.w;
        }
    };
    auto store_q = [&](uint32_t (&v0)[32], uint32_t (&v1)[32]) {
        tc_fence_after();
        tmem_st32(c.tmem + lane_base + TM_Q + 64 * cg, v0);
        tmem_st32(c.tmem + lane_base + TM_Q + 64 * cg + 32, v1);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(qtm0);
    };
    // E4M3 cache: the query of this thread's head as an E4M3 high part and remainder after
    // scaling by 2^e (the largest magnitude of its latent part, and separately of its RoPE
    // part, lands in [128, 256)), written into the shared-memory query boxes: exact for
    // bf16 values (a bf16 significand's eight bits minus the high part's four leave a
    // remainder of at most four).  The head's 36 16-code units (32 latent, 4 RoPE) are
    // shared by its four threads, nine each; their maxima meet in shared memory.
    float *qx_buf = reinterpret_cast<float *>(c.smem + OFF_QX);   // [latent / RoPE][4 parts][64]
    int q8_uses = 0;
    auto q8_src = [&](int b, int i) -> const uint4 * {   // 16-byte load i (0..17) of this thread's units
        const int unit = 9 * part + (i >> 1);
        const size_t row = (size_t)b * p.H + (realq ? head : 0);
        return unit < 32 ? reinterpret_cast<const uint4 *>(p.q_latent + row * 512) + 2 * unit + (i & 1)
                         : reinterpret_cast<const uint4 *>(p.q_rope + row * 64) + 2 * (unit - 32) + (i & 1);
    };
    // The 16 bytes of unit u's high part; its remainder's are e4::QPART further on.  The
    // unit's 32 raw bytes (bf16) are first parked in those same bytes, which no other
    // thread reads or writes, and converted in place.
    auto q8_dst = [&](int u) -> uint8_t * {
        const int box = u < 32 ? u >> 3 : 4;
        const int g = u < 32 ? u & 7 : u - 32;
        return c.smem + e4::OFF_Q + box * CHUNK + hh * 128 + ((g ^ (hh & 7)) << 4);
    };
    // First pass (the query boxes free): the 18 asynchronous copies all in flight at once,
    // then the largest magnitudes of this thread's latent and RoPE values.
    auto q8_load = [&](int b, float &mxl, float &mxr) {
#pragma unroll
        for (int i = 0; i < 18; ++i) {
            uint8_t *d = q8_dst(9 * part + (i >> 1)) + (i & 1) * e4::QPART;
            if (realq) cp_async16(d, q8_src(b, i));
            else *reinterpret_cast<uint4 *>(d) = make_uint4(0, 0, 0, 0);
        }
        cp_async_wait_all();
        mxl = 0.f;
        mxr = 0.f;
#pragma unroll
        for (int i = 0; i < 18; ++i) {
            const uint4 x = *reinterpret_cast<const uint4 *>(q8_dst(9 * part + (i >> 1)) + (i & 1) * e4::QPART);
            const uint32_t w[4] = {x.x, x.y, x.z, x.w};
            float m = 0.f;
#pragma unroll
            for (int t = 0; t < 4; ++t) m = fmaxf(m, fmaxf(fabsf(bf16_lo(w[t])), fabsf(bf16_hi(w[t]))));
            if (9 * part + (i >> 1) < 32) mxl = fmaxf(mxl, m); else mxr = fmaxf(mxr, m);
        }
    };
    // Second pass: the head's scales, then each parked unit split in place.
    auto q8_store = [&](float mxl, float mxr) -> bool {
        qx_buf[part * HC + hh] = mxl;
        qx_buf[4 * HC + part * HC + hh] = mxr;
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->qxbar);
        if (!wait_local(&bars->qxbar, (uint32_t)q8_uses & 1u, FLAG_FULL_WAIT, c)) return false;
        ++q8_uses;
        // 2^e that puts a part's largest magnitude in [128, 256)
        auto pow2_exp = [](float M) -> int {
            int e = 0;
            if (M > 0.f && M <= 3.0e38f) {
                int ex;
                frexpf(M, &ex);             // M in [2^(ex-1), 2^ex)
                e = min(max(8 - ex, -120), 120);
            }
            return e;
        };
        const float *qr = qx_buf + 4 * HC;
        const int el = pow2_exp(fmaxf(fmaxf(qx_buf[hh], qx_buf[HC + hh]), fmaxf(qx_buf[2 * HC + hh], qx_buf[3 * HC + hh])));
        const int er = pow2_exp(fmaxf(fmaxf(qr[hh], qr[HC + hh]), fmaxf(qr[2 * HC + hh], qr[3 * HC + hh])));
        sl2_lat = p.scale_log2 * p.latent_scale * __int_as_float((127 - el) << 23);
        sl2_rope = p.scale_log2 * p.rope_scale * __int_as_float((127 - er) << 23);
#pragma unroll 3
        for (int i = 0; i < 9; ++i) {
            const int unit = 9 * part + i;
            const float up = __int_as_float((127 + (unit < 32 ? el : er)) << 23);
            uint8_t *dst = q8_dst(unit);
            const uint4 xs[2] = {*reinterpret_cast<const uint4 *>(dst),
                                 *reinterpret_cast<const uint4 *>(dst + e4::QPART)};
            uint32_t hw[4], lw[4];
#pragma unroll
            for (int t = 0; t < 4; ++t) {   // codes 4t .. 4t + 3 of the unit: words 2t, 2t + 1 of the pair
                const uint4 &x = xs[t >> 1];
                const uint32_t w0 = (t & 1) ? x.z : x.x, w1 = (t & 1) ? x.w : x.y;
                uint16_t h0, l0, h1, l1;
                split_e4m3x2(bf16_lo(w0) * up, bf16_hi(w0) * up, h0, l0);
                split_e4m3x2(bf16_lo(w1) * up, bf16_hi(w1) * up, h1, l1);
                hw[t] = (uint32_t)h0 | ((uint32_t)h1 << 16);
                lw[t] = (uint32_t)l0 | ((uint32_t)l1 << 16);
            }
            *reinterpret_cast<uint4 *>(dst) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
            *reinterpret_cast<uint4 *>(dst + e4::QPART) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(qtm0);
        return true;
    };
    // Rescale block cg of this lane's O by alpha (warp-collective).
    auto rescale_o = [&](float alpha) {
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
            const uint32_t addr = c.tmem + lane_base + TM_O + 128 * cg + 32 * cc;
            uint32_t ov[32];
            tmem_ld32(addr, ov);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) ov[j] = __float_as_uint(__uint_as_float(ov[j]) * alpha);
            tmem_st32(addr, ov);
        }
        tmem_wait_st();
    };

    // This warp's block of O: rows head0 + [0, 32) (this CTA's heads 32 (q & 1) + ..), columns
    // col0 + [0, 128) of the 512.
    const int head0 = HC * (int)c.r + 32 * (q & 1);
    const int col0 = 256 * cg + 128 * half;
    // 16-byte unit u (0 .. SU - 1) of row rr (0..31) of the warp's transpose scratch: the
    // warp's own units of the weights buffer.  bf16: row 32 (q & 1) + rr of its half's
    // chunk, units 4cg..4cg+3 of the high part for u < 4, of the remainder for u >= 4 (SU =
    // 8, 4 KB).  E4M3: row 32 (q & 1) + rr, units 4 half + 2 cg + {0, 1} of the high part for
    // u < 2, of the remainder for u >= 2 (SU = 4, 2 KB).
    constexpr int SU = KV8 ? 4 : 8;
    auto scratch_unit = [&](int rr, int u) -> uint8_t * {
        const int row = 32 * (q & 1) + rr;
        if constexpr (KV8)
            return c.smem + e4::OFF_P + (u >> 1) * e4::PPART + row * 128 +
                   (((4 * half + 2 * cg + (u & 1)) ^ (row & 7)) * 16);
        return c.smem + OFF_P + half * CHUNK + (u >> 2) * 2 * CHUNK + row * 128 +
               (((4 * cg + (u & 3)) ^ (row & 7)) * 16);
    };
    // Merge of the partial blocks of sequence b written by its n_parts workers (all
    // arrived): out = sum_c exp(lse_c - lse) o_c, lse = log sum_c exp(lse_c).  Lane L
    // takes the log-sum-exp of row L and puts the row's weights exp(lse_c - lse) in the
    // warp's scratch (32 parts at a time); each load instruction then reads four rows'
    // 128 contiguous bytes (eight lanes per row).  The partials are read through L2
    // (other SMs wrote them), and the merge is a chain of L2 round trips, so it keeps
    // many loads in flight: up to NPR parts' log-sum-exps are read once, together, and
    // two parts' loads of one column chunk go together.
    auto merge_block = [&](int b, long long ustart, int n_parts) {
        const long long c_first = ustart / c.W;
        auto part_row = [&](int j, int h) -> size_t {
            const long long cw = c_first + j;
            const int slot = (ustart <= cw * c.W) ? 0 : 1;
            return ((size_t)cw * 2 + slot) * HR + h;
        };
        const int hl = head0 + lane;
        constexpr int NPR = 4;
        const bool few = n_parts <= NPR;
        float lv[NPR];
        float M = -INFINITY;
        if (few) {
#pragma unroll
            for (int u = 0; u < NPR; ++u) lv[u] = u < n_parts ? __ldcg(p.ws_lse + part_row(u, hl)) : -INFINITY;
#pragma unroll
            for (int u = 0; u < NPR; ++u) M = fmaxf(M, lv[u]);
        } else {
            for (int j0 = 0; j0 < n_parts; j0 += 4) {
                float v[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) v[u] = j0 + u < n_parts ? __ldcg(p.ws_lse + part_row(j0 + u, hl)) : -INFINITY;
#pragma unroll
                for (int u = 0; u < 4; ++u) M = fmaxf(M, v[u]);
            }
        }
        float S = 0.f;
        if (M != -INFINITY) {
            if (few) {
#pragma unroll
                for (int u = 0; u < NPR; ++u)
                    S += lv[u] == -INFINITY ? 0.f : fast_exp2((lv[u] - M) * 1.4426950408889634f);
            } else {
                for (int j0 = 0; j0 < n_parts; j0 += 4) {
                    float v[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) v[u] = j0 + u < n_parts ? __ldcg(p.ws_lse + part_row(j0 + u, hl)) : -INFINITY;
#pragma unroll
                    for (int u = 0; u < 4; ++u) S += v[u] == -INFINITY ? 0.f : fast_exp2((v[u] - M) * 1.4426950408889634f);
                }
            }
        }
        const float lse_all = S > 0.f ? M + __logf(S) : -INFINITY;
        // the scratch as [JB parts][32 rows] floats (the warp's own units of the weights
        // buffer: scratch_unit(r, u), 4 floats each)
        constexpr int JB = 4 * SU;
        auto wslot = [&](int j, int rr) -> float * {   // weight of part j (< JB) for row rr
            const int e = 32 * j + rr;
            return reinterpret_cast<float *>(scratch_unit(e / (4 * SU), (e % (4 * SU)) >> 2)) + (e & 3);
        };
        for (int jb = 0; jb < n_parts; jb += JB) {
            const int nj = n_parts - jb < JB ? n_parts - jb : JB;
            __syncwarp();
            if (few) {   // (jb = 0, nj = n_parts)
#pragma unroll
                for (int u = 0; u < NPR; ++u)
                    if (u < nj)
                        *wslot(u, lane) = (lse_all == -INFINITY || lv[u] == -INFINITY)
                                              ? 0.f : fast_exp2((lv[u] - lse_all) * 1.4426950408889634f);
            } else {
                for (int j = 0; j < nj; ++j) {
                    const float lj = __ldcg(p.ws_lse + part_row(jb + j, hl));
                    *wslot(j, lane) = (lse_all == -INFINITY || lj == -INFINITY)
                                          ? 0.f : fast_exp2((lj - lse_all) * 1.4426950408889634f);
                }
            }
            __syncwarp();
#pragma unroll 1
            for (int cc = 0; cc < 4; ++cc) {
                float4 acc[8];
                if (jb == 0) {
#pragma unroll
                    for (int i = 0; i < 8; ++i) acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
                } else {   // more than 32 parts: continue from what the earlier parts stored
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        acc[i] = __ldcg(reinterpret_cast<const float4 *>(
                            p.out + ((size_t)b * p.H + (head0 + 4 * i + (lane >> 3) < p.H ? head0 + 4 * i + (lane >> 3) : 0)) * 512 +
                            col0 + 32 * cc + 4 * (lane & 7)));
                }
#pragma unroll 1
                for (int j = 0; j < nj; j += 2) {
                    const bool two = j + 1 < nj;
                    float4 x0[8], x1[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int rr = 4 * i + (lane >> 3);
                        const size_t off = (size_t)col0 + 32 * cc + 4 * (lane & 7);
                        x0[i] = __ldcg(reinterpret_cast<const float4 *>(p.ws_o + part_row(jb + j, head0 + rr) * 512 + off));
                        x1[i] = two ? __ldcg(reinterpret_cast<const float4 *>(p.ws_o + part_row(jb + j + 1, head0 + rr) * 512 + off))
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
                    }
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int rr = 4 * i + (lane >> 3);
                        const float w0 = *wslot(j, rr);
                        const float w1 = two ? *wslot(j + 1, rr) : 0.f;
                        acc[i].x = fmaf(w1, x1[i].x, fmaf(w0, x0[i].x, acc[i].x));
                        acc[i].y = fmaf(w1, x1[i].y, fmaf(w0, x0[i].y, acc[i].y));
                        acc[i].z = fmaf(w1, x1[i].z, fmaf(w0, x0[i].z, acc[i].z));
                        acc[i].w = fmaf(w1, x1[i].w, fmaf(w0, x0[i].w, acc[i].w));
                    }
                }
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int h_r = head0 + 4 * i + (lane >> 3);
                    if (h_r < p.H)
                        *reinterpret_cast<float4 *>(p.out + ((size_t)b * p.H + h_r) * 512 + col0 + 32 * cc +
                                                    4 * (lane & 7)) = acc[i];
                }
            }
            if (jb + JB < n_parts) __threadfence_block();   // this warp reads its stores back
        }
        if (part == 0 && hl < p.H) p.lse[(size_t)b * p.H + hl] = lse_all;
    };

    // Merge of a sequence cut in two, by the warp that arrived last, after its worker's
    // last piece (its block of O is still in tensor memory, and `stage`, 16 KB of shared
    // memory, is idle): only the other part's block is read, with its log-sum-exp, in one
    // round trip -- a copy instruction moves one row of the block, stored in `stage` with
    // row rr's 16-byte unit u at unit u ^ rr, so that a lane then reads and rewrites its
    // own row at the 16-byte minimum of bank conflicts -- and this warp's own block comes
    // from tensor memory again (inv normalises it, lse_own is its log-sum-exp).  The
    // merged rows go out one row per store instruction.
    auto merge_pair_own = [&](int b, long long ustart, uint8_t *stage, float inv, float lse_own) {
        const long long c_first = ustart / c.W;
        const long long cw = c.worker == c_first ? c_first + 1 : c_first;   // the other part's worker
        const int slot = (ustart <= cw * c.W) ? 0 : 1;
        const size_t row0 = ((size_t)cw * 2 + slot) * HR + head0;
        const float *src = p.ws_o + row0 * 512 + col0 + 4 * lane;
#pragma unroll
        for (int rr = 0; rr < 32; ++rr) cp_async16(stage + rr * 512 + ((lane ^ rr) << 4), src + (size_t)rr * 512);
        const float lse_oth = __ldcg(p.ws_lse + row0 + lane);
        const float M = fmaxf(lse_own, lse_oth);
        float lse_all = -INFINITY, w_own = 0.f, w_oth = 0.f;
        if (M != -INFINITY) {
            const float S = (lse_own == -INFINITY ? 0.f : fast_exp2((lse_own - M) * 1.4426950408889634f)) +
                            (lse_oth == -INFINITY ? 0.f : fast_exp2((lse_oth - M) * 1.4426950408889634f));
            lse_all = M + __logf(S);
            w_own = lse_own == -INFINITY ? 0.f : fast_exp2((lse_own - lse_all) * 1.4426950408889634f);
            w_oth = lse_oth == -INFINITY ? 0.f : fast_exp2((lse_oth - lse_all) * 1.4426950408889634f);
        }
        const float wi = w_own * inv;
        cp_async_wait_all();
        __syncwarp();   // every lane's copies, before any lane reads its row
        tc_fence_after();
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
            uint32_t ov[32];
            tmem_ld32(c.tmem + lane_base + TM_O + 128 * cg + 32 * cc, ov);
            tmem_wait_ld();
#pragma unroll
            for (int k4 = 0; k4 < 8; ++k4) {
                float4 *sx = reinterpret_cast<float4 *>(stage + lane * 512 + (((8 * cc + k4) ^ lane) << 4));
                float4 x = *sx;
                x.x = fmaf(w_oth, x.x, wi * __uint_as_float(ov[4 * k4]));
                x.y = fmaf(w_oth, x.y, wi * __uint_as_float(ov[4 * k4 + 1]));
                x.z = fmaf(w_oth, x.z, wi * __uint_as_float(ov[4 * k4 + 2]));
                x.w = fmaf(w_oth, x.w, wi * __uint_as_float(ov[4 * k4 + 3]));
                *sx = x;
            }
        }
        __syncwarp();
        float *dst = p.out + ((size_t)b * p.H + head0) * 512 + col0 + 4 * lane;
#pragma unroll 4
        for (int rr = 0; rr < 32; ++rr)
            if (head0 + rr < p.H)
                *reinterpret_cast<float4 *>(dst + (size_t)rr * 512) =
                    *reinterpret_cast<const float4 *>(stage + rr * 512 + ((lane ^ rr) << 4));
        if (part == 0 && head0 + lane < p.H) p.lse[(size_t)b * p.H + head0 + lane] = lse_all;
    };

    // Empty sequences (no tile, no worker): out 0, lse -inf, spread over the workers.
    for (int b = c.worker; b < p.B; b += p.workers) {
        if (c.s_prefix[b + 1] != c.s_prefix[b]) continue;
#pragma unroll 1
        for (int i = 0; i < 32; ++i) {
            const int rr = (i >> 2) * 4 + (lane >> 3), cc = i & 3;
            const int h_r = head0 + rr;
            if (h_r < p.H)
                *reinterpret_cast<float4 *>(p.out + ((size_t)b * p.H + h_r) * 512 + col0 + 32 * cc + 4 * (lane & 7)) =
                    make_float4(0.f, 0.f, 0.f, 0.f);
        }
        if (part == 0 && realq) p.lse[(size_t)b * p.H + head] = -INFINITY;
    }

    int k = 0, pi = 0;
    for (long long pos = c.p0; pos < c.p1; ++pi) {
        const Piece pc = piece_at(c.s_prefix, p.B, 1, pos, c.p1, c.p0);
        pos = pc.ustart + pc.lt1;
        const int len = clamp_len(__ldg(p.seq_lens + pc.b), p.T_max);
        const int nt = pc.lt1 - pc.lt0;
        if (pi == 0) {
            if constexpr (KV8) {
                float mxl, mxr;
                q8_load(pc.b, mxl, mxr);
                if (!q8_store(mxl, mxr)) return;
            } else {
                uint32_t v0[32], v1[32];
                load_q(pc.b, v0, v1);
                store_q(v0, v1);
            }
        }
        // the next piece's sequence (-1: none); its query rows are fetched into L2 during
        // this piece's last tile
        const int next_b = pos < c.p1 ? piece_at(c.s_prefix, p.B, 1, pos, c.p1, c.p0).b : -1;
        float m_ref = -INFINITY;      // running max (log2 units), shared by the four parts of the head
        float l = 0.f;                // row sum of this thread's weights, relative to m_ref
        for (int t = 0; t < nt; ++t) {
            const int kt = k + t;
            const int sb = kt & 1;
            if (t == nt - 1 && next_b >= 0 && realq) {   // the next query into L2
                if constexpr (KV8) {
                    prefetch_l2(q8_src(next_b, 0));
                    prefetch_l2(q8_src(next_b, 8));
                    prefetch_l2(q8_src(next_b, 16));
                } else {
                    const uint4 *qn = q_row(next_b);
                    prefetch_l2(qn);
                    prefetch_l2(qn + 8);
                }
            }
            // first valid column of this thread's 32 (masked: rows of the half below lo)
            const int lo = half_source(p, pc.b, len, pc.lt0 + t, half).lo - 32 * cg;
            // ---- this thread's 32 scores
            if (!wait_local(&bars->sready[sb], (uint32_t)(kt >> 1) & 1u, FLAG_MMA_WAIT, c)) return;
            tc_fence_after();
            float sv[32];
            {
                uint32_t a[32];
                tmem_ld32(c.tmem + lane_base + TM_S + 64 * sb + 32 * cg, a);
                if constexpr (KV8) {   // latent and RoPE parts, each with its scale: log2 units
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j) sv[j] = __uint_as_float(a[j]) * sl2_lat;
                    tmem_ld32(c.tmem + lane_base + e4::TM_SR + 64 * sb + 32 * cg, a);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j) sv[j] = fmaf(__uint_as_float(a[j]), sl2_rope, sv[j]);
                } else {
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j) sv[j] = __uint_as_float(a[j]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(sb ? sfree1 : sfree0);
            // ---- partial tile maximum (log2 units; masked columns excluded)
            if (lo > 0) {
#pragma unroll
                for (int i = 0; i < 32; ++i) sv[i] = i >= lo ? sv[i] : (sl2 >= 0.f ? -INFINITY : INFINITY);
            }
            float mx;
            {
                float m8[8];
#pragma unroll
                for (int g = 0; g < 8; ++g) m8[g] = sv[g];
                if (sl2 >= 0.f) {
#pragma unroll
                    for (int i = 8; i < 32; ++i) m8[i & 7] = fmaxf(m8[i & 7], sv[i]);
                } else {   // a negative scale turns the smallest raw score into the largest
#pragma unroll
                    for (int i = 8; i < 32; ++i) m8[i & 7] = fminf(m8[i & 7], sv[i]);
                }
                mx = fmaxf(fmaxf(fmaxf(m8[0] * sl2, m8[1] * sl2), fmaxf(m8[2] * sl2, m8[3] * sl2)),
                           fmaxf(fmaxf(m8[4] * sl2, m8[5] * sl2), fmaxf(m8[6] * sl2, m8[7] * sl2)));
                if (mx != mx) mx = -INFINITY;   // every column masked: (+-inf) * 0 is not a maximum
            }
            // ---- the head's tile maximum over its four parts, then the running max
            mx_buf[(sb * 4 + part) * HC + hh] = mx;
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->mxbar[sb]);
            if (!wait_local(&bars->mxbar[sb], (uint32_t)(kt >> 1) & 1u, FLAG_FULL_WAIT, c)) return;
            const float *mxs = mx_buf + sb * 4 * HC + hh;
            const float M = fmaxf(fmaxf(mxs[0], mxs[HC]), fmaxf(mxs[2 * HC], mxs[3 * HC]));
            const float m_new = (t == 0 || M > m_ref + RESCALE) ? M : m_ref;
            const bool rescale = t > 0 && m_new != m_ref;
            const float alpha = rescale ? fast_exp2(m_ref - m_new) : 1.f;
            m_ref = m_new;
            // ---- weights 2^(s * scale - m): a bf16 high part and a bf16 remainder (E4M3 cache:
            //      2^6 times that, as three E4M3 parts, four codes per word)
            uint32_t whi[16], wlo[16], wmid[8];
            float ls4[4] = {0.f, 0.f, 0.f, 0.f};
            const float m_off = KV8 ? e4::P_LOG2 - m_new : -m_new;
            uint32_t ph = 0, pm = 0, pl = 0;   // E4M3: the codes of the previous (even) pair
            auto put = [&](int j, float a, float b) {
                if constexpr (KV8) {
                    uint16_t h2, m2, l2;
                    split3_e4m3x2(a, b, h2, m2, l2);
                    if (j & 1) {
                        whi[j >> 1] = ph | ((uint32_t)h2 << 16);
                        wmid[j >> 1] = pm | ((uint32_t)m2 << 16);
                        wlo[j >> 1] = pl | ((uint32_t)l2 << 16);
                    } else {
                        ph = h2;
                        pm = m2;
                        pl = l2;
                    }
                } else {
                    split_bf16x2(a, b, whi[j], wlo[j]);
                }
            };
            if (lo <= 0) {
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const float a = fast_exp2(fmaf(sv[2 * j], sl2, m_off));
                    const float b = fast_exp2(fmaf(sv[2 * j + 1], sl2, m_off));
                    ls4[j & 3] += a + b;
                    put(j, a, b);
                }
            } else {   // masked columns get weight 0 (whatever the scale)
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const float a = 2 * j >= lo ? fast_exp2(fmaf(sv[2 * j], sl2, m_off)) : 0.f;
                    const float b = 2 * j + 1 >= lo ? fast_exp2(fmaf(sv[2 * j + 1], sl2, m_off)) : 0.f;
                    ls4[j & 3] += a + b;
                    put(j, a, b);
                }
            }
            l = l * alpha + ((ls4[0] + ls4[1]) + (ls4[2] + ls4[3]));
            // ---- the weights into shared memory.  The half-h weights of tile kt - 1 are free
            //      once the half-h step of its value product is done; a rescale of O needs
            //      the whole product done, and must be finished before tile kt's first step,
            //      which is why every warp arrives on the first step's barrier.
            const int kp = kt - 1;
            const bool any_rescale = __any_sync(0xffffffffu, rescale);   // only when t > 0, so kp >= 0
            auto store_p = [&]() {
                if constexpr (KV8) {
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int slot = ((4 * half + 2 * cg + u) ^ (hh & 7)) * 16;
                        *reinterpret_cast<uint4 *>(row8_hi + slot) =
                            make_uint4(whi[4 * u], whi[4 * u + 1], whi[4 * u + 2], whi[4 * u + 3]);
                        *reinterpret_cast<uint4 *>(row8_hi + e4::PPART + slot) =
                            make_uint4(wmid[4 * u], wmid[4 * u + 1], wmid[4 * u + 2], wmid[4 * u + 3]);
                        *reinterpret_cast<uint4 *>(row8_hi + 2 * e4::PPART + slot) =
                            make_uint4(wlo[4 * u], wlo[4 * u + 1], wlo[4 * u + 2], wlo[4 * u + 3]);
                    }
                } else {
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int slot = ((4 * cg + u) ^ (hh & 7)) * 16;
                        *reinterpret_cast<uint4 *>(row_hi + slot) =
                            make_uint4(whi[4 * u], whi[4 * u + 1], whi[4 * u + 2], whi[4 * u + 3]);
                        *reinterpret_cast<uint4 *>(row_lo + slot) =
                            make_uint4(wlo[4 * u], wlo[4 * u + 1], wlo[4 * u + 2], wlo[4 * u + 3]);
                    }
                }
                fence_proxy_async_smem();
            };
            if (half == 0) {
                if (kt >= 1 && !wait_local(&bars->odone[0][kp & 1], (uint32_t)(kp >> 1) & 1u, FLAG_MMA_WAIT, c))
                    return;
                if (any_rescale) {
                    if (!wait_local(&bars->odone[1][kp & 1], (uint32_t)(kp >> 1) & 1u, FLAG_MMA_WAIT, c)) return;
                    tc_fence_after();
                    rescale_o(alpha);
                }
                store_p();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_remote(sb ? pready_own1 : pready_own0);
            } else {
                const bool need_prev = kt >= 1;
                if (any_rescale) {
                    if (!wait_local(&bars->odone[1][kp & 1], (uint32_t)(kp >> 1) & 1u, FLAG_MMA_WAIT, c)) return;
                    tc_fence_after();
                    rescale_o(alpha);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_remote(sb ? pready_first1 : pready_first0);   // O of these lanes is settled
                if (need_prev && !any_rescale &&
                    !wait_local(&bars->odone[1][kp & 1], (uint32_t)(kp >> 1) & 1u, FLAG_MMA_WAIT, c))
                    return;
                store_p();
                __syncwarp();
                if (lane == 0) mbar_arrive_remote(sb ? pready_own1 : pready_own0);
            }
        }
        // ---- end of the piece.  First the next piece's query, so that its score products
        //      can start while this epilogue runs (this piece's have read Q: qempty).
        if (next_b >= 0) {
            if constexpr (KV8) {
                float mxl, mxr;
                if (!wait_local(&bars->qempty, (uint32_t)pi & 1u, FLAG_MMA_WAIT, c)) return;
                q8_load(next_b, mxl, mxr);
                if (!q8_store(mxl, mxr)) return;
            } else {
                uint32_t v0[32], v1[32];
                load_q(next_b, v0, v1);
                if (!wait_local(&bars->qempty, (uint32_t)pi & 1u, FLAG_MMA_WAIT, c)) return;
                store_q(v0, v1);
            }
        }
        // ---- the head's row sum (four parts), normalise, write this warp's block of O:
        //      rows 32 (q & 1) + [0, 32) of this CTA's heads, columns col0 + [0, 128)
        const int klast = k + nt - 1;
        k += nt;
        lx_buf[part * HC + hh] = l;
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->lxbar);
        if (!wait_local(&bars->lxbar, (uint32_t)pi & 1u, FLAG_FULL_WAIT, c)) return;
        const float ltot = (lx_buf[hh] + lx_buf[HC + hh]) + (lx_buf[2 * HC + hh] + lx_buf[3 * HC + hh]);
        // (E4M3 cache: the weights and their sum carry 2^6; a value code counts latent_scale)
        const float lse_v =
            ltot > 0.f ? (m_ref + __log2f(ltot) - (KV8 ? e4::P_LOG2 : 0.f)) * 0.69314718055994531f : -INFINITY;
        const float inv = ltot > 0.f ? (KV8 ? p.latent_scale : 1.f) / ltot : 0.f;
        if (!wait_local(&bars->odone[1][klast & 1], (uint32_t)(klast >> 1) & 1u, FLAG_MMA_WAIT, c)) return;
        tc_fence_after();
        float *dst = pc.whole ? p.out + (size_t)pc.b * p.H * 512
                              : p.ws_o + ((size_t)c.worker * 2 + pc.slot) * HR * 512;
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
            uint32_t ov[32];
            tmem_ld32(c.tmem + lane_base + TM_O + 128 * cg + 32 * cc, ov);
            tmem_wait_ld();
            // transpose through this warp's own bytes of the weights buffer (free: every
            // value product of the piece is done), SU * 4 columns at a time, so that SU
            // lanes store one row's SU * 16 contiguous bytes
#pragma unroll
            for (int ps = 0; ps < 8 / SU; ++ps) {
#pragma unroll
                for (int u = 0; u < SU; ++u) {
                    const int o = 4 * SU * ps + 4 * u;
                    *reinterpret_cast<float4 *>(scratch_unit(lane, u)) =
                        make_float4(__uint_as_float(ov[o]) * inv, __uint_as_float(ov[o + 1]) * inv,
                                    __uint_as_float(ov[o + 2]) * inv, __uint_as_float(ov[o + 3]) * inv);
                }
                __syncwarp();
#pragma unroll
                for (int i = 0; i < SU; ++i) {
                    const int rr = (32 / SU) * i + lane / SU, u = lane % SU;
                    const int h_r = head0 + rr;
                    const float4 x = *reinterpret_cast<const float4 *>(scratch_unit(rr, u));
                    if (h_r < p.H)
                        *reinterpret_cast<float4 *>(dst + (size_t)h_r * 512 + col0 + 32 * cc + 4 * SU * ps + 4 * u) = x;
                }
                __syncwarp();
            }
        }
        // a partial's log-sum-exp is written by every warp for its own rows (the four parts
        // of a head hold the same value), so that this warp's arrival below orders it
        // before the merging warp, the same warp of another worker, reads it
        if (realq && (part == 0 || !pc.whole)) {
            if (pc.whole)
                p.lse[(size_t)pc.b * p.H + head] = lse_v;
            else
                p.ws_lse[((size_t)c.worker * 2 + pc.slot) * HR + head] = lse_v;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(ofree0);
        // ---- a cut sequence: the last of its workers to finish this block merges the
        //      block's partials (no waiting on the others)
        if (!pc.whole) {
            const long long ustart = c.s_prefix[pc.b];
            const int n_parts = (int)((ustart + pc.n_tiles - 1) / c.W - ustart / c.W) + 1;
            __threadfence();   // this warp's partial rows, before the arrival
            __syncwarp();
            bool last = false;
            if (lane == 0)
                last = merge_arrive_last(&g_mla_merge_count[((size_t)pc.b * 2 + c.r) * NSOFT + (warp - 4)], p.epoch,
                                         n_parts);
            last = __shfl_sync(0xffffffffu, last, 0);
            if (last) {
                __threadfence();   // the other workers' partials, after their arrivals
                // After a worker's last piece its key ring and value slots are idle (every
                // load of the piece has landed and every product that reads them is done:
                // odone of the last tile): 16 KB of them per softmax warp stage the merge.
                uint8_t *stage = nullptr;
                if (next_b < 0) {
                    const int w = warp - 4;
                    if constexpr (KV8)
                        stage = w < 5 ? c.smem + e4::OFF_Q + w * 16384 : c.smem + e4::OFF_SR + (w - 5) * 16384;
                    else
                        stage = c.smem + OFF_SR + w * 16384;
                }
                if (n_parts == 2 && stage != nullptr)
                    merge_pair_own(pc.b, ustart, stage, inv, lse_v);
                else
                    merge_block(pc.b, ustart, n_parts);
            }
        }
    }
}
}  // namespace mla

template <bool KV8>
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
        for (int g = 0; g < NKS; ++g) mbar_init(&bars->kfull[g], 1);
        for (int g = 0; g < NKS - 1; ++g) mbar_init(&bars->kempty[g], 1);
        mbar_init(&bars->qxbar, NSOFT);
        for (int j = 0; j < NVS; ++j) mbar_init(&bars->vfull[j], 1);
        mbar_init(&bars->qfull, 1);
        mbar_init(&bars->qtm, 2 * NSOFT);    // one arrival per softmax warp of either CTA
        mbar_init(&bars->qempty, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars->sready[i], 1);
            mbar_init(&bars->sfree[i], 2 * NSOFT);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars->odone[0][i], 1);
            mbar_init(&bars->odone[1][i], 1);
            mbar_init(&bars->pready[0][i], 2 * NSOFT);   // every softmax warp of either CTA
            mbar_init(&bars->pready[1][i], NSOFT);       // the half-1 warps of either CTA
        }
        mbar_init(&bars->ofree, 2 * NSOFT);
        mbar_init(&bars->mxbar[0], NSOFT);
        mbar_init(&bars->mxbar[1], NSOFT);
        mbar_init(&bars->lxbar, NSOFT);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(tmem_ptr), TM_COLS);
        tmem_relinquish_pair();
    }
    if (warp == 2) build_tile_prefix(p.seq_lens, p.B, p.T_max, TILE, s_prefix, lane);
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&maps.latk);
        prefetch_tensormap(&maps.latv);
        prefetch_tensormap(&maps.rope);
        if (!KV8) prefetch_tensormap(&maps.latk2);
        if (!KV8) {
            prefetch_tensormap(&maps.qlatc);
            prefetch_tensormap(&maps.qrope);
        }
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
    // Tiles per worker.  When every sequence has the same number of tiles n, W may be
    // rounded up so that worker boundaries fall on sequence or equal-part boundaries (each
    // sequence in k equal parts, or whole sequences): a boundary inside a worker's range
    // costs a partial result, its merge and a pipeline drain, more than the few tiles the
    // coarser split adds.
    const long long W = split_tiles(total, p.workers, p.min_tiles, uniform_tile_count(s_prefix, p.B));
    c.W = W;
    c.p0 = (long long)c.worker * W;
    c.p1 = (c.p0 + W < total) ? c.p0 + W : total;

    if (c.p0 < total) {
        if (warp == 0 && lane == 0) key_producer<KV8>(p, maps, c);
        if (warp == 2 && lane == 0) value_producer<KV8>(p, maps, c);
        if (warp == 1 && lane == 0 && c.r == 0) score_issuer<KV8>(p, c);
        if (warp == 3 && lane == 0 && c.r == 0) value_issuer<KV8>(p, c);
    }
    if (warp >= 4) softmax_warps<KV8>(p, c, warp, lane);   // also the empty sequences

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
