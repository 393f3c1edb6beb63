// schedule.cuh -- how the decode work is cut into pieces for the workers.
//
// The work is a stream of KV tiles.  A "unit" is everything one worker would need to
// finish one output block: for GQA one (sequence, KV head, head block), for MLA one
// sequence.  Unit u of sequence b holds ceil(len_b / TILE) tiles.  Units are laid end
// to end (sequence-major), and worker c takes the contiguous tile range
// [c*W, min((c+1)*W, total)), W = max(ceil(total / workers), min_tiles).  A unit that a
// worker covers completely is finished by that worker (final out/lse); a unit cut by
// a worker boundary leaves one partial result per worker that touched it, and the
// combine kernel merges those by log-sum-exp.
//
// Because seq_lens lives on the device, every CTA computes the same decomposition from
// it (a prefix sum over the batch in shared memory); CTA 0 also publishes it (W, total,
// the prefix) in the workspace for the combine kernel.  Tiles never straddle two
// units, and a unit's last tile is loaded shifted back so that it ends at len_b: no
// load ever touches a cache position >= len_b (a negative start row is zero-filled by
// the TMA unit).
#pragma once
#include <stdint.h>

namespace kvattn {

struct Piece {
    int b;              // sequence
    int i;              // unit index within the sequence (GQA: kv_head * n_hb + head block)
    int n_tiles;        // tiles of this unit
    int lt0, lt1;       // tiles [lt0, lt1) of the unit belong to this piece
    long long ustart;   // global tile index of the unit's first tile
    bool whole;         // the piece is the entire unit
    int slot;           // workspace slot of a partial piece: 0 or 1
};

__device__ __forceinline__ int tiles_of(int len, int tile) { return (len + tile - 1) / tile; }

__device__ __forceinline__ int clamp_len(int len, int T_max) {
    return len < 0 ? 0 : (len > T_max ? T_max : len);
}

// First cached position any query of a sequence of length len can see: 0, unless the
// L newest tokens attend through a sliding window of `window` tokens (window > 0), in
// which case the oldest of them, at position len - L, sees back to len - L + 1 - window.
// The tiles of a sequence cover [active_start, len).
__device__ __forceinline__ int active_start(int len, int q_len, int window) {
    if (window <= 0) return 0;
    const int s = len - q_len + 1 - window;
    return s > 0 ? s : 0;
}

// Warp 0 of the block fills s_prefix[0..B] with the exclusive prefix of tiles per
// sequence (tiles of its active range).  The caller synchronises the block afterwards.
__device__ __forceinline__ void build_tile_prefix(const int32_t *seq_lens, int B, int T_max,
                                                  int tile, int *s_prefix, int lane, int q_len = 1,
                                                  int window = 0) {
    int running = 0;
    if (lane == 0) s_prefix[0] = 0;
    for (int base = 0; base < B; base += 32) {
        const int idx = base + lane;
        int v = 0;
        if (idx < B) {
            const int len = clamp_len(__ldg(seq_lens + idx), T_max);
            v = tiles_of(len - active_start(len, q_len, window), tile);
        }
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, v, off);
            if (lane >= off) v += n;
        }
        if (idx < B) s_prefix[idx + 1] = running + v;
        running += __shfl_sync(0xffffffffu, v, 31);
    }
}

// Largest b in [0, B) with prefix[b] * U <= p  (p < total): the sequence holding tile p.
__device__ __forceinline__ int find_seq(const int *s_prefix, int B, int U, long long p) {
    int lo = 0, hi = B - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if ((long long)s_prefix[mid] * U <= p) lo = mid; else hi = mid - 1;
    }
    return lo;
}

__device__ __forceinline__ Piece piece_at(const int *s_prefix, int B, int U, long long p,
                                          long long p_end, long long worker_start) {
    Piece pc;
    pc.b = find_seq(s_prefix, B, U, p);
    pc.n_tiles = s_prefix[pc.b + 1] - s_prefix[pc.b];
    const long long base = (long long)s_prefix[pc.b] * U;
    pc.i = (int)((p - base) / pc.n_tiles);
    pc.ustart = base + (long long)pc.i * pc.n_tiles;
    pc.lt0 = (int)(p - pc.ustart);
    const long long rem = p_end - pc.ustart;
    pc.lt1 = rem < pc.n_tiles ? (int)rem : pc.n_tiles;
    pc.whole = (pc.lt0 == 0 && pc.lt1 == pc.n_tiles);
    pc.slot = (pc.ustart <= worker_start) ? 0 : 1;
    return pc;
}

// Where the TMA finds tile lt of sequence b (the tile starting at position start +
// lt * tile; start is the active range's first position, a page boundary or 0 for a
// paged cache).  The cache is a sequence of pages of
// page_size rows (a contiguous cache is one page per sequence, page_size = its capacity,
// page = b); a tile never straddles two pages (page_size is a multiple of the tile).
// The last tile of a sequence is loaded shifted back inside its page so that it ends at
// the sequence's last row: its first rows then repeat rows of the previous tile, or lie
// before the page (a negative row, zero-filled by the TMA unit), and the consumers mask
// them (tile rows below TILE - valid).  No load touches a row at or past the length.
struct TileSrc {
    int y;      // first row inside the page
    int page;   // physical page
};
__device__ __forceinline__ TileSrc tile_source(const int32_t *block_table, int max_pages, int page_size,
                                               int b, int lt, int tile, int len, int start = 0) {
    const int tok0 = start + lt * tile;
    const int lp = tok0 / page_size;
    const int valid = min(tile, len - tok0);
    TileSrc s;
    s.y = tok0 - lp * page_size + valid - tile;
    s.page = block_table != nullptr ? __ldg(block_table + (size_t)b * max_pages + lp) : b;
    return s;
}

// Tiles per worker, identical on every CTA and in the combine kernel.
__device__ __forceinline__ long long tiles_per_worker(long long total, int workers, int min_tiles) {
    long long w = (total + workers - 1) / workers;
    if (w < min_tiles) w = min_tiles;
    if (w < 1) w = 1;
    return w;
}

// When every sequence has the same number of tiles n (per unit), the share w0 may be
// rounded so that worker boundaries fall on unit boundaries or cut units into equal
// parts (a multiple or a divisor of n), if that adds at most max(2, w0 / 4) tiles: a
// boundary inside a worker's range costs a partial result, its merge and a pipeline
// restart, more than the few tiles the coarser split adds.
__device__ __forceinline__ long long uniform_tiles_per_worker(long long w0, int n) {
    long long w = n;
    if (w0 >= n) {
        w = ((w0 + n - 1) / n) * n;
    } else {
        for (int k = (int)(n / w0); k > 1; --k)
            if (n % k == 0) {
                w = n / k;
                break;
            }
    }
    const long long slack = w0 / 4 > 2 ? w0 / 4 : 2;
    return w - w0 <= slack ? w : w0;
}
// The MLA kernel's work split: tiles_per_worker, rounded as above when n_uniform (the
// common tile count of every sequence) is > 0.  (The GQA kernels keep tiles_per_worker:
// measured, the rounding cost them more than the cuts it removed.)
__device__ __forceinline__ long long split_tiles(long long total, int workers, int min_tiles, int n_uniform) {
    const long long w = tiles_per_worker(total, workers, min_tiles);
    return n_uniform > 0 ? uniform_tiles_per_worker(w, n_uniform) : w;
}
// The common tile count of every sequence from a tile prefix (0 if they differ or are
// empty); block-wide (every thread of the block must call it).
__device__ __forceinline__ int uniform_tile_count(const int *s_prefix, int B) {
    const int n0 = s_prefix[1] - s_prefix[0];
    int same = 1;
    for (int i = threadIdx.x; i < B; i += blockDim.x) same &= (s_prefix[i + 1] - s_prefix[i]) == n0;
    same = __syncthreads_and(same);
    return same && n0 > 0 ? n0 : 0;
}

// Unit parts (the tcgen05 GQA kernel and its combine): when every unit has the same
// number of tiles n and there are at least as many workers as units, unit u is cut into
// k consecutive parts of at most ceil(n / k) tiles (k = workers / units, parts of at least
// min_tiles), worker u * k + i taking part i -- so no worker spans two units (a worker
// that does pays a second query load, epilogue and pipeline restart and finishes last).
// Returns the tiles per part and k, or 0 where it does not apply.
__device__ __forceinline__ long long unit_part_tiles(int n, long long units, int workers, int min_tiles, int *k_out) {
    if (n <= 0 || units <= 0 || units > workers) return 0;
    long long k = workers / units;
    const long long kmax = (n + (min_tiles > 0 ? min_tiles : 1) - 1) / (min_tiles > 0 ? min_tiles : 1);
    if (k > kmax) k = kmax;
    if (k < 1) k = 1;
    *k_out = (int)k;
    return (n + k - 1) / k;
}

// Layout of the published decomposition at the start of the workspace.
struct MetaView {
    long long *w_total;  // [0] = W, [1] = total
    int *prefix;         // [B + 1]
};
__device__ __forceinline__ MetaView meta_view(void *ws) {
    MetaView m;
    m.w_total = reinterpret_cast<long long *>(ws);
    m.prefix = reinterpret_cast<int *>(reinterpret_cast<long long *>(ws) + 2);
    return m;
}

}  // namespace kvattn
