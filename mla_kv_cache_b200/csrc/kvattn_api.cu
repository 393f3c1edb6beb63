// kvattn_api.cu -- the C ABI of kvattn (include/kvattn.h): argument checks, the work
// plan, the per-device workspace, TMA descriptors and kernel launches.
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdio>
#include <cstring>
#include <atomic>
#include <mutex>

#include "../../include/kvattn.h"
#include "combine.cuh"
#include "common.cuh"
#include "gqa_decode.cuh"
#include "gqa_tc_decode.cuh"
#include "mla_decode.cuh"
#include "rope_append.cuh"

using namespace kvattn;

namespace {

constexpr int kMaxDevices = 64;
constexpr int kMaxBatch = 4096;

thread_local char t_detail[256] = "";

int fail_cuda(cudaError_t e, const char *where) {
    snprintf(t_detail, sizeof(t_detail), "%s: %s", where, cudaGetErrorString(e));
    return KVATTN_ERR_CUDA;
}

struct DeviceState {
    bool init = false;
    int id = 0;
    int sms = 0;
    int max_smem_optin = 0;
    void *ws = nullptr;
    size_t ws_bytes = 0;
    void *aux = nullptr;          // the virtual batch of a multi-token call (lengths, block table)
    size_t aux_bytes = 0;
    struct Func {
        const void *kern;
        int smem;
    } funcs[64] = {};
    int n_funcs = 0;
    int mla_clusters = 0;   // co-resident MLA CTA pairs (0: not queried yet)
    std::atomic<unsigned int> mla_calls{0};   // MLA decode calls issued (tags the merge counters)
};
DeviceState g_dev[kMaxDevices];
std::mutex g_mutex;
int g_force_workers = 0;
int g_force_min_tiles = 0;
int g_gqa_kernel = 0;   // 0: heuristic, 1: warp-level MMA kernel, 2: tcgen05 kernel

int device_state(DeviceState **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail_cuda(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) {
        snprintf(t_detail, sizeof(t_detail), "device ordinal %d out of range", dev);
        return KVATTN_ERR_UNSUPPORTED;
    }
    DeviceState &s = g_dev[dev];
    if (!s.init) {
        s.id = dev;
        e = cudaDeviceGetAttribute(&s.sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return fail_cuda(e, "cudaDeviceGetAttribute(SMs)");
        e = cudaDeviceGetAttribute(&s.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        if (e != cudaSuccess) return fail_cuda(e, "cudaDeviceGetAttribute(smem)");
        s.init = true;
    }
    *out = &s;
    return KVATTN_OK;
}

// Grows the calling device's workspace to at least `bytes` (caller holds g_mutex).
int ensure_workspace(DeviceState *s, size_t bytes, void **ws) {
    if (s->ws_bytes < bytes) {
        if (s->ws) {
            cudaError_t e = cudaDeviceSynchronize();
            if (e != cudaSuccess) return fail_cuda(e, "cudaDeviceSynchronize (workspace grow)");
            cudaFree(s->ws);
            s->ws = nullptr;
            s->ws_bytes = 0;
        }
        size_t want = bytes < (1u << 20) ? (1u << 20) : bytes;
        cudaError_t e = cudaMalloc(&s->ws, want);
        if (e != cudaSuccess) {
            cudaGetLastError();
            snprintf(t_detail, sizeof(t_detail), "cudaMalloc(%zu): %s", want, cudaGetErrorString(e));
            return KVATTN_ERR_NO_MEMORY;
        }
        s->ws_bytes = want;
    }
    *ws = s->ws;
    return KVATTN_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        cudaDriverEntryPointQueryResult q;
        void *p = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// Recently encoded tensor maps of this host thread (a decode loop calls the library
// with the same cache tensors every step; encoding costs microseconds of host time).
struct MapKey {
    const void *base;
    uint64_t d0, d1, d2;
    uint32_t b0, b1;
    int swz;
    bool operator==(const MapKey &o) const {
        return base == o.base && d0 == o.d0 && d1 == o.d1 && d2 == o.d2 && b0 == o.b0 && b1 == o.b1 &&
               swz == o.swz;
    }
};
struct MapEntry {
    MapKey key;
    CUtensorMap map;
    bool valid;
};
constexpr int kMapCache = 16;
thread_local MapEntry t_maps[kMapCache];
thread_local int t_map_next = 0;

int encode_map_3d(CUtensorMap *map, const void *base, uint64_t dim0, uint64_t dim1, uint64_t dim2,
                  uint32_t box0, uint32_t box1, CUtensorMapSwizzle swz);

// 3-D bf16 tensor [dim2][dim1][dim0] (dim0 fastest), box {box0, box1, 1}.
int make_map_3d(CUtensorMap *map, const void *base, uint64_t dim0, uint64_t dim1, uint64_t dim2,
                uint32_t box0, uint32_t box1, CUtensorMapSwizzle swz) {
    const MapKey key{base, dim0, dim1, dim2, box0, box1, (int)swz};
    for (int i = 0; i < kMapCache; ++i)
        if (t_maps[i].valid && t_maps[i].key == key) {
            *map = t_maps[i].map;
            return KVATTN_OK;
        }
    int st = encode_map_3d(map, base, dim0, dim1, dim2, box0, box1, swz);
    if (st != KVATTN_OK) return st;
    MapEntry &e = t_maps[t_map_next];
    t_map_next = (t_map_next + 1) % kMapCache;
    e.key = key;
    e.map = *map;
    e.valid = true;
    return KVATTN_OK;
}

int encode_map_3d(CUtensorMap *map, const void *base, uint64_t dim0, uint64_t dim1, uint64_t dim2,
                  uint32_t box0, uint32_t box1, CUtensorMapSwizzle swz) {
    auto fn = encode_fn();
    if (!fn) {
        snprintf(t_detail, sizeof(t_detail), "cuTensorMapEncodeTiled unavailable");
        return KVATTN_ERR_CUDA;
    }
    cuuint64_t dims[3] = {dim0, dim1, dim2};
    cuuint64_t strides[2] = {dim0 * 2, dim0 * dim1 * 2};
    cuuint32_t box[3] = {box0, box1, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        snprintf(t_detail, sizeof(t_detail), "cuTensorMapEncodeTiled failed (%d)", (int)r);
        return KVATTN_ERR_CUDA;
    }
    return KVATTN_OK;
}

// A strided view of a 16-bit tensor (rank 3..5): dims[0] contiguous, strides[i] the byte
// stride of dims[i + 1] -- not necessarily increasing, e.g. a [rows][chunks][64] view of
// rows whose chunk dimension strides 128 bytes inside a row, so that one copy moves
// several 64-column chunks of a row block.  Cached like make_map_3d.
struct ViewKey {
    const void *base;
    int rank;
    uint64_t dims[5], strides[4];
    uint32_t box[5];
    bool operator==(const ViewKey &o) const {
        if (base != o.base || rank != o.rank) return false;
        for (int i = 0; i < 5; ++i)
            if (dims[i] != o.dims[i] || box[i] != o.box[i]) return false;
        for (int i = 0; i < 4; ++i)
            if (strides[i] != o.strides[i]) return false;
        return true;
    }
};
struct ViewEntry {
    ViewKey key;
    CUtensorMap map;
    bool valid;
};
constexpr int kViewCache = 16;
thread_local ViewEntry t_views[kViewCache];
thread_local int t_view_next = 0;

int make_map_view(CUtensorMap *map, const void *base, int rank, const uint64_t *dims, const uint64_t *strides,
                  const uint32_t *box) {
    ViewKey key = {};
    key.base = base;
    key.rank = rank;
    for (int i = 0; i < rank; ++i) {
        key.dims[i] = dims[i];
        key.box[i] = box[i];
        if (i + 1 < rank) key.strides[i] = strides[i];
    }
    for (int i = 0; i < kViewCache; ++i)
        if (t_views[i].valid && t_views[i].key == key) {
            *map = t_views[i].map;
            return KVATTN_OK;
        }
    auto fn = encode_fn();
    if (!fn) {
        snprintf(t_detail, sizeof(t_detail), "cuTensorMapEncodeTiled unavailable");
        return KVATTN_ERR_CUDA;
    }
    cuuint64_t d[5], st[4];
    cuuint32_t bx[5], es[5];
    for (int i = 0; i < rank; ++i) {
        d[i] = dims[i];
        bx[i] = box[i];
        es[i] = 1;
        if (i + 1 < rank) st[i] = strides[i];
    }
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void *>(base), d, st, bx, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        snprintf(t_detail, sizeof(t_detail), "cuTensorMapEncodeTiled (%d-D view) failed (%d)", rank, (int)r);
        return KVATTN_ERR_CUDA;
    }
    ViewEntry &e = t_views[t_view_next];
    t_view_next = (t_view_next + 1) % kViewCache;
    e.key = key;
    e.map = *map;
    e.valid = true;
    return KVATTN_OK;
}

// 4-D bf16 tensor [dim3][dim2][dim1][dim0] (dim0 fastest, densely packed), box
// {box0, box1, box2, 1}.  Not cached (used once per call).
int make_map_4d(CUtensorMap *map, const void *base, uint64_t dim0, uint64_t dim1, uint64_t dim2, uint64_t dim3,
                uint32_t box0, uint32_t box1, uint32_t box2, CUtensorMapSwizzle swz) {
    auto fn = encode_fn();
    if (!fn) {
        snprintf(t_detail, sizeof(t_detail), "cuTensorMapEncodeTiled unavailable");
        return KVATTN_ERR_CUDA;
    }
    cuuint64_t dims[4] = {dim0, dim1, dim2, dim3};
    cuuint64_t strides[3] = {dim0 * 2, dim0 * dim1 * 2, dim0 * dim1 * dim2 * 2};
    cuuint32_t box[4] = {box0, box1, box2, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        snprintf(t_detail, sizeof(t_detail), "cuTensorMapEncodeTiled (4-D) failed (%d)", (int)r);
        return KVATTN_ERR_CUDA;
    }
    return KVATTN_OK;
}

// Raises a kernel's dynamic shared-memory limit once per device (the largest request
// seen so far is kept).
cudaError_t set_smem_limit(const void *kern, DeviceState *dev, int smem) {
    std::lock_guard<std::mutex> lk(g_mutex);
    for (int i = 0; i < dev->n_funcs; ++i) {
        auto &f = dev->funcs[i];
        if (f.kern == kern) {
            if (f.smem >= smem) return cudaSuccess;
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
            if (e == cudaSuccess) f.smem = smem;
            return e;
        }
    }
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e == cudaSuccess && dev->n_funcs < (int)(sizeof(dev->funcs) / sizeof(dev->funcs[0])))
        dev->funcs[dev->n_funcs++] = {kern, smem};
    return e;
}

// Kernels this library has launched from the calling thread (kvattn_kernel_launches).
thread_local unsigned long long t_launches = 0;

template <int D>
cudaError_t launch_combine_d(cudaLaunchConfig_t &cfg, const CombineParams &cp, int warps) {
    cfg.blockDim = dim3(warps * 32, 1, 1);
    cudaError_t e;
    switch (warps) {
        case 1: e = cudaLaunchKernelEx(&cfg, combine_kernel<D, 1>, cp); break;
        case 2: e = cudaLaunchKernelEx(&cfg, combine_kernel<D, 2>, cp); break;
        case 4: e = cudaLaunchKernelEx(&cfg, combine_kernel<D, 4>, cp); break;
        default: e = cudaLaunchKernelEx(&cfg, combine_kernel<D, 8>, cp); break;
    }
    if (e == cudaSuccess) ++t_launches;
    return e;
}

// Warps per combine CTA from the partials one unit is expected to have (about four
// partials per warp, so the loads of a warp overlap).
int combine_warps(long long tiles_per_unit_max, long long total_tiles_max, int workers) {
    const long long w = (total_tiles_max + workers - 1) / workers;
    const long long parts = (tiles_per_unit_max + (w > 0 ? w : 1) - 1) / (w > 0 ? w : 1) + 1;
    if (parts <= 4) return 1;
    if (parts <= 8) return 2;
    if (parts <= 16) return 4;
    return 8;
}

int launch_combine(int D, const CombineParams &cp, int units, int rows, cudaStream_t stream, int warps) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3(units, rows, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e;
    if (D == 64)
        e = launch_combine_d<64>(cfg, cp, warps);
    else if (D == 128)
        e = launch_combine_d<128>(cfg, cp, warps);
    else
        e = launch_combine_d<512>(cfg, cp, warps);
    if (e != cudaSuccess) return fail_cuda(e, "combine launch");
    return KVATTN_OK;
}

// ---------------------------------------------------------------------------------------
// Scratch of kvattn_gqa_decode_noalloc.
//
// Some callers cannot let a library call cudaMalloc: a serving engine that reserves
// almost all of the GPU's memory up front for its paged KV-cache pool (a stray
// allocation can fail or fragment that pool), and latency-critical loops where the
// implicit device synchronisation of cudaMalloc / cudaFree is unacceptable.  For them
// kvattn_gqa_decode_noalloc runs the same warp-level decode and combine kernels as
// kvattn_gqa_decode, through the same code below, but keeps the split-KV scratch (the
// published work split and the per-worker partial outputs) in this fixed array, which
// every GPU that loads the library holds until the process exits.  Its size bounds the
// plans it accepts: the built-in plan of the warp-level kernel needs the work split
// (at most 16 + 4 * (4096 + 1) bytes, rounded to 256) plus, per worker (one per SM),
// two partial slots of 32 head rows x (128 + 1) floats, so the array serves every
// device of up to kStaticScratchMaxSms SMs (a B200 has 148).
// ---------------------------------------------------------------------------------------
constexpr int kStaticScratchMaxSms = 160;
constexpr size_t kStaticScratchBytes = 6u << 20;   // 6 MiB
static_assert(((16 + 4 * (4096 + 1) + 255) / 256) * 256 + (size_t)kStaticScratchMaxSms * 2 * 32 * (128 + 1) * 4 +
                      256 <= kStaticScratchBytes,
              "the static scratch does not hold the default plan of a device with kStaticScratchMaxSms SMs");
__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// Device address of g_static_scratch, looked up once per device with that device
// current (a host-side reference to the array is a host stand-in, not a device address).
void *g_static_scratch_ptr[kMaxDevices] = {};

int static_scratch(int dev, void **ptr) {
    std::lock_guard<std::mutex> lk(g_mutex);
    if (!g_static_scratch_ptr[dev]) {
        void *p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
        if (e != cudaSuccess) return fail_cuda(e, "cudaGetSymbolAddress(static scratch)");
        g_static_scratch_ptr[dev] = p;
    }
    *ptr = g_static_scratch_ptr[dev];
    return KVATTN_OK;
}

// Scratch of a warp-level GQA plan of `bytes`: the per-device workspace (grown with
// cudaMalloc when needed), or, when fixed_scratch is set, the static array above (plans
// that do not fit are refused; nothing is allocated).
int gqa_scratch(DeviceState *dev, size_t bytes, bool fixed_scratch, void **ws) {
    if (fixed_scratch) {
        if (bytes > kStaticScratchBytes) {
            snprintf(t_detail, sizeof(t_detail), "plan needs %zu B of scratch; the static scratch holds %zu B",
                     bytes, kStaticScratchBytes);
            return KVATTN_ERR_UNSUPPORTED;
        }
        // Nothing in the scratch has to start at zero: the decode kernel writes the work
        // split and every partial before the combine kernel reads them.
        return static_scratch(dev->id, ws);
    }
    std::lock_guard<std::mutex> lk(g_mutex);
    return ensure_workspace(dev, bytes, ws);
}

template <int D, int MT>
int run_gqa(const GqaParams &base, const CUtensorMap &kmap, const CUtensorMap &vmap,
            DeviceState *dev, int units_per_seq, cudaStream_t stream, bool fixed_scratch) {
    using C = GqaCfg<D, MT>;
    GqaParams p = base;
    const int smem = C::smem_bytes(p.B);
    if (smem > dev->max_smem_optin) {
        snprintf(t_detail, sizeof(t_detail), "needs %d B shared memory", smem);
        return KVATTN_ERR_UNSUPPORTED;
    }
    // Workers: one persistent CTA per SM unless the work is smaller than that.
    const long long max_tiles =
        (long long)p.B * units_per_seq * ((p.T_max + C::TILE - 1) / C::TILE);
    p.min_tiles = g_force_min_tiles > 0 ? g_force_min_tiles : 4;
    long long workers = g_force_workers > 0 ? g_force_workers : dev->sms;
    const long long by_size = (max_tiles + p.min_tiles - 1) / p.min_tiles;
    if (g_force_workers <= 0 && workers > by_size) workers = by_size;
    if (workers < 1) workers = 1;
    p.workers = (int)workers;
    // Small problems: one worker per unit when every unit fits on its own SM and a unit's
    // whole cache is at most 128 KB -- a split would save less than the combine launch
    // costs (measured: a unit's tiles cost ~0.5 us each in a row on one SM, so at 16 tiles
    // of d = 64 the split with its combine is faster); each unit is then finished in its
    // CTA and no combine runs.
    const long long units = (long long)p.B * units_per_seq;
    const long long unit_bytes = (long long)((p.T_max + C::TILE - 1) / C::TILE) * C::STAGE_BYTES;
    p.unit_mode = g_force_workers <= 0 && units <= dev->sms && unit_bytes <= (128 << 10) ? 1 : 0;
    if (p.unit_mode) {
        p.workers = (int)units;
        auto kern = gqa_decode_kernel<D, MT>;
        cudaError_t e = set_smem_limit(reinterpret_cast<const void *>(kern), dev, smem);
        if (e != cudaSuccess) return fail_cuda(e, "cudaFuncSetAttribute(gqa)");
        kern<<<p.workers, C::NTHREADS, smem, stream>>>(p, kmap, vmap);
        e = cudaGetLastError();
        if (e != cudaSuccess) return fail_cuda(e, "gqa decode launch");
        ++t_launches;
        return KVATTN_OK;
    }

    void *ws = nullptr;
    const size_t meta_bytes = ((16 + (size_t)(p.B + 1) * 4) + 255) & ~size_t(255);
    const size_t lse_bytes = (((size_t)p.workers * 2 * C::HEADS * 4) + 255) & ~size_t(255);
    const size_t o_bytes = (size_t)p.workers * 2 * C::HEADS * D * 4;
    {
        int st = gqa_scratch(dev, meta_bytes + lse_bytes + o_bytes, fixed_scratch, &ws);
        if (st != KVATTN_OK) return st;
    }
    p.ws_meta = ws;
    p.ws_lse = reinterpret_cast<float *>(static_cast<char *>(ws) + meta_bytes);
    p.ws_o = reinterpret_cast<float *>(static_cast<char *>(ws) + meta_bytes + lse_bytes);

    auto kern = gqa_decode_kernel<D, MT>;
    cudaError_t e = set_smem_limit(reinterpret_cast<const void *>(kern), dev, smem);
    if (e != cudaSuccess) return fail_cuda(e, "cudaFuncSetAttribute(gqa)");
    kern<<<p.workers, C::NTHREADS, smem, stream>>>(p, kmap, vmap);
    e = cudaGetLastError();
    if (e != cudaSuccess) return fail_cuda(e, "gqa decode launch");
    ++t_launches;

    CombineParams cp;
    cp.seq_lens = p.seq_lens;
    cp.ws_lse = p.ws_lse;
    cp.ws_o = p.ws_o;
    cp.out = p.out;
    cp.lse = p.lse;
    cp.B = p.B;
    cp.n_q = p.n_q;
    cp.units_per_seq = units_per_seq;
    cp.heads_per_unit = C::HEADS;
    cp.n_hb = p.n_hb;
    cp.n_kv = p.n_kv;
    cp.g = p.g;
    cp.T_max = p.T_max;
    cp.tile = C::TILE;
    cp.workers = p.workers;
    cp.min_tiles = p.min_tiles;
    cp.q_len = 1;
    cp.window = 0;
    cp.unit_split = 0;
    const int rows = p.g < C::HEADS ? p.g : C::HEADS;
    return launch_combine(D, cp, p.B * units_per_seq, rows, stream,
                          combine_warps((p.T_max + C::TILE - 1) / C::TILE, max_tiles, p.workers));
}

// The tcgen05 kernel (gqa_tc_decode.cuh): tokens on the MMA rows, up to 64 query heads
// per unit, NR head columns processed.
template <int NR, bool KV8>
int run_gqa_tc(const GqaParams &base, const CUtensorMap &kmap, const CUtensorMap &vmap,
               const CUtensorMap &qmap, DeviceState *dev, int units_per_seq, cudaStream_t stream) {
    GqaParams p = base;
    p.unit_split = 1;   // equal units are cut into parts of one unit each (schedule.cuh)
    const int smem = gqatc::smem_bytes(p.B);
    if (smem > dev->max_smem_optin) {
        snprintf(t_detail, sizeof(t_detail), "needs %d B shared memory", smem);
        return KVATTN_ERR_UNSUPPORTED;
    }
    const int unit_tiles = (p.T_max + gqatc::TILE - 1) / gqatc::TILE;
    const long long max_tiles = (long long)p.B * units_per_seq * unit_tiles;
    // at least two tiles a worker, but never more than a unit can have: units shorter
    // than that then get a worker each instead of sharing one in turn
    p.min_tiles = g_force_min_tiles > 0 ? g_force_min_tiles : (unit_tiles < 2 ? (unit_tiles > 0 ? unit_tiles : 1) : 2);
    long long workers = g_force_workers > 0 ? g_force_workers : dev->sms;
    const long long by_size = (max_tiles + p.min_tiles - 1) / p.min_tiles;
    if (g_force_workers <= 0 && workers > by_size) workers = by_size;
    if (workers < 1) workers = 1;
    p.workers = (int)workers;

    void *ws = nullptr;
    const size_t meta_bytes = ((16 + (size_t)(p.B + 1) * 4) + 255) & ~size_t(255);
    const size_t lse_bytes = (((size_t)p.workers * 2 * gqatc::HB * 4) + 255) & ~size_t(255);
    const size_t o_bytes = (size_t)p.workers * 2 * gqatc::HB * gqatc::D * 4;
    {
        std::lock_guard<std::mutex> lk(g_mutex);
        int st = ensure_workspace(dev, meta_bytes + lse_bytes + o_bytes, &ws);
        if (st != KVATTN_OK) return st;
    }
    p.ws_meta = ws;
    p.ws_lse = reinterpret_cast<float *>(static_cast<char *>(ws) + meta_bytes);
    p.ws_o = reinterpret_cast<float *>(static_cast<char *>(ws) + meta_bytes + lse_bytes);

    // several new tokens or a window: the instantiation with the visibility mask
    auto kern = (p.q_len > 1 || p.window > 0) ? gqa_tc_decode_kernel<NR, KV8, true> : gqa_tc_decode_kernel<NR, KV8, false>;
    cudaError_t e = set_smem_limit(reinterpret_cast<const void *>(kern), dev, smem);
    if (e != cudaSuccess) return fail_cuda(e, "cudaFuncSetAttribute(gqa tc)");
    kern<<<p.workers, gqatc::Cfg<NR, KV8>::NTHREADS, smem, stream>>>(p, kmap, vmap, qmap);
    e = cudaGetLastError();
    if (e != cudaSuccess) return fail_cuda(e, "gqa tc decode launch");
    ++t_launches;

    CombineParams cp;
    cp.seq_lens = p.seq_lens;
    cp.ws_lse = p.ws_lse;
    cp.ws_o = p.ws_o;
    cp.out = p.out;
    cp.lse = p.lse;
    cp.B = p.B;
    cp.n_q = p.n_q;
    cp.units_per_seq = units_per_seq;
    cp.heads_per_unit = gqatc::HB;
    cp.n_hb = p.n_hb;
    cp.n_kv = p.n_kv;
    cp.g = p.g;
    cp.T_max = p.T_max;
    cp.tile = gqatc::TILE;
    cp.workers = p.workers;
    cp.min_tiles = p.min_tiles;
    cp.q_len = p.q_len;
    cp.window = p.window;
    cp.unit_split = p.unit_split;
    const int rows = p.g * p.q_len < gqatc::HB ? p.g * p.q_len : gqatc::HB;
    return launch_combine(gqatc::D, cp, p.B * units_per_seq, rows, stream,
                          combine_warps((p.T_max + gqatc::TILE - 1) / gqatc::TILE, max_tiles, p.workers));
}

// Which GQA kernel runs: the tcgen05 kernel for head_dim 128 once a group has a few
// query heads (its tensor work per KV byte grows with the group, and the warp-level
// MMA path runs out of tensor throughput first), the warp-level kernel otherwise.
bool use_tc_kernel(int head_dim, int g, int batch, const DeviceState *dev) {
    const bool possible = head_dim == 128 && gqatc::smem_bytes(batch) <= dev->max_smem_optin;
    if (g_gqa_kernel == 1) return false;
    if (g_gqa_kernel == 2) return possible;
    return possible && g >= 4;
}

// A K/V cache as the decode kernels see it: pages of page_size rows per (page, KV head);
// a contiguous cache is one page per sequence (page_size = capacity, no block table).
struct GqaCache {
    const void *k, *v;
    const int32_t *block_table;   // [batch, max_pages] or null (contiguous)
    int capacity;                 // rows addressable per sequence (seq_lens are clamped to it)
    int page_size;
    int max_pages;
    long long pages;              // pages in the pool (contiguous: batch)
    bool e4m3 = false;            // E4M3 codes (value = code * scale) instead of bf16
    float k_scale = 1.f, v_scale = 1.f;
    bool one_page = false;        // every sequence's rows lie in its first page
};

// ---------------------------------------------------------------------------------------
// Several new tokens through the single-token kernels.  New token i (0 <= i < L) of
// sequence b sits at position len_b - L + i and attends, causally, to the cache rows
// [0, len_b - L + i] (optionally the last `window` of them): exactly a single-token decode
// of a sequence of length len_b - L + 1 + i over the same cache.  The call becomes a
// batch of B * L such virtual sequences (v = b * L + i, so q [B, L, ...] and out / lse
// [B, L, ...] are already in its layout), each reading sequence b's pages through a
// block table built here on the device.  A contiguous cache is one page per sequence.
// The cache is read once per new token; the L readers of a page run side by side in the
// work split, so the repeats mostly come from L2.
// ---------------------------------------------------------------------------------------
__global__ void virtual_batch_kernel(const int32_t *seq_lens, const int32_t *block_table, int B, int L,
                                     int max_pages, int capacity, int32_t *vlens, int32_t *vtable) {
    const long long n = (long long)B * L;
    for (long long v = blockIdx.x * (long long)blockDim.x + threadIdx.x; v < n; v += (long long)gridDim.x * blockDim.x) {
        const int b = (int)(v / L), i = (int)(v % L);
        int len = __ldg(seq_lens + b);
        len = len < 0 ? 0 : (len > capacity ? capacity : len);
        const int lv = len - L + 1 + i;
        vlens[v] = lv > 0 ? lv : 0;
        if (block_table)
            for (int m = 0; m < max_pages; ++m) vtable[v * max_pages + m] = __ldg(block_table + (size_t)b * max_pages + m);
        else
            vtable[v] = b;
    }
}

// Builds the virtual batch's lengths and block table in the device's aux buffer.
int virtual_batch(DeviceState *dev, const int32_t *seq_lens, const int32_t *block_table, int B, int L,
                  int max_pages, int capacity, cudaStream_t s, int32_t **vlens, int32_t **vtable) {
    const int mp = block_table ? max_pages : 1;
    const size_t lens_bytes = (((size_t)B * L * 4) + 255) & ~size_t(255);
    const size_t need = lens_bytes + (size_t)B * L * mp * 4;
    {
        std::lock_guard<std::mutex> lk(g_mutex);
        if (dev->aux_bytes < need) {
            if (dev->aux) {
                cudaError_t e = cudaDeviceSynchronize();
                if (e != cudaSuccess) return fail_cuda(e, "cudaDeviceSynchronize (aux grow)");
                cudaFree(dev->aux);
                dev->aux = nullptr;
                dev->aux_bytes = 0;
            }
            cudaError_t e = cudaMalloc(&dev->aux, need);
            if (e != cudaSuccess) {
                cudaGetLastError();
                snprintf(t_detail, sizeof(t_detail), "cudaMalloc(%zu): %s", need, cudaGetErrorString(e));
                return KVATTN_ERR_NO_MEMORY;
            }
            dev->aux_bytes = need;
        }
    }
    *vlens = static_cast<int32_t *>(dev->aux);
    *vtable = reinterpret_cast<int32_t *>(static_cast<char *>(dev->aux) + lens_bytes);
    const long long n = (long long)B * L;
    const int blocks = (int)((n + 255) / 256 < 1024 ? (n + 255) / 256 : 1024);
    virtual_batch_kernel<<<blocks, 256, 0, s>>>(seq_lens, block_table, B, L, mp, capacity, *vlens, *vtable);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail_cuda(e, "virtual batch launch");
    ++t_launches;
    return KVATTN_OK;
}

// noalloc: the warp-level kernel with its scratch in the static array (one new token,
// no window, bf16 contiguous cache).
int gqa_decode_impl(const uint16_t *q, const GqaCache &cache, const int32_t *seq_lens, int batch,
                    int n_q_heads, int n_kv_heads, int head_dim, float scale, float *out, float *lse,
                    void *stream, int q_len = 1, int window = 0, bool noalloc = false) {
    DeviceState *dev = nullptr;
    int st = device_state(&dev);
    if (st != KVATTN_OK) return st;

    const int g = n_q_heads / n_kv_heads;
    // a paged cache needs pages made of whole 128-token tiles for the tcgen05 kernel
    const bool tiles_fit = cache.block_table == nullptr || cache.one_page || cache.page_size % gqatc::TILE == 0;
    // several new tokens the multi-token kernel cannot take (head_dim 64, g * q_len > 64,
    // pages it cannot tile): a virtual batch of single-token sequences (windows only where
    // the tcgen05 kernel serves the single-token form)
    if (q_len > 1 && !noalloc &&
        !(tiles_fit && head_dim == 128 && g * q_len <= gqatc::HB && gqatc::smem_bytes(batch) <= dev->max_smem_optin)) {
        if ((long long)batch * q_len > kMaxBatch) {
            snprintf(t_detail, sizeof(t_detail), "batch * q_len exceeds %d", kMaxBatch);
            return KVATTN_ERR_UNSUPPORTED;
        }
        const bool tc1 = head_dim == 128 && g <= gqatc::HB &&
                         gqatc::smem_bytes(batch * q_len) <= dev->max_smem_optin;
        if ((window > 0 || cache.e4m3) && !tc1) {
            snprintf(t_detail, sizeof(t_detail), "a window or an E4M3 cache needs head_dim 128 and g <= %d",
                     gqatc::HB);
            return KVATTN_ERR_UNSUPPORTED;
        }
        int32_t *vlens = nullptr, *vtable = nullptr;
        st = virtual_batch(dev, seq_lens, cache.block_table, batch, q_len, cache.max_pages, cache.capacity,
                           static_cast<cudaStream_t>(stream), &vlens, &vtable);
        if (st != KVATTN_OK) return st;
        GqaCache vc = cache;
        vc.block_table = vtable;
        vc.max_pages = cache.block_table ? cache.max_pages : 1;
        vc.one_page = cache.block_table == nullptr;
        return gqa_decode_impl(q, vc, vlens, batch * q_len, n_q_heads, n_kv_heads, head_dim, scale, out, lse,
                               stream, 1, window);
    }
    if (!noalloc && g_gqa_kernel == 2 && !(tiles_fit && use_tc_kernel(head_dim, g, batch, dev))) {
        snprintf(t_detail, sizeof(t_detail),
                 "tcgen05 GQA kernel needs head_dim 128, batch <= %d and pages of multiples of 128 rows",
                 (dev->max_smem_optin - gqatc::smem_bytes(0)) / 4);
        return KVATTN_ERR_UNSUPPORTED;
    }
    // several new tokens, or a window: the tcgen05 kernel, whose score columns are the
    // (position, head) pairs of a group
    const bool multi = q_len > 1 || window > 0;
    if (multi && !(tiles_fit && head_dim == 128 && gqatc::smem_bytes(batch) <= dev->max_smem_optin &&
                   g * q_len <= gqatc::HB)) {
        snprintf(t_detail, sizeof(t_detail), "multi-token decode needs head_dim 128 and g * q_len <= %d",
                 gqatc::HB);
        return KVATTN_ERR_UNSUPPORTED;
    }
    // an E4M3 cache: the tcgen05 kernel (8-bit MMAs straight from the tiles)
    if (cache.e4m3 && (g_gqa_kernel == 1 || !(tiles_fit && head_dim == 128 && g * q_len <= gqatc::HB &&
                                              gqatc::smem_bytes(batch) <= dev->max_smem_optin))) {
        snprintf(t_detail, sizeof(t_detail), "E4M3 cache needs head_dim 128, g * q_len <= %d and pages of "
                 "multiples of 128 rows", gqatc::HB);
        return KVATTN_ERR_UNSUPPORTED;
    }
    const bool tc = !noalloc && (multi || cache.e4m3 || (tiles_fit && use_tc_kernel(head_dim, g, batch, dev)));
    const int MT = g <= 16 ? 1 : 2;
    const int heads = tc ? gqatc::HB : 16 * MT;
    const int n_hb = (g * q_len + heads - 1) / heads;
    const uint32_t box_rows = tc ? gqatc::TILE : 64;

    // (an E4M3 row of head_dim codes is mapped as head_dim / 2 two-byte elements: the TMA
    // moves bytes, and its zero fill is zero codes)
    const uint64_t row_elems = cache.e4m3 ? (uint64_t)head_dim / 2 : (uint64_t)head_dim;
    CUtensorMap kmap, vmap, qmap;
    st = make_map_3d(&kmap, cache.k, row_elems, cache.page_size, (uint64_t)cache.pages * n_kv_heads, 64, box_rows,
                     CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != KVATTN_OK) return st;
    st = make_map_3d(&vmap, cache.v, row_elems, cache.page_size, (uint64_t)cache.pages * n_kv_heads, 64, box_rows,
                     CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != KVATTN_OK) return st;
    const int gl = g * q_len;    // score columns of a unit
    if (tc && q_len == 1) {
        // box rows = the score product's N for this group size (query heads per block)
        const uint32_t q_rows = g > 32 ? 64 : g > 16 ? 32 : 16;
        st = make_map_3d(&qmap, q, head_dim, n_q_heads, batch, 64, q_rows, CU_TENSOR_MAP_SWIZZLE_128B);
        if (st != KVATTN_OK) return st;
    } else if (tc) {
        // q [B, q_len, n_q, d]: box of the group's g heads at all q_len positions
        st = make_map_4d(&qmap, q, head_dim, n_q_heads, q_len, batch, 64, g, q_len, CU_TENSOR_MAP_SWIZZLE_128B);
        if (st != KVATTN_OK) return st;
    }

    GqaParams p = {};
    p.q = reinterpret_cast<const __nv_bfloat16 *>(q);
    p.seq_lens = seq_lens;
    p.out = out;
    p.lse = lse;
    p.B = batch;
    p.n_q = n_q_heads;
    p.n_kv = n_kv_heads;
    p.T_max = cache.capacity;
    p.g = g;
    p.n_hb = n_hb;
    p.scale_log2 = (float)((double)scale * 1.4426950408889634);
    p.block_table = cache.block_table;
    p.max_pages = cache.max_pages;
    p.page_size = cache.page_size;
    p.q_len = q_len;
    p.window = window;
    p.k_scale = cache.k_scale;
    p.v_scale = cache.v_scale;
    const int U = n_kv_heads * n_hb;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (tc && cache.e4m3) {
        if (gl > 32) return run_gqa_tc<64, true>(p, kmap, vmap, qmap, dev, U, s);
        if (gl > 16) return run_gqa_tc<32, true>(p, kmap, vmap, qmap, dev, U, s);
        if (gl > 8) return run_gqa_tc<16, true>(p, kmap, vmap, qmap, dev, U, s);
        return run_gqa_tc<8, true>(p, kmap, vmap, qmap, dev, U, s);
    }
    if (tc) {
        if (gl > 32) return run_gqa_tc<64, false>(p, kmap, vmap, qmap, dev, U, s);
        if (gl > 16) return run_gqa_tc<32, false>(p, kmap, vmap, qmap, dev, U, s);
        if (gl > 8) return run_gqa_tc<16, false>(p, kmap, vmap, qmap, dev, U, s);
        return run_gqa_tc<8, false>(p, kmap, vmap, qmap, dev, U, s);
    }
    if (head_dim == 128)
        return MT == 1 ? run_gqa<128, 1>(p, kmap, vmap, dev, U, s, noalloc)
                       : run_gqa<128, 2>(p, kmap, vmap, dev, U, s, noalloc);
    return MT == 1 ? run_gqa<64, 1>(p, kmap, vmap, dev, U, s, noalloc)
                   : run_gqa<64, 2>(p, kmap, vmap, dev, U, s, noalloc);
}

// A latent + rotary-key cache as the MLA kernel sees it (pages of page_size rows; a
// contiguous cache is one page per sequence).
struct MlaCache {
    const void *lat, *rope;       // bf16, or E4M3 codes (e4m3)
    const int32_t *block_table;   // [batch, max_pages] or null (contiguous)
    int capacity;
    int page_size;
    int max_pages;
    long long pages;
    bool e4m3;
    float latent_scale, rope_scale;   // E4M3: a code's value times these
};

int mla_decode_impl(const uint16_t *q_latent, const uint16_t *q_rope, const MlaCache &cache,
                    const int32_t *seq_lens, int batch, int n_heads, float scale, float *out, float *lse,
                    void *stream) {
    DeviceState *dev = nullptr;
    int st = device_state(&dev);
    if (st != KVATTN_OK) return st;

    MlaMaps maps;
    if (cache.e4m3) {
        // E4M3 codes, two to an element of the map: a box of [64 rows x 128 codes]; the
        // RoPE map is 64 codes wide, so its box reads 64 codes and zero-fills the other 64
        st = make_map_3d(&maps.rope, cache.rope, 32, cache.page_size, (uint64_t)cache.pages, 64, mla::SUB,
                         CU_TENSOR_MAP_SWIZZLE_128B);
        if (st != KVATTN_OK) return st;
        // key slot: the 4 latent chunks of a row block in one copy; value slot: chunks r and
        // 2 + r (128-byte units of a 512-byte row) in one copy
        const uint64_t rowb = 512, pageb = rowb * (uint64_t)cache.page_size;
        const uint64_t kd[4] = {64, (uint64_t)cache.page_size, 4, (uint64_t)cache.pages};
        const uint64_t ks[3] = {rowb, 128, pageb};
        const uint32_t kb[4] = {64, (uint32_t)mla::SUB, 4, 1};
        st = make_map_view(&maps.latk, cache.lat, 4, kd, ks, kb);
        if (st != KVATTN_OK) return st;
        maps.latk2 = maps.latk;
        const uint64_t vd[5] = {64, (uint64_t)cache.page_size, 2, 2, (uint64_t)cache.pages};
        const uint64_t vs[4] = {rowb, 128, 256, pageb};
        const uint32_t vb[5] = {64, (uint32_t)mla::SUB, 1, 2, 1};
        st = make_map_view(&maps.latv, cache.lat, 5, vd, vs, vb);
        if (st != KVATTN_OK) return st;
        maps.qlatc = maps.latk;   // (the query is read by the threads)
        maps.qrope = maps.latk;
    } else {
        st = make_map_3d(&maps.rope, cache.rope, 64, cache.page_size, (uint64_t)cache.pages, 64, mla::SUB,
                         CU_TENSOR_MAP_SWIZZLE_128B);
        if (st != KVATTN_OK) return st;
        st = make_map_3d(&maps.qrope, q_rope, 64, n_heads, batch, 64, mla::HC, CU_TENSOR_MAP_SWIZZLE_128B);
        if (st != KVATTN_OK) return st;
        // [rows][8 chunks][64] views of the latent rows: key slots of 3 and 2 chunks, the
        // value slot (chunks 4j + 2r + {0, 1}, j = 0, 1) and the query's chunks 4..7, each
        // in one copy
        const uint64_t rowb = 1024, pageb = rowb * (uint64_t)cache.page_size;
        const uint64_t kd[4] = {64, (uint64_t)cache.page_size, 8, (uint64_t)cache.pages};
        const uint64_t ks[3] = {rowb, 128, pageb};
        const uint32_t kb3[4] = {64, (uint32_t)mla::SUB, 3, 1};
        const uint32_t kb2[4] = {64, (uint32_t)mla::SUB, 2, 1};
        st = make_map_view(&maps.latk, cache.lat, 4, kd, ks, kb3);
        if (st != KVATTN_OK) return st;
        st = make_map_view(&maps.latk2, cache.lat, 4, kd, ks, kb2);
        if (st != KVATTN_OK) return st;
        const uint64_t vd[5] = {64, (uint64_t)cache.page_size, 4, 2, (uint64_t)cache.pages};
        const uint64_t vs[4] = {rowb, 128, 512, pageb};
        const uint32_t vb[5] = {64, (uint32_t)mla::SUB, 2, 2, 1};
        st = make_map_view(&maps.latv, cache.lat, 5, vd, vs, vb);
        if (st != KVATTN_OK) return st;
        const uint64_t qd[4] = {64, (uint64_t)n_heads, 8, (uint64_t)batch};
        const uint64_t qs[3] = {1024, 128, 1024 * (uint64_t)n_heads};
        const uint32_t qb[4] = {64, (uint32_t)mla::HC, (uint32_t)mla::NQS - 1, 1};
        st = make_map_view(&maps.qlatc, q_latent, 4, qd, qs, qb);
        if (st != KVATTN_OK) return st;
    }
    const void *kern = cache.e4m3 ? reinterpret_cast<const void *>(mla_decode_kernel<true>)
                                  : reinterpret_cast<const void *>(mla_decode_kernel<false>);

    MlaParams p = {};
    p.q_latent = reinterpret_cast<const __nv_bfloat16 *>(q_latent);
    p.q_rope = reinterpret_cast<const __nv_bfloat16 *>(q_rope);
    p.seq_lens = seq_lens;
    p.out = out;
    p.lse = lse;
    p.B = batch;
    p.H = n_heads;
    p.T_max = cache.capacity;
    p.block_table = cache.block_table;
    p.max_pages = cache.max_pages;
    p.page_size = cache.page_size;
    p.scale_log2 = (float)((double)scale * 1.4426950408889634);
    unsigned int epoch = ++dev->mla_calls;
    if (epoch == 0) epoch = ++dev->mla_calls;   // 0 is the counters' state at load
    p.epoch = epoch;
    p.latent_scale = cache.e4m3 ? cache.latent_scale : 1.f;
    p.rope_scale = cache.e4m3 ? cache.rope_scale : 1.f;
    const int smem = mla::smem_bytes(batch);
    if (smem > dev->max_smem_optin) {
        snprintf(t_detail, sizeof(t_detail), "needs %d B shared memory", smem);
        return KVATTN_ERR_UNSUPPORTED;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = set_smem_limit(kern, dev, smem);
    if (e != cudaSuccess) return fail_cuda(e, "cudaFuncSetAttribute(mla)");
    // Workers are CTA pairs; a persistent grid must not exceed the pairs that can be
    // resident at once (a pair needs two SMs of one GPC).
    if (dev->mla_clusters == 0) {
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.gridDim = dim3(2 * (dev->sms / 2), 1, 1);
        cfg.blockDim = dim3(mla::NTHREADS, 1, 1);
        cfg.dynamicSmemBytes = smem;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        e = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
        if (e != cudaSuccess || n <= 0) {
            cudaGetLastError();
            n = dev->sms / 2;
        }
        dev->mla_clusters = n < dev->sms / 2 ? n : dev->sms / 2;
    }
    const int seq_tiles = (cache.capacity + mla::TILE - 1) / mla::TILE;
    const long long max_tiles = (long long)batch * seq_tiles;
    // at least four tiles a worker, but never more than a sequence can have: a batch of
    // short sequences then gets a CTA pair per sequence instead of pairs that take
    // several sequences in turn (a query load, a first tile and an epilogue each)
    p.min_tiles = g_force_min_tiles > 0 ? g_force_min_tiles : (seq_tiles < 4 ? (seq_tiles > 0 ? seq_tiles : 1) : 4);
    long long workers = g_force_workers > 0 ? g_force_workers : dev->mla_clusters;
    const long long by_size = (max_tiles + p.min_tiles - 1) / p.min_tiles;
    if (g_force_workers <= 0 && workers > by_size) workers = by_size;
    if (workers < 1) workers = 1;
    p.workers = (int)workers;

    // Partial results of the sequences cut by a worker boundary, merged inside the kernel
    // by the last worker to finish each block.
    void *ws = nullptr;
    const size_t wlse_bytes = (((size_t)p.workers * 2 * mla::HR * 4) + 255) & ~size_t(255);
    const size_t wo_bytes = (size_t)p.workers * 2 * mla::HR * 512 * 4;
    {
        std::lock_guard<std::mutex> lk(g_mutex);
        st = ensure_workspace(dev, wlse_bytes + wo_bytes, &ws);
        if (st != KVATTN_OK) return st;
    }
    p.ws_lse = reinterpret_cast<float *>(ws);
    p.ws_o = reinterpret_cast<float *>(static_cast<char *>(ws) + wlse_bytes);

    if (cache.e4m3)
        mla_decode_kernel<true><<<2 * p.workers, mla::NTHREADS, smem, s>>>(p, maps);
    else
        mla_decode_kernel<false><<<2 * p.workers, mla::NTHREADS, smem, s>>>(p, maps);
    e = cudaGetLastError();
    if (e != cudaSuccess) return fail_cuda(e, "mla decode launch");
    ++t_launches;
    return KVATTN_OK;
}

// Argument checks of kvattn_gqa_decode (and of kvattn_gqa_decode_noalloc, which takes the
// same arguments).
int check_gqa_args(const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache, const int32_t *seq_lens,
                   int max_seq_len, int batch, int n_q_heads, int n_kv_heads, int head_dim, float scale,
                   const float *out, const float *lse) {
    if (!q || !k_cache || !v_cache || !seq_lens || !out || !lse) return KVATTN_ERR_INVALID_ARG;
    if (batch <= 0 || n_q_heads <= 0 || n_kv_heads <= 0 || max_seq_len <= 0)
        return KVATTN_ERR_INVALID_ARG;
    if (n_q_heads % n_kv_heads != 0) return KVATTN_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return KVATTN_ERR_INVALID_ARG;
    if (head_dim != 64 && head_dim != 128) return KVATTN_ERR_UNSUPPORTED;
    if (batch > kMaxBatch) return KVATTN_ERR_UNSUPPORTED;
    if ((long long)batch * n_kv_heads * max_seq_len >= (1ll << 31)) return KVATTN_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(seq_lens) ||
        !aligned16(out) || !aligned16(lse))
        return KVATTN_ERR_MISALIGNED;
    const size_t q_bytes = (size_t)batch * n_q_heads * head_dim * 2;
    const size_t kv_bytes = (size_t)batch * n_kv_heads * max_seq_len * head_dim * 2;
    const size_t out_bytes = (size_t)batch * n_q_heads * head_dim * 4;
    const size_t lse_bytes = (size_t)batch * n_q_heads * 4;
    const void *ins[4] = {q, k_cache, v_cache, seq_lens};
    const size_t in_sz[4] = {q_bytes, kv_bytes, kv_bytes, (size_t)batch * 4};
    for (int i = 0; i < 4; ++i)
        if (overlaps(out, out_bytes, ins[i], in_sz[i]) || overlaps(lse, lse_bytes, ins[i], in_sz[i]))
            return KVATTN_ERR_INVALID_ARG;
    if (overlaps(out, out_bytes, lse, lse_bytes)) return KVATTN_ERR_INVALID_ARG;
    return KVATTN_OK;
}

}  // namespace

extern "C" {

int kvattn_gqa_decode(const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                      const int32_t *seq_lens, int max_seq_len, int batch, int n_q_heads,
                      int n_kv_heads, int head_dim, float scale, float *out, float *lse,
                      void *stream) {
    const int st = check_gqa_args(q, k_cache, v_cache, seq_lens, max_seq_len, batch, n_q_heads, n_kv_heads,
                                  head_dim, scale, out, lse);
    if (st != KVATTN_OK) return st;
    const GqaCache cache{k_cache, v_cache, nullptr, max_seq_len, max_seq_len, 1, batch};
    return gqa_decode_impl(q, cache, seq_lens, batch, n_q_heads, n_kv_heads, head_dim, scale, out, lse, stream);
}

int kvattn_gqa_decode_paged(const uint16_t *q, const uint16_t *k_pages, const uint16_t *v_pages,
                            const int32_t *block_table, const int32_t *seq_lens, int num_pages,
                            int page_size, int max_pages_per_seq, int batch, int n_q_heads,
                            int n_kv_heads, int head_dim, float scale, float *out, float *lse,
                            void *stream) {
    if (!q || !k_pages || !v_pages || !block_table || !seq_lens || !out || !lse) return KVATTN_ERR_INVALID_ARG;
    if (batch <= 0 || n_q_heads <= 0 || n_kv_heads <= 0 || num_pages <= 0 || page_size <= 0 ||
        max_pages_per_seq <= 0)
        return KVATTN_ERR_INVALID_ARG;
    if (n_q_heads % n_kv_heads != 0) return KVATTN_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return KVATTN_ERR_INVALID_ARG;
    if (head_dim != 64 && head_dim != 128) return KVATTN_ERR_UNSUPPORTED;
    if (page_size % 64 != 0) return KVATTN_ERR_UNSUPPORTED;
    if (batch > kMaxBatch) return KVATTN_ERR_UNSUPPORTED;
    if ((long long)num_pages * n_kv_heads * page_size >= (1ll << 31) ||
        (long long)max_pages_per_seq * page_size >= (1ll << 31))
        return KVATTN_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k_pages) || !aligned16(v_pages) || !aligned16(block_table) ||
        !aligned16(seq_lens) || !aligned16(out) || !aligned16(lse))
        return KVATTN_ERR_MISALIGNED;
    const size_t q_bytes = (size_t)batch * n_q_heads * head_dim * 2;
    const size_t kv_bytes = (size_t)num_pages * n_kv_heads * page_size * head_dim * 2;
    const size_t out_bytes = (size_t)batch * n_q_heads * head_dim * 4;
    const size_t lse_bytes = (size_t)batch * n_q_heads * 4;
    const void *ins[5] = {q, k_pages, v_pages, seq_lens, block_table};
    const size_t in_sz[5] = {q_bytes, kv_bytes, kv_bytes, (size_t)batch * 4,
                             (size_t)batch * max_pages_per_seq * 4};
    for (int i = 0; i < 5; ++i)
        if (overlaps(out, out_bytes, ins[i], in_sz[i]) || overlaps(lse, lse_bytes, ins[i], in_sz[i]))
            return KVATTN_ERR_INVALID_ARG;
    if (overlaps(out, out_bytes, lse, lse_bytes)) return KVATTN_ERR_INVALID_ARG;
    const GqaCache cache{k_pages, v_pages, block_table, max_pages_per_seq * page_size, page_size,
                         max_pages_per_seq, num_pages};
    return gqa_decode_impl(q, cache, seq_lens, batch, n_q_heads, n_kv_heads, head_dim, scale, out, lse, stream);
}

int kvattn_gqa_decode_multi(const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                            const int32_t *seq_lens, int max_seq_len, int batch, int q_len, int n_q_heads,
                            int n_kv_heads, int head_dim, float scale, int window, float *out, float *lse,
                            void *stream) {
    if (!q || !k_cache || !v_cache || !seq_lens || !out || !lse) return KVATTN_ERR_INVALID_ARG;
    if (batch <= 0 || q_len <= 0 || n_q_heads <= 0 || n_kv_heads <= 0 || max_seq_len <= 0 || window < 0)
        return KVATTN_ERR_INVALID_ARG;
    if (n_q_heads % n_kv_heads != 0) return KVATTN_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return KVATTN_ERR_INVALID_ARG;
    if (head_dim != 64 && head_dim != 128) return KVATTN_ERR_UNSUPPORTED;
    if (window > 0 && (head_dim != 128 || n_q_heads / n_kv_heads > gqatc::HB)) return KVATTN_ERR_UNSUPPORTED;
    if (batch > kMaxBatch || (long long)batch * q_len > kMaxBatch) return KVATTN_ERR_UNSUPPORTED;
    if ((long long)batch * n_kv_heads * max_seq_len >= (1ll << 31)) return KVATTN_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(seq_lens) ||
        !aligned16(out) || !aligned16(lse))
        return KVATTN_ERR_MISALIGNED;
    const size_t q_bytes = (size_t)batch * q_len * n_q_heads * head_dim * 2;
    const size_t kv_bytes = (size_t)batch * n_kv_heads * max_seq_len * head_dim * 2;
    const size_t out_bytes = (size_t)batch * q_len * n_q_heads * head_dim * 4;
    const size_t lse_bytes = (size_t)batch * q_len * n_q_heads * 4;
    const void *ins[4] = {q, k_cache, v_cache, seq_lens};
    const size_t in_sz[4] = {q_bytes, kv_bytes, kv_bytes, (size_t)batch * 4};
    for (int i = 0; i < 4; ++i)
        if (overlaps(out, out_bytes, ins[i], in_sz[i]) || overlaps(lse, lse_bytes, ins[i], in_sz[i]))
            return KVATTN_ERR_INVALID_ARG;
    if (overlaps(out, out_bytes, lse, lse_bytes)) return KVATTN_ERR_INVALID_ARG;
    const GqaCache cache{k_cache, v_cache, nullptr, max_seq_len, max_seq_len, 1, batch};
    return gqa_decode_impl(q, cache, seq_lens, batch, n_q_heads, n_kv_heads, head_dim, scale, out, lse, stream,
                           q_len, window);
}

int kvattn_gqa_decode_fp8(const uint16_t *q, const uint8_t *k_cache, const uint8_t *v_cache,
                          const int32_t *seq_lens, int max_seq_len, int batch, int q_len, int n_q_heads,
                          int n_kv_heads, int head_dim, float scale, float k_scale, float v_scale, int window,
                          float *out, float *lse, void *stream) {
    if (!q || !k_cache || !v_cache || !seq_lens || !out || !lse) return KVATTN_ERR_INVALID_ARG;
    if (batch <= 0 || q_len <= 0 || n_q_heads <= 0 || n_kv_heads <= 0 || max_seq_len <= 0 || window < 0)
        return KVATTN_ERR_INVALID_ARG;
    if (n_q_heads % n_kv_heads != 0) return KVATTN_ERR_INVALID_ARG;
    if (!std::isfinite(scale) || !std::isfinite(k_scale) || !std::isfinite(v_scale) || !(k_scale > 0.f) ||
        !(v_scale > 0.f))
        return KVATTN_ERR_INVALID_ARG;
    if (head_dim != 128 || n_q_heads / n_kv_heads > gqatc::HB) return KVATTN_ERR_UNSUPPORTED;
    if (batch > kMaxBatch || (long long)batch * q_len > kMaxBatch) return KVATTN_ERR_UNSUPPORTED;
    if ((long long)batch * n_kv_heads * max_seq_len >= (1ll << 31)) return KVATTN_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(seq_lens) ||
        !aligned16(out) || !aligned16(lse))
        return KVATTN_ERR_MISALIGNED;
    const size_t q_bytes = (size_t)batch * q_len * n_q_heads * head_dim * 2;
    const size_t kv_bytes = (size_t)batch * n_kv_heads * max_seq_len * head_dim;
    const size_t out_bytes = (size_t)batch * q_len * n_q_heads * head_dim * 4;
    const size_t lse_bytes = (size_t)batch * q_len * n_q_heads * 4;
    const void *ins[4] = {q, k_cache, v_cache, seq_lens};
    const size_t in_sz[4] = {q_bytes, kv_bytes, kv_bytes, (size_t)batch * 4};
    for (int i = 0; i < 4; ++i)
        if (overlaps(out, out_bytes, ins[i], in_sz[i]) || overlaps(lse, lse_bytes, ins[i], in_sz[i]))
            return KVATTN_ERR_INVALID_ARG;
    if (overlaps(out, out_bytes, lse, lse_bytes)) return KVATTN_ERR_INVALID_ARG;
    GqaCache cache{k_cache, v_cache, nullptr, max_seq_len, max_seq_len, 1, batch};
    cache.e4m3 = true;
    cache.k_scale = k_scale;
    cache.v_scale = v_scale;
    return gqa_decode_impl(q, cache, seq_lens, batch, n_q_heads, n_kv_heads, head_dim, scale, out, lse, stream,
                           q_len, window);
}

int kvattn_gqa_decode_fp8_paged(const uint16_t *q, const uint8_t *k_pages, const uint8_t *v_pages,
                                const int32_t *block_table, const int32_t *seq_lens, int num_pages, int page_size,
                                int max_pages_per_seq, int batch, int n_q_heads, int n_kv_heads, int head_dim,
                                float scale, float k_scale, float v_scale, float *out, float *lse, void *stream) {
    if (!q || !k_pages || !v_pages || !block_table || !seq_lens || !out || !lse) return KVATTN_ERR_INVALID_ARG;
    if (batch <= 0 || n_q_heads <= 0 || n_kv_heads <= 0 || num_pages <= 0 || page_size <= 0 ||
        max_pages_per_seq <= 0)
        return KVATTN_ERR_INVALID_ARG;
    if (n_q_heads % n_kv_heads != 0) return KVATTN_ERR_INVALID_ARG;
    if (!std::isfinite(scale) || !std::isfinite(k_scale) || !std::isfinite(v_scale) || !(k_scale > 0.f) ||
        !(v_scale > 0.f))
        return KVATTN_ERR_INVALID_ARG;
    if (head_dim != 128 || n_q_heads / n_kv_heads > gqatc::HB || page_size % gqatc::TILE != 0)
        return KVATTN_ERR_UNSUPPORTED;
    if (batch > kMaxBatch) return KVATTN_ERR_UNSUPPORTED;
    if ((long long)num_pages * n_kv_heads * page_size >= (1ll << 31) ||
        (long long)max_pages_per_seq * page_size >= (1ll << 31))
        return KVATTN_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k_pages) || !aligned16(v_pages) || !aligned16(block_table) ||
        !aligned16(seq_lens) || !aligned16(out) || !aligned16(lse))
        return KVATTN_ERR_MISALIGNED;
    const size_t q_bytes = (size_t)batch * n_q_heads * head_dim * 2;
    const size_t kv_bytes = (size_t)num_pages * n_kv_heads * page_size * head_dim;
    const size_t out_bytes = (size_t)batch * n_q_heads * head_dim * 4;
    const size_t lse_bytes = (size_t)batch * n_q_heads * 4;
    const void *ins[5] = {q, k_pages, v_pages, seq_lens, block_table};
    const size_t in_sz[5] = {q_bytes, kv_bytes, kv_bytes, (size_t)batch * 4, (size_t)batch * max_pages_per_seq * 4};
    for (int i = 0; i < 5; ++i)
        if (overlaps(out, out_bytes, ins[i], in_sz[i]) || overlaps(lse, lse_bytes, ins[i], in_sz[i]))
            return KVATTN_ERR_INVALID_ARG;
    if (overlaps(out, out_bytes, lse, lse_bytes)) return KVATTN_ERR_INVALID_ARG;
    GqaCache cache{k_pages, v_pages, block_table, max_pages_per_seq * page_size, page_size, max_pages_per_seq,
                   num_pages};
    cache.e4m3 = true;
    cache.k_scale = k_scale;
    cache.v_scale = v_scale;
    return gqa_decode_impl(q, cache, seq_lens, batch, n_q_heads, n_kv_heads, head_dim, scale, out, lse, stream);
}

// Checks and launch shared by the four MLA entry points: a contiguous cache is one page
// per sequence (block_table null, num_pages = batch, page_size = max_pages_per_seq =
// max_seq_len).  code_bytes = 2 (bf16) or 1 (E4M3).
static int mla_entry(const uint16_t *q_latent, const uint16_t *q_rope, const void *lat, const void *rope,
              const int32_t *block_table, const int32_t *seq_lens, int num_pages, int page_size,
              int max_pages_per_seq, int batch, int n_heads, int latent_dim, int rope_dim, float scale, bool e4m3,
              float latent_scale, float rope_scale, float *out, float *lse, void *stream, int q_len = 1) {
    const bool paged = block_table != nullptr;
    if (q_len <= 0) return KVATTN_ERR_INVALID_ARG;
    if ((long long)batch * q_len > mla::MAX_BATCH) return KVATTN_ERR_UNSUPPORTED;
    if (!q_latent || !q_rope || !lat || !rope || !seq_lens || !out || !lse) return KVATTN_ERR_INVALID_ARG;
    if (batch <= 0 || n_heads <= 0 || num_pages <= 0 || page_size <= 0 || max_pages_per_seq <= 0 ||
        latent_dim <= 0 || rope_dim < 0)
        return KVATTN_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return KVATTN_ERR_INVALID_ARG;
    if (e4m3 && (!std::isfinite(latent_scale) || !std::isfinite(rope_scale) || !(latent_scale > 0.f) ||
                 !(rope_scale > 0.f)))
        return KVATTN_ERR_INVALID_ARG;
    if (latent_dim != 512 || rope_dim != 64 || n_heads > 128) return KVATTN_ERR_UNSUPPORTED;
    if (paged && page_size % mla::SUB != 0) return KVATTN_ERR_UNSUPPORTED;
    if (batch > mla::MAX_BATCH) return KVATTN_ERR_UNSUPPORTED;
    if ((long long)num_pages * page_size >= (1ll << 31) || (long long)max_pages_per_seq * page_size >= (1ll << 31))
        return KVATTN_ERR_UNSUPPORTED;
    if (!aligned16(q_latent) || !aligned16(q_rope) || !aligned16(lat) || !aligned16(rope) ||
        (paged && !aligned16(block_table)) || !aligned16(seq_lens) || !aligned16(out) || !aligned16(lse))
        return KVATTN_ERR_MISALIGNED;
    const size_t cb = e4m3 ? 1 : 2;
    const size_t ql_bytes = (size_t)batch * q_len * n_heads * latent_dim * 2;
    const size_t qr_bytes = (size_t)batch * q_len * n_heads * rope_dim * 2;
    const size_t lat_bytes = (size_t)num_pages * page_size * latent_dim * cb;
    const size_t rope_bytes = (size_t)num_pages * page_size * rope_dim * cb;
    const size_t out_bytes = (size_t)batch * q_len * n_heads * latent_dim * 4;
    const size_t lse_bytes = (size_t)batch * q_len * n_heads * 4;
    const void *ins[6] = {q_latent, q_rope, lat, rope, seq_lens, block_table};
    const size_t in_sz[6] = {ql_bytes, qr_bytes, lat_bytes, rope_bytes, (size_t)batch * 4,
                             paged ? (size_t)batch * max_pages_per_seq * 4 : 0};
    for (int i = 0; i < 6; ++i)
        if (overlaps(out, out_bytes, ins[i], in_sz[i]) || overlaps(lse, lse_bytes, ins[i], in_sz[i]))
            return KVATTN_ERR_INVALID_ARG;
    if (overlaps(out, out_bytes, lse, lse_bytes)) return KVATTN_ERR_INVALID_ARG;
    MlaCache cache{lat, rope, block_table, max_pages_per_seq * page_size, page_size, max_pages_per_seq,
                   num_pages, e4m3, latent_scale, rope_scale};
    if (q_len == 1) return mla_decode_impl(q_latent, q_rope, cache, seq_lens, batch, n_heads, scale, out, lse, stream);
    // several new tokens: a virtual batch of single-token sequences over the same pages
    DeviceState *dev = nullptr;
    int st = device_state(&dev);
    if (st != KVATTN_OK) return st;
    int32_t *vlens = nullptr, *vtable = nullptr;
    st = virtual_batch(dev, seq_lens, block_table, batch, q_len, max_pages_per_seq, cache.capacity,
                       static_cast<cudaStream_t>(stream), &vlens, &vtable);
    if (st != KVATTN_OK) return st;
    cache.block_table = vtable;
    if (!paged) cache.max_pages = 1;   // one page (the whole capacity) per sequence
    return mla_decode_impl(q_latent, q_rope, cache, vlens, batch * q_len, n_heads, scale, out, lse, stream);
}

int kvattn_mla_decode(const uint16_t *q_latent, const uint16_t *q_rope,
                      const uint16_t *latent_cache, const uint16_t *rope_cache,
                      const int32_t *seq_lens, int max_seq_len, int batch, int n_heads,
                      int latent_dim, int rope_dim, float scale, float *out, float *lse,
                      void *stream) {
    return mla_entry(q_latent, q_rope, latent_cache, rope_cache, nullptr, seq_lens, batch, max_seq_len, 1,
                     batch, n_heads, latent_dim, rope_dim, scale, false, 1.f, 1.f, out, lse, stream);
}

int kvattn_mla_decode_paged(const uint16_t *q_latent, const uint16_t *q_rope, const uint16_t *latent_pages,
                            const uint16_t *rope_pages, const int32_t *block_table, const int32_t *seq_lens,
                            int num_pages, int page_size, int max_pages_per_seq, int batch, int n_heads,
                            int latent_dim, int rope_dim, float scale, float *out, float *lse, void *stream) {
    if (!block_table) return KVATTN_ERR_INVALID_ARG;
    return mla_entry(q_latent, q_rope, latent_pages, rope_pages, block_table, seq_lens, num_pages, page_size,
                     max_pages_per_seq, batch, n_heads, latent_dim, rope_dim, scale, false, 1.f, 1.f, out, lse,
                     stream);
}

int kvattn_mla_decode_fp8(const uint16_t *q_latent, const uint16_t *q_rope, const uint8_t *latent_cache,
                          const uint8_t *rope_cache, const int32_t *seq_lens, int max_seq_len, int batch,
                          int n_heads, int latent_dim, int rope_dim, float scale, float latent_scale,
                          float rope_scale, float *out, float *lse, void *stream) {
    return mla_entry(q_latent, q_rope, latent_cache, rope_cache, nullptr, seq_lens, batch, max_seq_len, 1,
                     batch, n_heads, latent_dim, rope_dim, scale, true, latent_scale, rope_scale, out, lse, stream);
}

int kvattn_mla_decode_multi(const uint16_t *q_latent, const uint16_t *q_rope, const void *latent_cache,
                            const void *rope_cache, const int32_t *seq_lens, int max_seq_len, int batch, int q_len,
                            int n_heads, int latent_dim, int rope_dim, float scale, int e4m3, float latent_scale,
                            float rope_scale, float *out, float *lse, void *stream) {
    return mla_entry(q_latent, q_rope, latent_cache, rope_cache, nullptr, seq_lens, batch, max_seq_len, 1,
                     batch, n_heads, latent_dim, rope_dim, scale, e4m3 != 0, e4m3 ? latent_scale : 1.f,
                     e4m3 ? rope_scale : 1.f, out, lse, stream, q_len);
}

int kvattn_mla_decode_fp8_paged(const uint16_t *q_latent, const uint16_t *q_rope, const uint8_t *latent_pages,
                                const uint8_t *rope_pages, const int32_t *block_table, const int32_t *seq_lens,
                                int num_pages, int page_size, int max_pages_per_seq, int batch, int n_heads,
                                int latent_dim, int rope_dim, float scale, float latent_scale, float rope_scale,
                                float *out, float *lse, void *stream) {
    if (!block_table) return KVATTN_ERR_INVALID_ARG;
    return mla_entry(q_latent, q_rope, latent_pages, rope_pages, block_table, seq_lens, num_pages, page_size,
                     max_pages_per_seq, batch, n_heads, latent_dim, rope_dim, scale, true, latent_scale, rope_scale,
                     out, lse, stream);
}

const char *kvattn_status_string(int status) {
    switch (status) {
        case KVATTN_OK: return "KVATTN_OK";
        case KVATTN_ERR_INVALID_ARG: return "KVATTN_ERR_INVALID_ARG";
        case KVATTN_ERR_UNSUPPORTED: return "KVATTN_ERR_UNSUPPORTED";
        case KVATTN_ERR_MISALIGNED: return "KVATTN_ERR_MISALIGNED";
        case KVATTN_ERR_CUDA: return "KVATTN_ERR_CUDA";
        case KVATTN_ERR_NO_MEMORY: return "KVATTN_ERR_NO_MEMORY";
        default: return "KVATTN_UNKNOWN_STATUS";
    }
}

const char *kvattn_last_error_detail(void) { return t_detail; }

int kvattn_version(void) { return KVATTN_VERSION; }

void kvattn_release_workspace(void) {
    std::lock_guard<std::mutex> lk(g_mutex);
    int cur = 0;
    if (cudaGetDevice(&cur) != cudaSuccess) return;
    for (int d = 0; d < kMaxDevices; ++d) {
        if (g_dev[d].ws) {
            cudaSetDevice(d);
            cudaDeviceSynchronize();
            cudaFree(g_dev[d].ws);
            g_dev[d].ws = nullptr;
            g_dev[d].ws_bytes = 0;
        }
        if (g_dev[d].aux) {
            cudaSetDevice(d);
            cudaDeviceSynchronize();
            cudaFree(g_dev[d].aux);
            g_dev[d].aux = nullptr;
            g_dev[d].aux_bytes = 0;
        }
    }
    cudaSetDevice(cur);
}

int kvattn_read_device_flags(unsigned int *flags) {
    if (!flags) return KVATTN_ERR_INVALID_ARG;
    cudaError_t e = cudaMemcpyFromSymbol(flags, kvattn::g_device_flags, sizeof(unsigned int));
    if (e != cudaSuccess) return fail_cuda(e, "cudaMemcpyFromSymbol(flags)");
    return KVATTN_OK;
}

int kvattn_clear_device_flags(void) {
    const unsigned int zero = 0;
    cudaError_t e = cudaMemcpyToSymbol(kvattn::g_device_flags, &zero, sizeof(unsigned int));
    if (e != cudaSuccess) return fail_cuda(e, "cudaMemcpyToSymbol(flags)");
    return KVATTN_OK;
}

// ---- test hook: a bounded wait that runs out
namespace kvattn {
// One thread waits, with the kernels' own bounded wait cut to `limit` cycles, for the
// first phase of a shared-memory barrier that nothing arrives on; the wait gives up,
// records FLAG_FULL_WAIT and the kernel returns.
__global__ void wait_probe_kernel(long long limit) {
    __shared__ uint64_t bar;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);
    fence_mbar_init();
    mbar_wait(&bar, 0u, FLAG_FULL_WAIT, nullptr, limit);
}
}  // namespace kvattn

unsigned long long kvattn_kernel_launches(void) { return t_launches; }

int kvattn_debug_wait_probe(int limit_us, void *stream) {
    if (limit_us <= 0 || limit_us > 1000000) return KVATTN_ERR_INVALID_ARG;
    DeviceState *dev = nullptr;
    int st = device_state(&dev);
    if (st != KVATTN_OK) return st;
    int khz = 0;
    cudaError_t e = cudaDeviceGetAttribute(&khz, cudaDevAttrClockRate, dev->id);
    if (e != cudaSuccess) return fail_cuda(e, "cudaDeviceGetAttribute(clock rate)");
    const long long limit = (long long)limit_us * (khz > 0 ? khz : 2000000) / 1000;
    kvattn::wait_probe_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit);
    e = cudaGetLastError();
    if (e != cudaSuccess) return fail_cuda(e, "wait probe launch");
    ++t_launches;
    return KVATTN_OK;
}

// ---- rotary embedding of the new token + cache append
static int launch_rope_append(RopeAppendParams &p, cudaStream_t s, bool kv8 = false) {
    DeviceState *dev = nullptr;
    int st = device_state(&dev);
    if (st != KVATTN_OK) return st;
    const long long total = p.n_q_pairs + p.n_k_pairs + p.n_v_words;
    long long blocks = (total + 255) / 256;
    const long long cap = (long long)dev->sms * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    if (kv8)
        rope_append_kernel<true><<<(unsigned)blocks, 256, 0, s>>>(p);
    else
        rope_append_kernel<false><<<(unsigned)blocks, 256, 0, s>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail_cuda(e, "rope append launch");
    ++t_launches;
    return KVATTN_OK;
}

int kvattn_rope_append(uint16_t *q, const uint16_t *k_new, const uint16_t *v_new, const int32_t *positions,
                       uint16_t *k_cache, uint16_t *v_cache, int max_seq_len, int batch, int n_q_heads,
                       int n_kv_heads, int head_dim, float rope_base, int interleaved, void *stream) {
    if (!q || !k_new || !v_new || !positions || !k_cache || !v_cache) return KVATTN_ERR_INVALID_ARG;
    if (batch <= 0 || n_q_heads <= 0 || n_kv_heads <= 0 || max_seq_len <= 0) return KVATTN_ERR_INVALID_ARG;
    if (n_q_heads % n_kv_heads != 0) return KVATTN_ERR_INVALID_ARG;
    if (head_dim <= 0 || (head_dim & 1) || head_dim > 1024) return KVATTN_ERR_UNSUPPORTED;
    if (!std::isfinite(rope_base) || rope_base <= 0.f) return KVATTN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(positions) ||
        !aligned16(k_cache) || !aligned16(v_cache))
        return KVATTN_ERR_MISALIGNED;
    const size_t q_bytes = (size_t)batch * n_q_heads * head_dim * 2;
    const size_t new_bytes = (size_t)batch * n_kv_heads * head_dim * 2;
    const size_t cache_bytes = (size_t)batch * n_kv_heads * max_seq_len * head_dim * 2;
    const void *w[3] = {q, k_cache, v_cache};
    const size_t wn[3] = {q_bytes, cache_bytes, cache_bytes};
    const void *r[3] = {k_new, v_new, positions};
    const size_t rn[3] = {new_bytes, new_bytes, (size_t)batch * 4};
    for (int i = 0; i < 3; ++i) {
        for (int j = 0; j < 3; ++j)
            if (overlaps(w[i], wn[i], r[j], rn[j])) return KVATTN_ERR_INVALID_ARG;
        for (int j = i + 1; j < 3; ++j)
            if (overlaps(w[i], wn[i], w[j], wn[j])) return KVATTN_ERR_INVALID_ARG;
    }
    RopeAppendParams p = {};
    p.q = reinterpret_cast<__nv_bfloat16 *>(q);
    p.k_new = reinterpret_cast<const __nv_bfloat16 *>(k_new);
    p.v_new = reinterpret_cast<const __nv_bfloat16 *>(v_new);
    p.positions = positions;
    p.k_cache = k_cache;
    p.v_cache = v_cache;
    p.B = batch;
    p.n_q = n_q_heads;
    p.n_kv = n_kv_heads;
    p.dq = p.dk = p.dv = head_dim;
    p.T_max = max_seq_len;
    p.log2_base = std::log2((double)rope_base);
    p.interleaved = interleaved ? 1 : 0;
    p.n_q_pairs = (long long)batch * n_q_heads * (head_dim / 2);
    p.n_k_pairs = (long long)batch * n_kv_heads * (head_dim / 2);
    p.n_v_words = (long long)batch * n_kv_heads * (head_dim / 2);
    return launch_rope_append(p, static_cast<cudaStream_t>(stream));
}

int kvattn_rope_append_fp8(uint16_t *q, const uint16_t *k_new, const uint16_t *v_new, const int32_t *positions,
                           uint8_t *k_cache, uint8_t *v_cache, int max_seq_len, int batch, int n_q_heads,
                           int n_kv_heads, int head_dim, float rope_base, int interleaved, float k_scale,
                           float v_scale, void *stream) {
    if (!q || !k_new || !v_new || !positions || !k_cache || !v_cache) return KVATTN_ERR_INVALID_ARG;
    if (batch <= 0 || n_q_heads <= 0 || n_kv_heads <= 0 || max_seq_len <= 0) return KVATTN_ERR_INVALID_ARG;
    if (n_q_heads % n_kv_heads != 0) return KVATTN_ERR_INVALID_ARG;
    if (head_dim <= 0 || (head_dim & 1) || head_dim > 1024) return KVATTN_ERR_UNSUPPORTED;
    if (!std::isfinite(rope_base) || rope_base <= 0.f) return KVATTN_ERR_INVALID_ARG;
    if (!std::isfinite(k_scale) || !std::isfinite(v_scale) || !(k_scale > 0.f) || !(v_scale > 0.f))
        return KVATTN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(positions) ||
        !aligned16(k_cache) || !aligned16(v_cache))
        return KVATTN_ERR_MISALIGNED;
    const size_t q_bytes = (size_t)batch * n_q_heads * head_dim * 2;
    const size_t new_bytes = (size_t)batch * n_kv_heads * head_dim * 2;
    const size_t cache_bytes = (size_t)batch * n_kv_heads * max_seq_len * head_dim;
    const void *w[3] = {q, k_cache, v_cache};
    const size_t wn[3] = {q_bytes, cache_bytes, cache_bytes};
    const void *r[3] = {k_new, v_new, positions};
    const size_t rn[3] = {new_bytes, new_bytes, (size_t)batch * 4};
    for (int i = 0; i < 3; ++i) {
        for (int j = 0; j < 3; ++j)
            if (overlaps(w[i], wn[i], r[j], rn[j])) return KVATTN_ERR_INVALID_ARG;
        for (int j = i + 1; j < 3; ++j)
            if (overlaps(w[i], wn[i], w[j], wn[j])) return KVATTN_ERR_INVALID_ARG;
    }
    RopeAppendParams p = {};
    p.q = reinterpret_cast<__nv_bfloat16 *>(q);
    p.k_new = reinterpret_cast<const __nv_bfloat16 *>(k_new);
    p.v_new = reinterpret_cast<const __nv_bfloat16 *>(v_new);
    p.positions = positions;
    p.k_cache = k_cache;
    p.v_cache = v_cache;
    p.k_scale = k_scale;
    p.v_scale = v_scale;
    p.B = batch;
    p.n_q = n_q_heads;
    p.n_kv = n_kv_heads;
    p.dq = p.dk = p.dv = head_dim;
    p.T_max = max_seq_len;
    p.log2_base = std::log2((double)rope_base);
    p.interleaved = interleaved ? 1 : 0;
    p.n_q_pairs = (long long)batch * n_q_heads * (head_dim / 2);
    p.n_k_pairs = (long long)batch * n_kv_heads * (head_dim / 2);
    p.n_v_words = (long long)batch * n_kv_heads * (head_dim / 2);
    return launch_rope_append(p, static_cast<cudaStream_t>(stream), true);
}

static int mla_append(uint16_t *q_rope, const uint16_t *latent_new, const uint16_t *rope_new,
                      const int32_t *positions, void *latent_cache, void *rope_cache, int max_seq_len, int batch,
                      int n_heads, int latent_dim, int rope_dim, float rope_base, int interleaved, bool e4m3,
                      float latent_scale, float rope_scale, void *stream) {
    if (!q_rope || !latent_new || !rope_new || !positions || !latent_cache || !rope_cache)
        return KVATTN_ERR_INVALID_ARG;
    if (batch <= 0 || n_heads <= 0 || max_seq_len <= 0 || latent_dim <= 0 || rope_dim <= 0)
        return KVATTN_ERR_INVALID_ARG;
    if ((rope_dim & 1) || (latent_dim & 1) || rope_dim > 1024 || latent_dim > 4096) return KVATTN_ERR_UNSUPPORTED;
    if (!std::isfinite(rope_base) || rope_base <= 0.f) return KVATTN_ERR_INVALID_ARG;
    if (e4m3 && (!std::isfinite(latent_scale) || !std::isfinite(rope_scale) || !(latent_scale > 0.f) ||
                 !(rope_scale > 0.f)))
        return KVATTN_ERR_INVALID_ARG;
    const size_t cb = e4m3 ? 1 : 2;
    if (!aligned16(q_rope) || !aligned16(latent_new) || !aligned16(rope_new) || !aligned16(positions) ||
        !aligned16(latent_cache) || !aligned16(rope_cache))
        return KVATTN_ERR_MISALIGNED;
    const void *w[3] = {q_rope, latent_cache, rope_cache};
    const size_t wn[3] = {(size_t)batch * n_heads * rope_dim * 2, (size_t)batch * max_seq_len * latent_dim * cb,
                          (size_t)batch * max_seq_len * rope_dim * cb};
    const void *r[3] = {latent_new, rope_new, positions};
    const size_t rn[3] = {(size_t)batch * latent_dim * 2, (size_t)batch * rope_dim * 2, (size_t)batch * 4};
    for (int i = 0; i < 3; ++i) {
        for (int j = 0; j < 3; ++j)
            if (overlaps(w[i], wn[i], r[j], rn[j])) return KVATTN_ERR_INVALID_ARG;
        for (int j = i + 1; j < 3; ++j)
            if (overlaps(w[i], wn[i], w[j], wn[j])) return KVATTN_ERR_INVALID_ARG;
    }
    RopeAppendParams p = {};
    p.q = reinterpret_cast<__nv_bfloat16 *>(q_rope);
    p.k_new = reinterpret_cast<const __nv_bfloat16 *>(rope_new);
    p.v_new = reinterpret_cast<const __nv_bfloat16 *>(latent_new);
    p.positions = positions;
    p.k_cache = rope_cache;
    p.v_cache = latent_cache;
    p.k_scale = e4m3 ? rope_scale : 1.f;
    p.v_scale = e4m3 ? latent_scale : 1.f;
    p.B = batch;
    p.n_q = n_heads;
    p.n_kv = 1;                    // one shared latent / rotary key per token
    p.dq = p.dk = rope_dim;
    p.dv = latent_dim;
    p.T_max = max_seq_len;
    p.log2_base = std::log2((double)rope_base);
    p.interleaved = interleaved ? 1 : 0;
    p.n_q_pairs = (long long)batch * n_heads * (rope_dim / 2);
    p.n_k_pairs = (long long)batch * (rope_dim / 2);
    p.n_v_words = (long long)batch * (latent_dim / 2);
    return launch_rope_append(p, static_cast<cudaStream_t>(stream), e4m3);
}

int kvattn_mla_rope_append(uint16_t *q_rope, const uint16_t *latent_new, const uint16_t *rope_new,
                           const int32_t *positions, uint16_t *latent_cache, uint16_t *rope_cache,
                           int max_seq_len, int batch, int n_heads, int latent_dim, int rope_dim,
                           float rope_base, int interleaved, void *stream) {
    return mla_append(q_rope, latent_new, rope_new, positions, latent_cache, rope_cache, max_seq_len, batch, n_heads,
                      latent_dim, rope_dim, rope_base, interleaved, false, 1.f, 1.f, stream);
}

int kvattn_mla_rope_append_fp8(uint16_t *q_rope, const uint16_t *latent_new, const uint16_t *rope_new,
                               const int32_t *positions, uint8_t *latent_cache, uint8_t *rope_cache,
                               int max_seq_len, int batch, int n_heads, int latent_dim, int rope_dim,
                               float rope_base, int interleaved, float latent_scale, float rope_scale,
                               void *stream) {
    return mla_append(q_rope, latent_new, rope_new, positions, latent_cache, rope_cache, max_seq_len, batch, n_heads,
                      latent_dim, rope_dim, rope_base, interleaved, true, latent_scale, rope_scale, stream);
}

void kvattn_debug_set_workers(int workers, int min_tiles) {
    std::lock_guard<std::mutex> lk(g_mutex);
    g_force_workers = workers > 0 ? workers : 0;
    g_force_min_tiles = workers > 0 && min_tiles > 0 ? min_tiles : 0;
}

void kvattn_debug_set_gqa_kernel(int which) {
    std::lock_guard<std::mutex> lk(g_mutex);
    g_gqa_kernel = (which == 1 || which == 2) ? which : 0;
}

}  // extern "C"


// Decode without any allocation by the library: kvattn_gqa_decode's checks and code path
// with the warp-level kernel and the static scratch above.
extern "C" int kvattn_gqa_decode_noalloc(const uint16_t *q, const uint16_t *k_cache,
                                         const uint16_t *v_cache, const int32_t *seq_lens,
                                         int max_seq_len, int batch, int n_q_heads, int n_kv_heads,
                                         int head_dim, float scale, float *out, float *lse,
                                         void *stream) {
    const int st = check_gqa_args(q, k_cache, v_cache, seq_lens, max_seq_len, batch, n_q_heads, n_kv_heads,
                                  head_dim, scale, out, lse);
    if (st != KVATTN_OK) return st;
    const GqaCache cache{k_cache, v_cache, nullptr, max_seq_len, max_seq_len, 1, batch};
    return gqa_decode_impl(q, cache, seq_lens, batch, n_q_heads, n_kv_heads, head_dim, scale, out, lse, stream,
                           1, 0, true);
}
