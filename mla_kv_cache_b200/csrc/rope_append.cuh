// rope_append.cuh -- the step either side of the decode kernels: rotary position
// embedding of the new token's query and key, and the append of its key and value
// (or, for MLA, its latent and rotary key) to the cache at the token's position.
//
// What it computes: the pages apply RoPE to queries and keys before they meet the cache
// and append the new token's entry before attending ("Attention variants: MQA, GQA, and
// MLA", section "MLA: cache a latent, not the keys and values": the decoupled rotary
// key is cached alongside the latent; the new token is written to the cache, then
// attended to).  They do not write the rotation out, so it is the textbook one: pair i
// of a d-wide vector at position p turns by theta_i = p * base^(-2i/d), with the pairs
// (2i, 2i+1) (interleaved) or (i, i + d/2) (split halves).
//
// One thread per feature pair (rotations) or per 4-byte word (copies).  The angle is
// formed and reduced in fp64 (positions reach tens of thousands of radians, where an
// fp32 angle would be off by ~1e-3), then the pair is turned in fp32 and rounded to
// bf16 once.  A position outside [0, T_max) is not written into the cache (the query
// is still rotated with it).  For an E4M3 cache (KV8) the rotated key and the value are
// divided by their tensor's scale in fp32 (correctly rounded) and stored as the nearest
// E4M3 codes (ties to even, magnitudes past 448 saturated): the cached value is code *
// scale, as the decode reads it.
#pragma once
#include "common.cuh"

namespace kvattn {

struct RopeAppendParams {
    __nv_bfloat16 *q;              // [B, n_q, dq]: rotated in place (null: none)
    const __nv_bfloat16 *k_new;    // [B, n_kv, dk]: rotated into k_cache
    const __nv_bfloat16 *v_new;    // [B, n_kv, dv]: copied into v_cache (null: none)
    const int32_t *positions;      // [B]
    void *k_cache;                 // [B, n_kv, T_max, dk] bf16, or E4M3 codes (KV8)
    void *v_cache;                 // [B, n_kv, T_max, dv] bf16, or E4M3 codes (KV8)
    float k_scale, v_scale;        // E4M3 cache: value = code * scale
    int B, n_q, n_kv, dq, dk, dv, T_max;
    double log2_base;
    int interleaved;
    long long n_q_pairs, n_k_pairs, n_v_words;   // work items of the three parts
};

// Turns the pair (a, b) of row `row` (d features) at position p; returns the two
// rotated values.
__device__ __forceinline__ void rope_pair(const __nv_bfloat16 *row, int d, int i, int p, double log2_base,
                                          int interleaved, int &ia, int &ib, float &ya, float &yb) {
    const int half = d >> 1;
    ia = interleaved ? 2 * i : i;
    ib = interleaved ? 2 * i + 1 : i + half;
    const double theta = (double)p * exp2(-2.0 * (double)i / (double)d * log2_base);
    double s, c;
    sincos(theta, &s, &c);
    const float xa = __bfloat162float(row[ia]), xb = __bfloat162float(row[ib]);
    const float cf = (float)c, sf = (float)s;
    ya = fmaf(xa, cf, -xb * sf);
    yb = fmaf(xa, sf, xb * cf);
}

template <bool KV8>
__global__ void __launch_bounds__(256) rope_append_kernel(const RopeAppendParams p) {
    const long long total = p.n_q_pairs + p.n_k_pairs + p.n_v_words;
    for (long long w = (long long)blockIdx.x * blockDim.x + threadIdx.x; w < total;
         w += (long long)gridDim.x * blockDim.x) {
        if (w < p.n_q_pairs) {
            // ---- query: in place
            const int hp = p.dq >> 1;
            const long long row = w / hp;
            const int i = (int)(w % hp);
            const int b = (int)(row / p.n_q);
            __nv_bfloat16 *x = p.q + row * p.dq;
            int ia, ib;
            float ya, yb;
            rope_pair(x, p.dq, i, __ldg(p.positions + b), p.log2_base, p.interleaved, ia, ib, ya, yb);
            x[ia] = __float2bfloat16_rn(ya);
            x[ib] = __float2bfloat16_rn(yb);
        } else if (w < p.n_q_pairs + p.n_k_pairs) {
            // ---- key: rotated into the cache row of the new position
            const long long u = w - p.n_q_pairs;
            const int hp = p.dk >> 1;
            const long long row = u / hp;            // b * n_kv + j
            const int i = (int)(u % hp);
            const int b = (int)(row / p.n_kv);
            const int pos = __ldg(p.positions + b);
            if (pos < 0 || pos >= p.T_max) continue;
            int ia, ib;
            float ya, yb;
            rope_pair(p.k_new + row * p.dk, p.dk, i, pos, p.log2_base, p.interleaved, ia, ib, ya, yb);
            const long long base = (row * p.T_max + pos) * p.dk;
            if constexpr (KV8) {
                uint8_t *dst = static_cast<uint8_t *>(p.k_cache) + base;
                dst[ia] = __nv_cvt_float_to_fp8(__fdiv_rn(ya, p.k_scale), __NV_SATFINITE, __NV_E4M3);
                dst[ib] = __nv_cvt_float_to_fp8(__fdiv_rn(yb, p.k_scale), __NV_SATFINITE, __NV_E4M3);
            } else {
                __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(p.k_cache) + base;
                dst[ia] = __float2bfloat16_rn(ya);
                dst[ib] = __float2bfloat16_rn(yb);
            }
        } else {
            // ---- value (or latent): copied into the cache row, one 4-byte word each
            const long long u = w - p.n_q_pairs - p.n_k_pairs;
            const int wpr = p.dv >> 1;
            const long long row = u / wpr;
            const int c = (int)(u % wpr);
            const int b = (int)(row / p.n_kv);
            const int pos = __ldg(p.positions + b);
            if (pos < 0 || pos >= p.T_max) continue;
            const uint32_t *src = reinterpret_cast<const uint32_t *>(p.v_new + row * p.dv);
            const long long base = (row * p.T_max + pos) * p.dv;
            if constexpr (KV8) {
                // two values: bf16 pair -> two E4M3 codes (element order kept)
                const uint32_t w2 = __ldg(src + c);
                const float2 x = make_float2(__fdiv_rn(__uint_as_float(w2 << 16), p.v_scale),
                                             __fdiv_rn(__uint_as_float(w2 & 0xFFFF0000u), p.v_scale));
                *reinterpret_cast<__nv_fp8x2_storage_t *>(static_cast<uint8_t *>(p.v_cache) + base + 2 * c) =
                    __nv_cvt_float2_to_fp8x2(x, __NV_SATFINITE, __NV_E4M3);
            } else {
                uint32_t *dst = reinterpret_cast<uint32_t *>(static_cast<__nv_bfloat16 *>(p.v_cache) + base);
                dst[c] = __ldg(src + c);
            }
        }
    }
}

}  // namespace kvattn
