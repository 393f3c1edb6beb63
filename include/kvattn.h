/*
 * kvattn.h -- C ABI of the kvattn decode-attention library (NVIDIA B200, sm_100a).
 *
 * One decode step of attention for a batch of sequences: every sequence contributes
 * one query token, which attends to all of that sequence's cached keys and values.
 * Two forms share the library:
 *
 *  - kvattn_gqa_decode: multi-head (MHA), grouped-query (GQA) and multi-query (MQA)
 *    attention.  n_kv_heads KV heads are each shared by a group of
 *    g = n_q_heads / n_kv_heads consecutive query heads; query head h reads KV head
 *    h / g.  ("Attention variants: MQA, GQA, and MLA", sections "MQA: one KV head for
 *    everyone" and "GQA: interpolating with groups"; "Grouped-Query Attention: Fewer
 *    KV Heads, Same Quality", section "Writing the formula explicitly", where the
 *    1-based group index ceil(i * n_kv / n_q) is this h / g with 0-based indices.)
 *
 *  - kvattn_mla_decode: absorbed multi-head latent attention.  The key up-projection
 *    is already folded into the query, every head scores the one cached latent per
 *    token plus a decoupled RoPE key, and the output stays in latent space (the
 *    value up-projection is applied by the caller).  ("Attention variants: MQA, GQA,
 *    and MLA", section "MLA: cache a latent, not the keys and values".)
 *
 * For each sequence b and query head h, with T = seq_lens[b] and scaled scores
 * s_t (t < T), both entry points write
 *      out[b, h, :] = sum_t softmax(s)_t * value_t       (fp32)
 *      lse[b, h]    = log(sum_t exp(s_t))                 (fp32, natural log)
 * An empty sequence (T == 0) gives out = 0 and lse = -inf.
 *
 * Conventions for every entry point:
 *  - Pointers marked "device" must point to memory of the device that is current on
 *    the calling host thread; "host" pointers to host memory.  The library never
 *    frees, retains or reallocates caller memory.
 *  - bf16 data is passed as uint16_t bit patterns (IEEE bfloat16).
 *  - All arrays are dense and row-major in the shape given (last index fastest).
 *  - Every device pointer must be 16-byte aligned (else KVATTN_ERR_MISALIGNED).
 *  - out and lse are fully overwritten and must not overlap any input.
 *  - stream is a cudaStream_t (NULL = the legacy default stream).  The call only
 *    enqueues work: KVATTN_OK means the kernels were launched; their completion is
 *    observed through the stream.  Arguments are checked on the host before any work
 *    is enqueued; an argument error launches nothing.
 *  - Functions never throw or abort; they return a kvattn_status.
 *  - Scratch memory: the library keeps one workspace per device, grown with
 *    cudaMalloc when a call needs more than it holds and kept until
 *    kvattn_release_workspace().  A call that grows it is not capturable in a CUDA
 *    graph; issue one call of the largest shape before capturing.  A captured decode
 *    call may be replayed any number of times: its kernels derive the work split from
 *    the device-side seq_lens at every launch, so the lengths (not the shapes or
 *    pointers) may change between replays.  Calls that share a device must be ordered
 *    (same stream, or synchronised): they share the workspace.
 *  - Thread safety: entry points may be called from several host threads; the
 *    workspace is guarded by a mutex, but see the ordering rule above.
 */
#ifndef KVATTN_H
#define KVATTN_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define KVATTN_VERSION 10000 /* major * 10000 + minor * 100 + patch */

typedef enum {
    KVATTN_OK = 0,
    KVATTN_ERR_INVALID_ARG = 1, /* null pointer, non-positive size, n_q % n_kv != 0, non-finite scale, overlap */
    KVATTN_ERR_UNSUPPORTED = 2, /* valid but not implemented: head_dim, latent/rope width, size limits */
    KVATTN_ERR_MISALIGNED = 3,  /* a pointer is not 16-byte aligned */
    KVATTN_ERR_CUDA = 4,        /* a CUDA runtime call failed (see kvattn_last_error_detail) */
    KVATTN_ERR_NO_MEMORY = 5    /* the workspace could not be allocated */
} kvattn_status;

/*
 * GQA / MQA / MHA decode.
 *   q         device bf16 [batch, n_q_heads, head_dim]   one query token per sequence
 *   k_cache   device bf16 [batch, n_kv_heads, max_seq_len, head_dim]
 *   v_cache   device bf16 [batch, n_kv_heads, max_seq_len, head_dim]
 *             (the pages' cache layout (batch, kv_heads, seq, head_dim), "The KV cache
 *             bill, worked numerically"; positions >= seq_lens[b] are never read)
 *   seq_lens  device int32 [batch]   tokens cached for each sequence, 0..max_seq_len;
 *             values outside that range are clamped on the device (the result for such
 *             a sequence is then unspecified, but no memory outside the caches is read)
 *   max_seq_len  cache capacity per sequence (the T stride of the caches), >= 1
 *   batch, n_q_heads, n_kv_heads   > 0, n_q_heads % n_kv_heads == 0, batch <= 4096
 *   head_dim  64 or 128 (others: KVATTN_ERR_UNSUPPORTED)
 *   scale     finite score scale (the pages use 1/sqrt(head_dim))
 *   out       device fp32 [batch, n_q_heads, head_dim]
 *   lse       device fp32 [batch, n_q_heads]  (required, natural log)
 *   stream    cudaStream_t
 * Limits: batch * n_kv_heads * max_seq_len < 2^31.
 */
int kvattn_gqa_decode(const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                      const int32_t *seq_lens, int max_seq_len, int batch, int n_q_heads,
                      int n_kv_heads, int head_dim, float scale, float *out, float *lse,
                      void *stream);

/*
 * Absorbed MLA decode (DeepSeek shape: latent_dim 512, rope_dim 64).
 *   q_latent      device bf16 [batch, n_heads, latent_dim]  queries already multiplied
 *                 by the key up-projection (they score the latents directly)
 *   q_rope        device bf16 [batch, n_heads, rope_dim]    rotated decoupled-RoPE queries
 *   latent_cache  device bf16 [batch, max_seq_len, latent_dim]  one latent per token,
 *                 shared by all heads; it is both key (with the RoPE part) and value
 *   rope_cache    device bf16 [batch, max_seq_len, rope_dim]    rotated RoPE keys
 *   seq_lens      device int32 [batch], as for kvattn_gqa_decode
 *   max_seq_len   cache capacity per sequence, >= 1
 *   batch         > 0, <= 1024;  n_heads 1..128
 *   latent_dim    512;  rope_dim 64 (others: KVATTN_ERR_UNSUPPORTED)
 *   scale         finite score scale (DeepSeek: 1/sqrt(128 + 64))
 *   out           device fp32 [batch, n_heads, latent_dim]  (latent space)
 *   lse           device fp32 [batch, n_heads]
 * Score of head h at token t: scale * (q_latent[h] . latent_t + q_rope[h] . rope_t).
 * Every bf16 value is accepted as is (no narrower intermediate format): the weights
 * enter the value product as a bf16 high part plus a bf16 remainder.
 */
int kvattn_mla_decode(const uint16_t *q_latent, const uint16_t *q_rope,
                      const uint16_t *latent_cache, const uint16_t *rope_cache,
                      const int32_t *seq_lens, int max_seq_len, int batch, int n_heads,
                      int latent_dim, int rope_dim, float scale, float *out, float *lse,
                      void *stream);

/*
 * Several new tokens per sequence in one call (multi-token decode: verifying drafted
 * tokens, or a short prompt continuation), with the causal mask of "Attention variants:
 * MQA, GQA, and MLA", section "Implementation, twice" (a query never sees a later
 * token), and optionally a sliding window (the Mistral-style window named in
 * "Grouped-Query Attention: Fewer KV Heads, Same Quality").
 *   q         device bf16 [batch, q_len, n_q_heads, head_dim]: the q_len newest tokens'
 *             queries, oldest first
 *   k_cache, v_cache, seq_lens, max_seq_len: as for kvattn_gqa_decode; the cache already
 *             holds the q_len new tokens at positions seq_lens[b] - q_len .. seq_lens[b] - 1
 *   window    0: no window; w > 0: query i, at position p = seq_lens[b] - q_len + i,
 *             attends to positions p - w < t <= p only (its last w tokens, itself included);
 *             otherwise to all t <= p.  Tiles wholly before the earliest visible position
 *             are not read.
 *   out       device fp32 [batch, q_len, n_q_heads, head_dim];  lse fp32 [batch, q_len, n_q_heads]
 * A query with no visible position (p < 0) gets out = 0 and lse = -inf.  q_len == 1 and
 * window == 0 is exactly kvattn_gqa_decode.  head_dim 64 or 128; a window needs head_dim
 * 128 and n_q_heads / n_kv_heads <= 64; batch * q_len <= 4096 (KVATTN_ERR_UNSUPPORTED
 * otherwise).  With head_dim 128 and (n_q_heads / n_kv_heads) * q_len <= 64 one kernel
 * scores a group's heads at all q_len positions against each cache tile; otherwise the
 * call runs as batch * q_len single-token sequences (query i of sequence b is a sequence
 * of length seq_lens[b] - q_len + 1 + i over b's cache rows), which reads the cache once
 * per new token (the repeats mostly from L2).
 */
int kvattn_gqa_decode_multi(const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                            const int32_t *seq_lens, int max_seq_len, int batch, int q_len,
                            int n_q_heads, int n_kv_heads, int head_dim, float scale, int window,
                            float *out, float *lse, void *stream);

/*
 * Decode over a quantised (fp8) KV cache.  The pages list quantised caches among what the
 * libraries build around the attention module ("Attention variants: MQA, GQA, and MLA",
 * section "Against the real libraries"); at one byte per cached value the cache a decode
 * step reads halves.  The format is E4M3 (1 sign, 4 exponent bits with bias 7, 3
 * mantissa bits; largest finite magnitude 448; codes 0x7F / 0xFF are NaN) with one
 * float scale per cache tensor: the cached key is value(code) * k_scale, the value
 * value(code) * v_scale.  The result is attention on those dequantised values, as
 * kvattn_gqa_decode_multi computes it (q_len = 1, window = 0: kvattn_gqa_decode).
 *   q           device bf16 [batch, q_len, n_q_heads, head_dim]
 *   k_cache, v_cache  device E4M3 codes (one byte each)
 *               [batch, n_kv_heads, max_seq_len, head_dim]
 *   k_scale, v_scale  finite, > 0
 *   out, lse    device fp32 [batch, q_len, n_q_heads, head_dim], [batch, q_len, n_q_heads]
 * head_dim must be 128 and n_q_heads / n_kv_heads <= 64 (else KVATTN_ERR_UNSUPPORTED);
 * everything else as for kvattn_gqa_decode_multi.  The query
 * and the softmax weights enter the tensor-core products as two E4M3 parts each (~8
 * significant bits), the codes exactly; accumulation is fp32.  Codes past a sequence's
 * length are never read.
 */
int kvattn_gqa_decode_fp8(const uint16_t *q, const uint8_t *k_cache, const uint8_t *v_cache,
                          const int32_t *seq_lens, int max_seq_len, int batch, int q_len,
                          int n_q_heads, int n_kv_heads, int head_dim, float scale, float k_scale,
                          float v_scale, int window, float *out, float *lse, void *stream);

/*
 * kvattn_gqa_decode_fp8 for one new token per sequence over a paged E4M3 cache:
 * k_pages, v_pages [num_pages, n_kv_heads, page_size, head_dim] codes, block_table and
 * seq_lens as for kvattn_gqa_decode_paged, page_size a multiple of 128; q [batch,
 * n_q_heads, head_dim] bf16, out [batch, n_q_heads, head_dim], lse [batch, n_q_heads].
 */
int kvattn_gqa_decode_fp8_paged(const uint16_t *q, const uint8_t *k_pages, const uint8_t *v_pages,
                                const int32_t *block_table, const int32_t *seq_lens, int num_pages,
                                int page_size, int max_pages_per_seq, int batch, int n_q_heads,
                                int n_kv_heads, int head_dim, float scale, float k_scale, float v_scale,
                                float *out, float *lse, void *stream);

/*
 * kvattn_mla_decode over an E4M3 (fp8) latent cache, the MLA form of
 * kvattn_gqa_decode_fp8 (same format; the pages list quantised caches among what the
 * libraries add, "Attention variants: MQA, GQA, and MLA", section "Against the real
 * libraries").  The cached latent of token t is value(latent_cache[b, t, :]) *
 * latent_scale -- the key's latent part and the value alike -- and its RoPE key
 * value(rope_cache[b, t, :]) * rope_scale; the result is kvattn_mla_decode on those
 * dequantised rows.
 *   q_latent, q_rope  device bf16 [batch, n_heads, 512], [batch, n_heads, 64]
 *   latent_cache, rope_cache  device E4M3 codes [batch, max_seq_len, 512],
 *                     [batch, max_seq_len, 64] (one byte each)
 *   latent_scale, rope_scale  finite, > 0
 *   out, lse    device fp32 [batch, n_heads, 512], [batch, n_heads]
 * Everything else, the results' layout and the errors as for kvattn_mla_decode.  The
 * query (each head's, after scaling by a power of two that puts its largest magnitude in
 * [128, 256)) and the softmax weights enter the tensor-core products as an E4M3 high part
 * plus an E4M3 remainder (~8 significant bits), the codes exactly; accumulation is fp32.
 * Codes past a sequence's length are never read.
 */
int kvattn_mla_decode_fp8(const uint16_t *q_latent, const uint16_t *q_rope, const uint8_t *latent_cache,
                          const uint8_t *rope_cache, const int32_t *seq_lens, int max_seq_len, int batch,
                          int n_heads, int latent_dim, int rope_dim, float scale, float latent_scale,
                          float rope_scale, float *out, float *lse, void *stream);

/*
 * Several new tokens per sequence for absorbed MLA (the causal mask as for
 * kvattn_gqa_decode_multi; no window): query i of sequence b, at position
 * p = seq_lens[b] - q_len + i, attends to the cached tokens t <= p.
 *   q_latent, q_rope  device bf16 [batch, q_len, n_heads, 512], [batch, q_len, n_heads, 64]
 *   latent_cache, rope_cache  device [batch, max_seq_len, 512], [batch, max_seq_len, 64]:
 *             bf16 (e4m3 == 0) or E4M3 codes with latent_scale / rope_scale as for
 *             kvattn_mla_decode_fp8 (e4m3 != 0; the scales are ignored otherwise)
 *   out, lse  device fp32 [batch, q_len, n_heads, 512], [batch, q_len, n_heads]
 * A query with no visible position gets out = 0 and lse = -inf.  batch * q_len <= 1024.
 * The call runs as batch * q_len single-token sequences over b's cache rows (the cache
 * read once per new token, the repeats mostly from L2); q_len == 1 is kvattn_mla_decode
 * (kvattn_mla_decode_fp8).  Everything else as for kvattn_mla_decode.
 */
int kvattn_mla_decode_multi(const uint16_t *q_latent, const uint16_t *q_rope, const void *latent_cache,
                            const void *rope_cache, const int32_t *seq_lens, int max_seq_len, int batch, int q_len,
                            int n_heads, int latent_dim, int rope_dim, float scale, int e4m3, float latent_scale,
                            float rope_scale, float *out, float *lse, void *stream);

/*
 * kvattn_mla_decode_fp8 over a paged cache: latent_pages [num_pages, page_size, 512] and
 * rope_pages [num_pages, page_size, 64] E4M3 codes, block_table and seq_lens as for
 * kvattn_gqa_decode_paged, page_size a multiple of 64.
 */
int kvattn_mla_decode_fp8_paged(const uint16_t *q_latent, const uint16_t *q_rope, const uint8_t *latent_pages,
                                const uint8_t *rope_pages, const int32_t *block_table, const int32_t *seq_lens,
                                int num_pages, int page_size, int max_pages_per_seq, int batch, int n_heads,
                                int latent_dim, int rope_dim, float scale, float latent_scale, float rope_scale,
                                float *out, float *lse, void *stream);

/*
 * kvattn_gqa_decode over a paged KV cache: the cache is a pool of pages and each
 * sequence lists its pages in a block table (the serving-engine layout the pages name,
 * "Attention variants: MQA, GQA, and MLA", section "Against the real libraries": vLLM's
 * PagedAttention).  Token t of sequence b lives in page block_table[b][t / page_size],
 * row t % page_size.
 *   k_pages, v_pages  device bf16 [num_pages, n_kv_heads, page_size, head_dim]
 *   block_table       device int32 [batch, max_pages_per_seq]: physical page of each
 *                     logical page; entries past a sequence's last page are not read.
 *                     Every entry that is read must lie in [0, num_pages).
 *   seq_lens          device int32 [batch], 0 <= len <= max_pages_per_seq * page_size
 *   page_size         a multiple of 64 (the tensor-core kernel for groups of >= 4 heads
 *                     runs when it is a multiple of 128; otherwise the warp-level kernel)
 * Everything else, the results and the errors are those of kvattn_gqa_decode.  Rows
 * of a sequence's last page past its length are never read.
 */
int kvattn_gqa_decode_paged(const uint16_t *q, const uint16_t *k_pages, const uint16_t *v_pages,
                            const int32_t *block_table, const int32_t *seq_lens, int num_pages,
                            int page_size, int max_pages_per_seq, int batch, int n_q_heads,
                            int n_kv_heads, int head_dim, float scale, float *out, float *lse,
                            void *stream);

/*
 * kvattn_mla_decode over a paged latent cache: latent_pages [num_pages, page_size,
 * latent_dim] and rope_pages [num_pages, page_size, rope_dim] bf16, block_table and
 * seq_lens as for kvattn_gqa_decode_paged; page_size a multiple of 64.  Everything else
 * as for kvattn_mla_decode.
 */
int kvattn_mla_decode_paged(const uint16_t *q_latent, const uint16_t *q_rope,
                            const uint16_t *latent_pages, const uint16_t *rope_pages,
                            const int32_t *block_table, const int32_t *seq_lens, int num_pages,
                            int page_size, int max_pages_per_seq, int batch, int n_heads,
                            int latent_dim, int rope_dim, float scale, float *out, float *lse,
                            void *stream);

/*
 * The step either side of the decode: rotary position embedding (RoPE) of the new
 * token's query and key, and the append of its key and value to the cache at its
 * position.  The pages rotate queries and keys before they meet the cache and write the
 * new token to the cache before attending ("Attention variants: MQA, GQA, and MLA",
 * section "MLA: cache a latent, not the keys and values"); the rotation itself is the
 * textbook one: pair i of a head_dim-wide vector at position p turns by the angle
 * p * rope_base^(-2i / head_dim), the pairs being (2i, 2i+1) when interleaved != 0 and
 * (i, i + head_dim/2) otherwise.  The angle is formed in fp64; results are rounded to
 * bf16 once.
 *   q          device bf16 [batch, n_q_heads, head_dim]: rotated in place
 *   k_new      device bf16 [batch, n_kv_heads, head_dim]: the new token's keys (not
 *              rotated); their rotation goes to k_cache[b, j, positions[b], :]
 *   v_new      device bf16 [batch, n_kv_heads, head_dim]: copied to
 *              v_cache[b, j, positions[b], :]
 *   positions  device int32 [batch]: the new token's position (its index in the cache).
 *              A position outside [0, max_seq_len) writes nothing into the caches (q is
 *              still rotated with it).  The caller's seq_lens for the following decode
 *              are positions + 1.
 *   k_cache, v_cache  device bf16 [batch, n_kv_heads, max_seq_len, head_dim]
 *   head_dim   even, <= 1024;  rope_base > 0 and finite (e.g. 10000)
 * Errors as for kvattn_gqa_decode; q and the caches must not overlap each other or the
 * inputs.  Asynchronous on `stream`.
 */
int kvattn_rope_append(uint16_t *q, const uint16_t *k_new, const uint16_t *v_new,
                       const int32_t *positions, uint16_t *k_cache, uint16_t *v_cache,
                       int max_seq_len, int batch, int n_q_heads, int n_kv_heads, int head_dim,
                       float rope_base, int interleaved, void *stream);

/*
 * kvattn_rope_append into an E4M3 (fp8) cache, the producer side of
 * kvattn_gqa_decode_fp8: q is rotated in place (bf16) as above; the new token's rotated
 * key is stored as E4M3 codes of key / k_scale and its value as codes of value /
 * v_scale (the quotient taken in fp32, correctly rounded; the nearest code, ties to
 * even, magnitudes past 448 saturated to +-448, NaN to the NaN code), so that the
 * cached value is code * scale as the decode reads it.
 *   k_cache, v_cache  device E4M3 codes [batch, n_kv_heads, max_seq_len, head_dim]
 *   k_scale, v_scale  finite, > 0 (the scales the cache was quantised with)
 * Everything else, including positions outside the cache, as for kvattn_rope_append.
 */
int kvattn_rope_append_fp8(uint16_t *q, const uint16_t *k_new, const uint16_t *v_new,
                           const int32_t *positions, uint8_t *k_cache, uint8_t *v_cache,
                           int max_seq_len, int batch, int n_q_heads, int n_kv_heads, int head_dim,
                           float rope_base, int interleaved, float k_scale, float v_scale,
                           void *stream);

/*
 * The same for absorbed MLA: q_rope [batch, n_heads, rope_dim] is rotated in place, the
 * new token's decoupled rotary key rope_new [batch, rope_dim] is rotated into
 * rope_cache[b, positions[b], :], and its latent latent_new [batch, latent_dim] is
 * copied (unrotated: the latent carries no position) into latent_cache[b, positions[b], :]
 * ("Attention variants: MQA, GQA, and MLA", section "MLA: cache a latent, not the keys
 * and values").  latent_dim and rope_dim even; the rest as for kvattn_rope_append.
 */
int kvattn_mla_rope_append(uint16_t *q_rope, const uint16_t *latent_new, const uint16_t *rope_new,
                           const int32_t *positions, uint16_t *latent_cache, uint16_t *rope_cache,
                           int max_seq_len, int batch, int n_heads, int latent_dim, int rope_dim,
                           float rope_base, int interleaved, void *stream);

/*
 * kvattn_mla_rope_append into an E4M3 cache, the producer side of kvattn_mla_decode_fp8:
 * q_rope is rotated in place (bf16); the rotated RoPE key is stored as E4M3 codes of
 * key / rope_scale and the latent as codes of latent / latent_scale (the quotient taken
 * in fp32, correctly rounded; nearest code, ties to even, saturated at 448, NaN to the
 * NaN code), as kvattn_rope_append_fp8 encodes.
 *   latent_cache, rope_cache  device E4M3 codes [batch, max_seq_len, latent_dim],
 *                             [batch, max_seq_len, rope_dim]
 *   latent_scale, rope_scale  finite, > 0
 * Everything else as for kvattn_mla_rope_append.
 */
int kvattn_mla_rope_append_fp8(uint16_t *q_rope, const uint16_t *latent_new, const uint16_t *rope_new,
                               const int32_t *positions, uint8_t *latent_cache, uint8_t *rope_cache,
                               int max_seq_len, int batch, int n_heads, int latent_dim, int rope_dim,
                               float rope_base, int interleaved, float latent_scale, float rope_scale,
                               void *stream);

/* Human-readable name of a kvattn_status value (static string, never NULL). */
const char *kvattn_status_string(int status);

/* Detail of the last KVATTN_ERR_CUDA / KVATTN_ERR_NO_MEMORY on this host thread. */
const char *kvattn_last_error_detail(void);

/* KVATTN_VERSION of the loaded library. */
int kvattn_version(void);

/* Frees the workspace of every device (waits for that device to be idle first). */
void kvattn_release_workspace(void);

/*
 * Device-side error flags of the current device.  Every wait inside the kernels is
 * bounded; a wait that runs out sets a bit here and the kernel returns early (its
 * output is then invalid).  Bit 0: pipeline data wait, bit 1: pipeline slot wait,
 * bit 2: cluster peer wait, bit 3: tensor-core completion wait.  Reading synchronises
 * the device.  Returns a kvattn_status; *flags receives the bits.
 */
int kvattn_read_device_flags(unsigned int *flags);
int kvattn_clear_device_flags(void);

/*
 * Kernels this library has launched (enqueued successfully) from the calling host thread
 * since the library was loaded: a decode call adds one (the decode kernel), or two when a
 * combine kernel merges units cut between workers, plus one when several new tokens run
 * as a virtual batch; an append adds one.  Read it before and after a call to count that
 * call's kernels.
 */
unsigned long long kvattn_kernel_launches(void);

/*
 * Test hook for the bounded waits: launches one CTA on `stream` (a cudaStream_t, NULL:
 * the default stream) whose thread waits, with the same bounded wait the kernels use but
 * cut to about limit_us microseconds of SM clock (1 .. 1000000), for a shared-memory
 * barrier that nothing completes.  The wait runs out, sets bit 0 of the device flags and
 * the kernel returns: no fault, no trap, the context stays usable.  Returns
 * KVATTN_ERR_INVALID_ARG for a limit out of range, else the launch status.
 */
int kvattn_debug_wait_probe(int limit_us, void *stream);

/*
 * Test and tuning knob (process-wide): when workers > 0 the next calls use exactly
 * that many workers (CTAs or CTA pairs) and at least min_tiles tiles per worker,
 * which forces the split/combine path on small inputs.  workers == 0 restores the
 * built-in heuristic.
 */
void kvattn_debug_set_workers(int workers, int min_tiles);

/*
 * Test and tuning knob (process-wide): which kernel kvattn_gqa_decode runs.
 *   0  built-in choice (the tensor-memory kernel for head_dim 128 and groups of at
 *      least 4 query heads, the warp-level kernel otherwise)
 *   1  always the warp-level MMA kernel
 *   2  always the tensor-memory (tcgen05) kernel; calls it cannot serve (head_dim 64,
 *      or a batch too large for its shared memory) return KVATTN_ERR_UNSUPPORTED
 * Other values mean 0.  kvattn_gqa_decode_noalloc always runs the warp-level kernel.
 */
void kvattn_debug_set_gqa_kernel(int which);

/*
 * kvattn_gqa_decode without any allocation by the library.  The pages have no
 * counterpart to this call; it exists for callers that must not have a library call
 * cudaMalloc: serving engines that reserve nearly all device memory for their own
 * KV-cache pool (a stray allocation can fail or fragment it), and loops that cannot
 * afford cudaMalloc's implicit synchronisation.
 *   Arguments, layouts, results and errors are those of kvattn_gqa_decode; the call
 *   always runs the warp-level kernel (see kvattn_debug_set_gqa_kernel).
 *   Scratch: a fixed 6 MiB array inside the library, present on every GPU that loads
 *   the library until the process exits.  It holds the built-in plan of any batch on a
 *   device of up to 160 SMs (one worker per SM); a plan that needs more (a larger
 *   device, or kvattn_debug_set_workers forcing many workers) returns
 *   KVATTN_ERR_UNSUPPORTED with the sizes in kvattn_last_error_detail.  It calls no
 *   cudaMalloc, cudaFree or other allocating routine.
 *   The first call on a device looks up the array's device address (once per device,
 *   with that device current); make that first call before any stream capture.
 *   All calls share the one array and it keeps the last call's contents: calls that
 *   overlap on the GPU (different streams without ordering, or several host threads)
 *   race on it and give wrong results.  Order them on one stream.
 */
int kvattn_gqa_decode_noalloc(const uint16_t *q, const uint16_t *k_cache,
                              const uint16_t *v_cache, const int32_t *seq_lens, int max_seq_len,
                              int batch, int n_q_heads, int n_kv_heads, int head_dim, float scale,
                              float *out, float *lse, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* KVATTN_H */
