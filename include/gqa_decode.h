/*
 * gqa_decode.h -- C ABI of the B200 grouped-query attention library.
 *
 * One gqa_decode call computes one decode step of one attention layer: every
 * query head of every sequence attends, with a single new query token, over
 * that sequence's cached keys and values.  Key/value head g of the cache
 * serves the R = H_Q / H_KV query heads h with g = floor(h / R) and is read
 * from HBM once for all of them.  gqa_prefill computes the multi-token step
 * (fresh prompts, or prompt chunks after a cached prefix) with the causal
 * mask; gqa_rope_append and gqa_decode_fp8kv cover the step before decode and
 * an 8-bit cache.
 *
 * Defining passages (cited by page title and section):
 *   [LLMS] "Grouped-Query Attention (GQA) and Multi-Query Attention (MQA):
 *          Mathematical Foundations, Arithmetic Intensity, and KV-Cache
 *          Scaling Mechanics" (llms.blog)
 *          - section 2, "Grouped-Query Attention": group size R = H_Q / G,
 *            H_KV = G, group index g(i) = floor((i-1)/R) + 1 (1-based), and
 *            Head_i = softmax(Q_i K_{g(i)}^T / sqrt(d_k) + M) V_{g(i)}.
 *            G = H_Q is MHA, G = 1 is MQA.
 *          - section 2, the K, V in R^{b x s x G x d_k} layout that the
 *            contiguous cache below follows.
 *          - section 1, "KV Cache Memory Footprint": the cache-size formula.
 *          - Sources list: PagedAttention (vLLM), the origin of the paged
 *            cache layout.
 *   [AIT]  "Grouped-Query Attention Shares Keys Without Sharing Every Query"
 *          (aitamer.news): the cache estimate 2 x layers x tokens x groups x
 *          head dim x bytes per element, and "paging" as a serving layout.
 *
 * What one call computes, for b < B and h < H_Q, with g = h / R, L_b the
 * clamped seq_lens[b], and t < L_b:
 *     s_t = scale * <q[b,h,:], K_b[t,g,:]>
 *     out[b,h,:] = sum_t softmax(s)_t * V_b[t,g,:]
 * The single query is the newest position, so the causal mask keeps all L_b
 * cached tokens (the current token's key/value already appended) and drops
 * positions >= L_b.  L_b = 0 gives out[b,h,:] = 0.
 *
 * Ownership and threading: the caller allocates every buffer (inputs, out
 * and workspace).  The library allocates no device memory, never
 * synchronises the stream in gqa_decode, and enqueues its kernels on the
 * caller's stream.  Calls on different streams must not share a workspace.
 * All entry points are thread-safe.
 */
#ifndef GQA_DECODE_H
#define GQA_DECODE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define GQA_DECODE_VERSION 1

typedef enum gqa_status {
    GQA_OK = 0,
    GQA_ERR_INVALID = 1,     /* an argument is invalid; nothing was launched */
    GQA_ERR_UNSUPPORTED = 2, /* valid but not implemented (e.g. head_dim 96) */
    GQA_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed */
    GQA_ERR_WORKSPACE = 4    /* workspace missing, misaligned or too small */
} gqa_status;

typedef enum gqa_dtype {
    GQA_BF16 = 0,
    GQA_F32 = 1
} gqa_dtype;

/* Coordinate pairs a rotary embedding turns together. */
typedef enum gqa_rope_pairing {
    GQA_ROPE_ADJACENT = 0,  /* (2i, 2i+1): the block-diagonal R_{Theta,m} as written */
    GQA_ROPE_HALVES = 1     /* (i, i + head_dim/2) */
} gqa_rope_pairing;

/* Which split kernel serves a call (both compute the same result). */
typedef enum gqa_kernel {
    GQA_KERNEL_AUTO = 0,     /* head_dim 128: tcgen05 for 8-bit caches (R <= 32) and for bf16 with
                                9 <= R <= 32; mma.sync for the other bf16 groups (R <= 64);
                                CUDA cores otherwise */
    GQA_KERNEL_MMA_SYNC = 1, /* warp-level mma.sync kernel: bf16 cache with R <= 64, or an 8-bit
                                cache with head_dim 128 and R <= 8 */
    GQA_KERNEL_TCGEN05 = 2   /* tcgen05 / tensor-memory kernel: head_dim 128, R <= 32, bf16 query,
                                bf16 or 8-bit cache */
} gqa_kernel;

/* Device status flags, accumulated (bitwise OR) in the workspace. */
#define GQA_FLAG_SEQ_LEN_CLAMPED 1u   /* a seq_lens entry was < 0 or > max_seq_len */
#define GQA_FLAG_BAD_BLOCK 2u         /* a live block_table entry was outside [0, num_blocks) */
#define GQA_FLAG_TIMEOUT 4u           /* an internal pipeline wait gave up; outputs invalid */
#define GQA_FLAG_BAD_POSITION 8u      /* a rope/append position was outside [0, max_seq_len) */
#define GQA_FLAG_BAD_QUERY_SPAN 16u   /* gqa_prefill: a cu_q_lens span was out of order, outside
                                         [0, total_q], longer than max_q_len or than L_b */

/*
 * Problem description.  All counts are element counts.
 *
 *  B, H_Q, H_KV     batch rows, query heads, key/value heads.  H_Q % H_KV == 0
 *                   ([LLMS] section 2: R = H_Q / G is a whole number).
 *  head_dim         d_k = d_v; 64 or 128.
 *  max_seq_len      contiguous cache: its sequence capacity S_max (the second
 *                   dimension of k_cache/v_cache).  Paged cache: the largest
 *                   allowed length, <= max_blocks_per_seq * page_size.
 *                   seq_lens entries are clamped to [0, max_seq_len].
 *  page_size        0 for a contiguous cache, 64 for a paged cache.
 *  max_blocks_per_seq, num_blocks   paged cache only (else 0): columns of the
 *                   block table, and pages held by k_cache/v_cache.
 *  qkv_dtype        element type of q, k_cache and v_cache.
 *  out_dtype        element type of out.  F32 keeps the fp32 accumulator.
 *  kernel           gqa_kernel; 0 (automatic) for normal use.  A kernel that
 *                   cannot serve the problem gives GQA_ERR_UNSUPPORTED.
 */
typedef struct gqa_decode_params {
    int32_t B;
    int32_t H_Q;
    int32_t H_KV;
    int32_t head_dim;
    int32_t max_seq_len;
    int32_t page_size;
    int32_t max_blocks_per_seq;
    int32_t num_blocks;
    gqa_dtype qkv_dtype;
    gqa_dtype out_dtype;
    int32_t kernel;
} gqa_decode_params;

/*
 * Bytes of workspace gqa_decode needs for these parameters on the CURRENT
 * CUDA device (the size depends on its SM count).  Writes *bytes.
 * The workspace holds one status word and the split-KV partial results.
 * Zero-fill it once after allocating it (the status word must start at 0);
 * later calls need no clearing.
 */
gqa_status gqa_decode_workspace_size(const gqa_decode_params* params, size_t* bytes);

/*
 * One decode step, enqueued on `stream` (a cudaStream_t; NULL = legacy default).
 *
 * Device pointers, row-major, innermost dimension last:
 *   q            [B, H_Q, head_dim]                       qkv_dtype, 16-byte aligned
 *   k_cache,     contiguous: [B, max_seq_len, H_KV, head_dim]
 *   v_cache      paged:      [num_blocks, 64, H_KV, head_dim]
 *                qkv_dtype, 16-byte aligned.  Rows at positions >= L_b are
 *                never used (they may hold anything, NaN included).
 *   seq_lens     int32 [B], cached tokens per sequence including the newest.
 *   block_table  int32 [B, max_blocks_per_seq] for a paged cache, else NULL.
 *                Token t of sequence b lives in page block_table[b][t / 64],
 *                slot t % 64.  Entries past ceil(L_b / 64) are not read.
 *   scale        softmax scale, usually 1/sqrt(head_dim) ([LLMS] section 2).
 *   out          [B, H_Q, head_dim] out_dtype, 8-byte aligned.
 *   workspace    >= gqa_decode_workspace_size bytes, 256-byte aligned.
 *
 * Errors: argument errors return GQA_ERR_INVALID / GQA_ERR_UNSUPPORTED /
 * GQA_ERR_WORKSPACE before anything is enqueued.  seq_lens and block_table
 * are device data and are not read on the host: out-of-range lengths are
 * clamped and out-of-range pages read as zeros, and both raise a flag in the
 * workspace status word (see gqa_read_status).  The kernels never trap.
 * A launch failure returns GQA_ERR_CUDA.
 */
gqa_status gqa_decode(const gqa_decode_params* params, const void* q, const void* k_cache,
                      const void* v_cache, const int32_t* seq_lens, const int32_t* block_table,
                      float scale, void* out, void* workspace, size_t workspace_bytes,
                      void* stream);

/*
 * gqa_decode over an 8-bit cache: k_cache and v_cache hold OCP E4M3 bytes
 * (sign, 4 exponent bits with bias 7, 3 mantissa bits; 0x7F/0xFF are NaN; max
 * 448) and the cached keys and values are
 *     K[b,t,g,:] = e4m3(k_cache[b,t,g,:]) * k_scale[g]
 *     V[b,t,g,:] = e4m3(v_cache[b,t,g,:]) * v_scale[g]
 * with per-KV-head fp32 factors k_scale[H_KV], v_scale[H_KV] (device).  This is
 * the bytes-per-element term of [AIT]'s cache estimate: the same attention
 * over a cache that moves half the bytes of bf16.  q stays bf16
 * (params->qkv_dtype must be GQA_BF16); layouts, seq_lens,
 * block_table, scale, out and the workspace (gqa_decode_workspace_size with
 * the same params suffices) are as for gqa_decode.  head_dim 128 with up to 32
 * query heads per KV head runs on the tcgen05 kernel (params->kernel =
 * GQA_KERNEL_MMA_SYNC selects the mma.sync kernel for up to 8, which widens to
 * f16 and so needs |q| < 65504); other shapes run on CUDA cores.  Cache bytes of
 * live tokens must not be the E4M3 NaN encodings.
 */
gqa_status gqa_decode_fp8kv(const gqa_decode_params* params, const void* q, const void* k_cache,
                            const void* v_cache, const float* k_scale, const float* v_scale,
                            const int32_t* seq_lens, const int32_t* block_table, float scale, void* out,
                            void* workspace, size_t workspace_bytes, void* stream);

/*
 * gqa_decode that also records `split_begin` just before and `split_end`
 * just after the split-KV kernel (both cudaEvent_t, either may be NULL).
 * For measuring the dominant kernel alone; the result equals gqa_decode's.
 */
gqa_status gqa_decode_timed(const gqa_decode_params* params, const void* q, const void* k_cache,
                            const void* v_cache, const int32_t* seq_lens,
                            const int32_t* block_table, float scale, void* out, void* workspace,
                            size_t workspace_bytes, void* stream, void* split_begin,
                            void* split_end);

/*
 * gqa_decode without a caller-supplied workspace, for callers that cannot
 * call cudaMalloc -- for example a plugin inside a host application that has
 * already handed all device memory to its own pool, or a latency-critical
 * loop that must not take cudaMalloc's implicit device-wide synchronisation.
 * The pages this library follows have no counterpart to this entry point; it
 * is a deployment convenience.
 *
 * The workspace is a fixed 8 MiB array inside the library (GQA_STATIC_WORKSPACE_BYTES),
 * held on every GPU that loads the library until the process exits.  The
 * call allocates nothing.  Arguments, layouts and results are those of
 * gqa_decode; the caller still provides q, the caches, seq_lens,
 * block_table and out.
 *
 *  - Returns GQA_ERR_WORKSPACE, before launching anything, when these
 *    parameters need more workspace than the array holds (see
 *    gqa_decode_workspace_size).
 *  - The first call on each device looks up the array's device address with
 *    that device current and clears its status word on `stream`; make that
 *    first call before any stream capture begins.
 *  - Every call on a device shares the one array, and it keeps the last
 *    call's contents.  Calls whose kernels overlap on the GPU (different
 *    streams, or different host threads) race on it: order them.
 *  - Device-side problems (clamped seq_lens, out-of-range pages, a pipeline
 *    wait that gave up) are flagged in the array's status word exactly as in
 *    a caller's workspace; read and clear them with
 *    gqa_static_workspace_status.  The flags accumulate until cleared.
 *  - The looked-up address is kept for the life of the process: after
 *    cudaDeviceReset (or anything else that destroys the device's primary
 *    context) this entry point must not be called again on that device.
 */
#define GQA_STATIC_WORKSPACE_BYTES (8u << 20)
gqa_status gqa_decode_static_workspace(const gqa_decode_params* params, const void* q,
                                       const void* k_cache, const void* v_cache,
                                       const int32_t* seq_lens, const int32_t* block_table,
                                       float scale, void* out, void* stream);

/*
 * The status word of gqa_decode_static_workspace's built-in array on the
 * CURRENT device: like gqa_read_status, it synchronises `stream`, writes the
 * accumulated GQA_FLAG_* bits to *flags and clears them when `clear` is
 * non-zero.  Allocates nothing.  On a device where gqa_decode_static_workspace
 * has not run yet it performs that call's one-time set-up (address lookup and
 * a cleared status word) and reports 0.  The pages this library follows have
 * no counterpart to it.
 */
gqa_status gqa_static_workspace_status(void* stream, uint32_t* flags, int clear);

/*
 * The step before gqa_decode for a new token: rotary position embedding of
 * its query heads, and the append of its key and value rows to the cache.
 * [LLMS] section 4, "Rotary Position Embeddings (RoPE) Interaction": RoPE is
 * applied to each of the H_Q query heads and once to each of the H_KV key
 * heads, R_{Theta,m} = diag(R_{theta_1,m}, ..., R_{theta_{d/2},m}) with the
 * token's position m; theta_i = rope_base^(-2i/head_dim), i = 0..head_dim/2-1
 * (the RoFormer frequencies the page cites; e.g. rope_base 10000).
 *
 * For every b, with m = positions[b] (the number of tokens already cached):
 *   q_out[b,h,:]              = RoPE_m(q[b,h,:])            h < H_Q
 *   cache row (b, m, g) of k  = RoPE_m(k_new[b,g,:])        g < H_KV
 *   cache row (b, m, g) of v  = v_new[b,g,:]
 *   seq_lens_out[b]           = m + 1                        (if not NULL)
 * The cache row is k_cache[b][m][g] (contiguous) or
 * k_cache[block_table[b][m/64]][m%64][g] (paged), as in gqa_decode.
 *
 *   params      as for gqa_decode (cache geometry, qkv_dtype; out_dtype unused)
 *   q, q_out    [B, H_Q, head_dim]; q_out may equal q (in place)
 *   k_new,v_new [B, H_KV, head_dim]
 *   positions   int32 [B], device
 *   pairing     gqa_rope_pairing
 *   seq_lens_out int32 [B] device or NULL; must not overlap positions
 *   workspace   a gqa_decode workspace (status word) or NULL
 * Angles and rotations are evaluated in double and rounded once to the
 * storage type.  A position outside [0, max_seq_len) (or a page outside
 * [0, num_blocks)) skips that sequence's cache write and raises
 * GQA_FLAG_BAD_POSITION (GQA_FLAG_BAD_BLOCK) in the workspace status word.
 * Enqueued on `stream`, chained so that a following gqa_decode may launch
 * early; argument errors return before anything is enqueued.
 */
gqa_status gqa_rope_append(const gqa_decode_params* params, const void* q, const void* k_new,
                           const void* v_new, const int32_t* positions, const int32_t* block_table,
                           double rope_base, int pairing, void* q_out, void* k_cache, void* v_cache,
                           int32_t* seq_lens_out, void* workspace, void* stream);

/*
 * Multi-token step: prefill of new prompts, or a chunk of a prompt after a
 * cached prefix, for every sequence of the batch at once.  [LLMS] opening
 * section: prompt processing (prefill) is the compute-bound phase; section 2:
 * Head_i = softmax(Q_i K_{g(i)}^T / sqrt(d_k) + M) V_{g(i)} with M the causal
 * mask.  Sequence b brings n_b = cu_q_lens[b+1] - cu_q_lens[b] new query
 * tokens, rows cu_q_lens[b] .. cu_q_lens[b+1]-1 of q, whose keys and values
 * are already the last n_b of its L_b = seq_lens[b] cached tokens (appended
 * beforehand, e.g. by the caller's projection).  Its query token j sits at
 * position p = L_b - n_b + j and attends to cache positions t <= p -- the
 * whole cached prefix and the new tokens up to itself.  With no prefix
 * (L_b = n_b) M is the s x s causal mask as written; n_b = 1 is gqa_decode's
 * step.  For every row i of sequence b, query head h, g = h / R:
 *     s_t = scale * <q[i,h,:], K_b[t,g,:]>,   t <= p
 *     out[i,h,:] = sum_t softmax(s)_t * V_b[t,g,:]
 *
 *   params      as for gqa_decode; head_dim 128, qkv_dtype GQA_BF16 and
 *               R = H_Q / H_KV <= 128 (else GQA_ERR_UNSUPPORTED); kernel AUTO
 *               or TCGEN05 (the only implementation: tcgen05 tensor cores).
 *   q           [total_q, H_Q, 128] bf16, 16-byte aligned, sequences' rows
 *               back to back in the order of cu_q_lens.
 *   cu_q_lens   int32 [B + 1] device, cu_q_lens[0] = 0, non-decreasing,
 *               cu_q_lens[B] = total_q; 0 <= n_b <= min(L_b, max_q_len).
 *   total_q     rows of q and out (host value).
 *   max_q_len   host upper bound on every n_b; sizes the launch.
 *   k_cache, v_cache, seq_lens, block_table   as for gqa_decode.
 *   scale       softmax scale, finite and > 0 (usually 1/sqrt(128)).
 *   out         [total_q, H_Q, 128] out_dtype, 16-byte aligned.  Rows of a
 *               sequence whose span is invalid are left untouched.
 *   workspace   >= gqa_prefill_workspace_size bytes (any gqa_decode
 *               workspace will do), 256-byte aligned, zero-filled once: it
 *               holds the status word.
 * cu_q_lens, seq_lens and block_table are device data and are not read on the
 * host: an invalid span skips that sequence and raises GQA_FLAG_BAD_QUERY_SPAN;
 * lengths and pages are handled as in gqa_decode.  Argument errors return
 * before anything is enqueued; the call allocates nothing and does not
 * synchronise.  Weights enter the value product as bf16 hi + lo parts (within
 * 2^-15 of each weight), accumulation is fp32.
 */
gqa_status gqa_prefill_workspace_size(const gqa_decode_params* params, size_t* bytes);

gqa_status gqa_prefill(const gqa_decode_params* params, const void* q, const int32_t* cu_q_lens,
                       int32_t total_q, int32_t max_q_len, const void* k_cache, const void* v_cache,
                       const int32_t* seq_lens, const int32_t* block_table, float scale, void* out,
                       void* workspace, size_t workspace_bytes, void* stream);

/*
 * Reads the workspace status word (GQA_FLAG_* bits) into *flags after
 * synchronising `stream`; clears it when `clear` is non-zero.
 */
gqa_status gqa_read_status(const void* workspace, void* stream, uint32_t* flags, int clear);

/*
 * Exercises, on the GPU and without any fault, the bounded wait every kernel
 * of this library uses for its pipeline barriers.  One CTA waits on an
 * mbarrier that nothing arrives on; the wait gives up after timeout_ns and
 * the kernel raises GQA_FLAG_TIMEOUT in *flags (device uint32, OR-ed) and
 * writes the nanoseconds it waited to *elapsed_ns (device uint64).  With
 * abort_early non-zero, a second warp sets the CTA's abort flag after
 * timeout_ns / 4 and the wait returns then (the flag is raised the same way).
 * timeout_ns must lie in [1000, 10^10].  Enqueued on `stream`; allocates
 * nothing.  For tests of failure detection: the context stays usable.
 */
gqa_status gqa_wait_selftest(uint64_t timeout_ns, int abort_early, uint32_t* flags, uint64_t* elapsed_ns,
                             void* stream);

/*
 * KV-cache size in bytes: 2 x layers x tokens x H_KV x head_dim x elem_bytes
 * ([LLMS] section 1 "KV Cache Memory Footprint"; [AIT] cache estimate).
 * tokens counts every cached token of every sequence.  Host-only, pure.
 */
uint64_t gqa_kv_cache_bytes(int64_t layers, int64_t tokens, int64_t H_KV, int64_t head_dim,
                            int64_t elem_bytes);

/* Static string for a status code. */
const char* gqa_status_string(gqa_status status);

/* GQA_DECODE_VERSION of the loaded library. */
int gqa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GQA_DECODE_H */
