/*
 * dsa.h -- C ABI of the DeepSeek Sparse Attention (DSA) hot path on B200.
 *
 * The path has three steps (ouchyi thread on DeepSeek Sparse Attention,
 * web3.ouchyi.pink, "Nasil calisiyor" paragraph; tenelement.pl, "DeepSeek
 * V3.2-Exp Cuts Long-Context Costs with DeepSeek Sparse Attention (DSA) While
 * Maintaining Benchmark Parity", section "Architektura DeepSeek V3.2-Exp: Od
 * MoE do DSA"):
 *
 *   A. lightning indexer: every query scores every visible context token with
 *      a few FP8 heads through a ReLU,
 *          I[t,s] = sum_j w[t,j] * ReLU(q_I[t,j] . k_I[s]);
 *   B. top-k: each query keeps the k (2048 on the pages) best-scoring keys;
 *   C. core attention of all heads over only the kept keys, with one KV row
 *      per token shared by every head (MLA used in MQA form): key = the whole
 *      row (latent + rope), value = its first d_v columns (the latent)
 *      (degnora.com, "DeepSeekV3, Farki Ne?", section "MLA - Multi-Latent
 *      Attention").
 *
 * Positions.  Query token t (0 <= t < T) of a sequence sits at position
 * pos(t) = (S - T) + t and sees keys s <= pos(t) (itself included).  A
 * prefill has T == S (pos = t); a decode step has T == 1 (pos = S - 1, all S
 * keys visible).
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers to contiguous row-major arrays in
 *    the layouts stated below, owned by the caller.  The library allocates no
 *    memory on any call; scratch comes from the caller's workspace.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every
 *    call only enqueues work on it and returns; nothing synchronises the host
 *    except dsa_get_device_error().
 *  - The current CUDA device must be the one that owns the buffers.
 *  - Argument and shape problems are reported synchronously through the
 *    return value, before anything is enqueued.  A failed launch returns
 *    DSA_ERR_CUDA.  Conditions found on the device (a bounded wait that gave
 *    up, an index out of range) never trap: they are recorded in a device
 *    error word that dsa_get_device_error() reads and clears.  No C++
 *    exception crosses this interface.
 *  - Preconditions not checked on the host: q_scale and k_scale finite and
 *    > 0 (this is what lets the kernels apply the scales after the ReLU);
 *    no NaN in the FP8 or BF16 inputs; idx entries in [-1, S) and <= pos(t).
 *
 * Supported shapes: D_I in {32, 64, 128}; H_I in {4, 8, 16, 32, 64};
 * d_k in {80, 576} with d_v in {64, 512} respectively (d_v < d_k);
 * 1 <= H <= 128 with H % 8 == 0; 1 <= k <= 2048; T <= S; S < 2^31 / 8.
 * Anything else returns DSA_ERR_UNSUPPORTED.
 */
#ifndef DSA_H
#define DSA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define DSA_API __attribute__((visibility("default")))
#else
#define DSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DSA_OK = 0,
  DSA_ERR_INVALID_ARG = 1,   /* null pointer, negative size, bad stride     */
  DSA_ERR_UNSUPPORTED = 2,   /* valid but outside the supported shapes      */
  DSA_ERR_WORKSPACE = 3,     /* workspace missing or smaller than required  */
  DSA_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed        */
  DSA_ERR_TIMEOUT = 5,       /* device: a bounded wait gave up              */
  DSA_ERR_DEVICE_BOUNDS = 6  /* device: an index outside its valid range    */
} dsa_status;

typedef enum { DSA_PREFILL = 0, DSA_DECODE = 1 } dsa_mode;

/* Problem description shared by all entry points. */
typedef struct {
  int mode;             /* dsa_mode; only dsa_forward looks at it            */
  int B;                /* sequences in the batch                            */
  int T;                /* query tokens per sequence                         */
  int S;                /* keys (context tokens) per sequence                */
  int H_I, D_I;         /* indexer heads and head dim                        */
  int H, d_k, d_v;      /* attention heads, key dim, value dim (V = kv[:d_v])*/
  int k;                /* keys kept per query                               */
  int q_block;          /* prefill: queries per score tile (<= 0: 4096)      */
  float softmax_scale;  /* <= 0 selects 1/sqrt(d_k)                          */
} dsa_shape;

/* Inputs of the whole path (device pointers). */
typedef struct {
  const uint8_t* q_I;      /* [B, T, H_I, D_I] FP8 e4m3 indexer queries       */
  const float* q_scale;    /* [B, T, H_I]      dequant scale per query head   */
  const float* w;          /* [B, T, H_I]      indexer head weights           */
  const uint8_t* k_I;      /* [B, S, D_I]      FP8 e4m3 indexer keys          */
  const float* k_scale;    /* [B, S]           dequant scale per key          */
  const uint16_t* q;       /* [B, T, H, d_k]   BF16 attention queries         */
  const uint16_t* kv;      /* [B, S, d_k]      BF16 cached latent+rope rows   */
} dsa_inputs;

/* Library version (major * 100 + minor). */
DSA_API int dsa_version(void);

/* Human-readable name of a status code (static string). */
DSA_API const char* dsa_status_string(dsa_status status);

/* Bytes of workspace dsa_forward / dsa_prefill / dsa_decode need for `shape`
 * (it covers dsa_topk and dsa_sparse_attn too).  0 if the shape is invalid. */
DSA_API size_t dsa_workspace_size(const dsa_shape* shape);

/* Step A -- lightning indexer scores for queries [q_begin, q_begin + q_count)
 * of every sequence.  scores row (b * q_count + i) holds query
 * t = q_begin + i of sequence b, with ld_scores floats between rows
 * (ld_scores >= S, and a multiple of 4).  Entry s of a row is written for
 * s <= pos(t) only; the rest of the row is left untouched.
 *   scores[b*q_count+i][s] = k_scale[b,s] *
 *        sum_j w[b,t,j] * q_scale[b,t,j] * ReLU(sum_d q8[b,t,j,d] * k8[b,s,d])
 * which equals I[t,s] on the dequantised operands since the scales are > 0.
 * The FP8 products are accumulated in FP32. */
DSA_API dsa_status dsa_indexer_scores(const dsa_shape* shape, const uint8_t* q_I,
                              const float* q_scale, const float* w,
                              const uint8_t* k_I, const float* k_scale,
                              int q_begin, int q_count, float* scores,
                              int64_t ld_scores, void* stream);

/* Step B -- top-k per score row.  Reads rows laid out as dsa_indexer_scores
 * writes them (only entries s <= pos(t) are read) and writes idx rows
 * idx[b, t, 0..k) for t in [q_begin, q_begin + q_count): the indices of the
 * min(k, pos(t) + 1) largest scores, ties going to the lower index, in no
 * particular order, followed by -1 in the unused slots.  -0.0 and +0.0 count
 * as equal.  ws is optional scratch.  For few long rows (B * q_count * 2
 * below the SM count and S >= 16384, as in decode), if ws_bytes is at least
 * 73,744 bytes per row (ws 16-byte aligned), each row is split over 16
 * blocks: histogram, candidate collection, then a per-row selection.
 * Otherwise, or with ws NULL, one block handles each row.  dsa_forward
 * reserves this scratch inside dsa_workspace_size. */
DSA_API dsa_status dsa_topk(const dsa_shape* shape, const float* scores,
                    int64_t ld_scores, int q_begin, int q_count, int32_t* idx,
                    void* ws, size_t ws_bytes, void* stream);

/* Step B without any allocation (an addition of this library; the sparse
 * attention papers have no counterpart).  Same arguments, output and error
 * checks as dsa_topk, minus the workspace: the per-row histograms of the split
 * top-k path live in a fixed array of DSA_TOPK_STATIC_MAX_ROWS x 2048 words
 * (512 KiB) compiled into the library, so neither this call nor anything it
 * calls allocates memory.  It is meant for callers that cannot allocate at
 * call time: a C host program given only the score and index buffers, or a
 * decode loop whose HBM is reserved up front for weights and the key cache,
 * where a late cudaMalloc could fail or synchronise the device.
 *   - B * q_count > DSA_TOPK_STATIC_MAX_ROWS: DSA_ERR_WORKSPACE, nothing
 *     launched (use dsa_topk for more rows);
 *   - each call first clears the histogram rows it uses, in stream order;
 *   - all calls on a device share the array: calls whose launches may run at
 *     the same time on the GPU (unordered streams, concurrent host threads)
 *     race on it and may return wrong indices; calls in sequence on one
 *     stream are safe;
 *   - the first call on a device looks up the array's address with that device
 *     current; make that first call before any stream capture begins. */
#define DSA_TOPK_STATIC_MAX_ROWS 64
DSA_API dsa_status dsa_topk_static(const dsa_shape* shape, const float* scores,
                           int64_t ld_scores, int q_begin, int q_count,
                           int32_t* idx, void* stream);

/* Step C -- sparse MQA/MLA attention over the selected keys.
 *   q   [B, T, H, d_k] BF16;  kv [B, S, d_k] BF16 (V = kv[..., :d_v]);
 *   idx [B, T, k] int32, -1 = empty slot (skipped), duplicates counted twice;
 *   out [B, T, H, d_v] BF16 (rounded to nearest even from FP32);
 *   lse [B, T, H] FP32 natural-log sum of exp of the scaled logits, or NULL.
 * out[b,t,h] = sum_{s in idx[b,t]} softmax_s(tau q[b,t,h].kv[b,s]) kv[b,s,:d_v].
 * A row with no valid index gives out = 0 and lse = -inf.
 * ws: dsa_workspace_size(shape) bytes (decode splits the keys and merges the
 * partial results there); may be NULL in prefill mode. */
DSA_API dsa_status dsa_sparse_attn(const dsa_shape* shape, const uint16_t* q,
                           const uint16_t* kv, const int32_t* idx,
                           uint16_t* out, float* lse, void* ws,
                           size_t ws_bytes, void* stream);

/* The whole path, A -> B -> C, in `shape->mode`.  Prefill scores the queries
 * in blocks of q_block rows so the T x S score matrix never exists in full.
 * idx_out: [B, T, k] int32 receives the selection (required).
 * ws: at least dsa_workspace_size(shape) bytes. */
DSA_API dsa_status dsa_forward(const dsa_shape* shape, const dsa_inputs* in,
                       uint16_t* out, float* lse, int32_t* idx_out, void* ws,
                       size_t ws_bytes, void* stream);

/* dsa_forward with mode forced to DSA_PREFILL / DSA_DECODE (T must be 1). */
DSA_API dsa_status dsa_prefill(const dsa_shape* shape, const dsa_inputs* in,
                       uint16_t* out, float* lse, int32_t* idx_out, void* ws,
                       size_t ws_bytes, void* stream);
DSA_API dsa_status dsa_decode(const dsa_shape* shape, const dsa_inputs* in,
                      uint16_t* out, float* lse, int32_t* idx_out, void* ws,
                      size_t ws_bytes, void* stream);

/* Synchronises `stream`, then reads and clears the device error word of the
 * current device.  Returns DSA_OK, DSA_ERR_TIMEOUT or DSA_ERR_DEVICE_BOUNDS
 * (the first error recorded since the last call), or DSA_ERR_CUDA if the
 * synchronisation itself failed.  *detail (if not NULL) receives a
 * kernel-specific code for the recorded error (0 if none). */
DSA_API dsa_status dsa_get_device_error(void* stream, int* detail);

/* Number of kernel launches this library has enqueued in this process so
 * far (all devices).  Diagnostics: lets a caller count the launches one call
 * or one timed region made. */
DSA_API unsigned long long dsa_launch_count(void);

/* Bounded waits: every wait inside a kernel gives up after this many
 * microseconds of wall-clock time (default 2,000,000 = 2 s) and the kernel
 * reports DSA_ERR_TIMEOUT instead of hanging.  Applies to later launches;
 * values <= 0 restore the default.  A small value is a test hook. */
DSA_API void dsa_set_wait_timeout_us(long long microseconds);

/* Failure-detection self test (no counterpart on the pages): launches one
 * small kernel whose bounded wait can never be satisfied, so it gives up after
 * the wait timeout (dsa_set_wait_timeout_us) and records DSA_ERR_TIMEOUT in
 * the device error word, which the caller then reads with
 * dsa_get_device_error().  Returns the launch status.  Nothing faults, traps
 * or hangs. */
DSA_API dsa_status dsa_selftest_wait_timeout(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* DSA_H */
