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
 * Positions with per-sequence lengths.  With shape->seqlens set, sequence b
 * holds L_b = seqlens[b] keys (T <= L_b <= S) and its query t sits at
 * pos(t) = (L_b - T) + t; keys s >= L_b are never read.  A ragged decode batch
 * (each sequence at its own length) is T == 1 with seqlens.  S stays the row
 * stride of the contiguous caches and the bound of every L_b.
 *
 * Paged caches.  With shape->page_size > 0, the key-side inputs (k_I,
 * k_scale, kv and a separate v) are pools of num_pages * page_size token rows
 * instead of [B, S, ...] arrays: token s of sequence b lives in row
 *   block_table[b * pages_per_seq + s / page_size] * page_size + s % page_size.
 * page_size must be a multiple of 16.  Pages holding no key below L_b are
 * never read, so their block_table entries may be anything; an entry of a
 * page that is read and lies outside [0, num_pages) is reported as
 * DSA_ERR_DEVICE_BOUNDS and its keys read as zeros.
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers to contiguous row-major arrays in
 *    the layouts stated below, owned by the caller.  Scratch comes from the
 *    caller's workspace.  The one exception is dsa_topk_static, whose scratch
 *    is a fixed array inside this library (see its comment below).
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every
 *    call only enqueues work on it and returns; nothing synchronises the host
 *    except dsa_get_device_error().  Exception: the first call of
 *    dsa_topk_static on a device looks up its array's address (see there).
 *  - The library caches, per device, the device addresses of its own error
 *    word and static array.  They stay valid for the life of the CUDA
 *    context; after cudaDeviceReset (or anything else that destroys the
 *    primary context) reload the library before calling it again.
 *  - The current CUDA device must be the one that owns the buffers.
 *  - Argument and shape problems are reported synchronously through the
 *    return value, before anything is enqueued.  A failed launch returns
 *    DSA_ERR_CUDA.  Conditions found on the device (a bounded wait that gave
 *    up, an index or a length out of range) never trap: they are recorded in
 *    a device error word that dsa_get_device_error() reads and clears.  No C++
 *    exception crosses this interface.
 *  - Preconditions not checked on the host: q_scale and k_scale finite and
 *    > 0 (this is what lets the kernels apply the scales after the ReLU);
 *    no NaN in the FP8 or BF16 inputs; idx entries in [-1, L_b) and <= pos(t);
 *    T <= seqlens[b] <= S (a length outside is reported on the device and
 *    clamped into that range).
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
  int S;                /* keys (context tokens) per sequence, at most       */
  int H_I, D_I;         /* indexer heads and head dim                        */
  int H, d_k, d_v;      /* attention heads, key dim, value dim (V = kv[:d_v])*/
  int k;                /* keys kept per query                               */
  int q_block;          /* prefill: queries per score tile (<= 0: 4096)      */
  float softmax_scale;  /* <= 0 selects 1/sqrt(d_k)                          */
  const int32_t* seqlens;      /* device int32[B]: keys of sequence b, or NULL
                                  (every sequence has S keys)                */
  int page_size;               /* 0: contiguous caches; > 0: paged caches,
                                  tokens per page (a multiple of 16)         */
  int pages_per_seq;           /* paged: row length of block_table           */
  int num_pages;               /* paged: pages in each cache pool            */
  const int32_t* block_table;  /* paged: device int32[B, pages_per_seq]      */
} dsa_shape;

/* Inputs of the whole path (device pointers).  With page_size > 0 the four
 * key-side arrays are pools of num_pages * page_size token rows. */
typedef struct {
  const uint8_t* q_I;      /* [B, T, H_I, D_I] FP8 e4m3 indexer queries       */
  const float* q_scale;    /* [B, T, H_I]      dequant scale per query head   */
  const float* w;          /* [B, T, H_I]      indexer head weights           */
  const uint8_t* k_I;      /* [B, S, D_I]      FP8 e4m3 indexer keys          */
  const float* k_scale;    /* [B, S]           dequant scale per key          */
  const uint16_t* q;       /* [B, T, H, d_k]   BF16 attention queries         */
  const uint16_t* kv;      /* [B, S, d_k]      BF16 cached latent+rope rows   */
  const uint16_t* v;       /* [B, S, d_v]      BF16 values kept apart from the
                              keys, or NULL: V = kv[..., :d_v] (MLA)          */
} dsa_inputs;

/* Library version (major * 100 + minor). */
DSA_API int dsa_version(void);

/* Human-readable name of a status code (static string). */
DSA_API const char* dsa_status_string(dsa_status status);

/* Bytes of workspace dsa_forward / dsa_prefill / dsa_decode need for `shape`
 * with the query block's FP32 score tile held in it (it covers dsa_topk,
 * dsa_select and dsa_sparse_attn too).  0 if the shape is invalid. */
DSA_API size_t dsa_workspace_size(const dsa_shape* shape);

/* Bytes of workspace for dsa_select, and the least a prefill dsa_forward
 * accepts, where the fused selection applies (prefill, contiguous caches,
 * S >= 32768, S a multiple of 32): its regions replace the score tile, about
 * a quarter of the tile's size (0.56 GiB instead of 2 GiB for a 4096-row block
 * of a 128K context).  Elsewhere equal to dsa_workspace_size.  0 if the shape
 * is invalid. */
DSA_API size_t dsa_select_workspace_size(const dsa_shape* shape);

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

/* Steps A and B together for queries [q_begin, q_begin + q_count): writes the
 * selection idx[b, t, 0..k) as dsa_topk does (ties to the lower index, -1
 * after the last).  ws: dsa_select_workspace_size(shape) bytes.
 * In prefill over long contexts (S >= 32768, S a multiple of 32, contiguous
 * caches) the query block's score matrix is never stored (the pages ask that
 * the selection be cache-aware and stay on the device: sider.ai blog on
 * DeepSeek Sparse Attention, "Uyarilar"): the
 * indexer scores every 32nd key, a per-row radix select on that sample gives
 * a threshold expected to admit about 2k keys, the indexer then scores every
 * key and keeps only (score, index) pairs at or above the row's threshold
 * (at most 8192 per row), and the top k are selected exactly among them.  A
 * row left with fewer than k candidates, or more than the list holds, is
 * scored again in full into a small tile and selected from it, so the result
 * is the same exact top-k on any input (up to 64 such rows per query block;
 * beyond that DSA_ERR_DEVICE_BOUNDS is reported).  Otherwise the block's
 * scores go through the workspace as dsa_indexer_scores + dsa_topk. */
DSA_API dsa_status dsa_select(const dsa_shape* shape, const uint8_t* q_I,
                      const float* q_scale, const float* w, const uint8_t* k_I,
                      const float* k_scale, int q_begin, int q_count,
                      int32_t* idx, void* ws, size_t ws_bytes, void* stream);

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
 *   q   [B, T, H, d_k] BF16;  kv [B, S, d_k] BF16 (key = the whole row);
 *   v_or_null [B, S, d_v] BF16 values, or NULL: V = kv[..., :d_v] (MLA, the
 *       form of the pages; a separate V is a generalisation);
 *   idx [B, T, k] int32, -1 = empty slot (skipped), duplicates counted twice;
 *   out [B, T, H, d_v] BF16 (rounded to nearest even from FP32);
 *   lse [B, T, H] FP32 natural-log sum of exp of the scaled logits, or NULL.
 * out[b,t,h] = sum_{s in idx[b,t]} softmax_s(tau q[b,t,h].kv[b,s]) V[b,s].
 * A row with no valid index gives out = 0 and lse = -inf.  An index outside
 * [0, L_b) is reported as DSA_ERR_DEVICE_BOUNDS and skipped.
 * ws: dsa_workspace_size(shape) bytes (decode splits the keys and merges the
 * partial results there); may be NULL in prefill mode. */
DSA_API dsa_status dsa_sparse_attn(const dsa_shape* shape, const uint16_t* q,
                           const uint16_t* kv, const uint16_t* v_or_null,
                           const int32_t* idx, uint16_t* out, float* lse,
                           void* ws, size_t ws_bytes, void* stream);

/* Dense causal attention of every query over all its visible keys
 * s <= pos(t), with no indexer and no selection: the "MHA with a mask" form
 * in which short prefills run (tenelement.pl, "DeepSeek V3.2-Exp Cuts
 * Long-Context Costs ...", section "Efektywnosc Kosztowa").  When k covers
 * every visible key this is exactly what the sparse path computes, and
 * dsa_forward uses it by itself for those rows.  Arguments as for
 * dsa_sparse_attn, without idx; ws: dsa_workspace_size(shape) bytes in
 * decode mode (the keys of a long row are split and merged there), may be
 * NULL in prefill mode. */
DSA_API dsa_status dsa_dense_attn(const dsa_shape* shape, const uint16_t* q,
                          const uint16_t* kv, const uint16_t* v_or_null,
                          uint16_t* out, float* lse, void* ws,
                          size_t ws_bytes, void* stream);

/* The whole path, A -> B -> C, in `shape->mode`.  Prefill scores the queries
 * in blocks of q_block rows so the T x S score matrix never exists in full.
 * Rows whose every visible key fits in k (pos(t) + 1 <= k for any length
 * up to S) skip steps A and B: their selection is all visible keys, written
 * to idx_out as 0..pos(t), and step C runs on them densely.
 * idx_out: [B, T, k] int32 receives the selection (required).
 * ws: dsa_workspace_size(shape) bytes, or in prefill at least
 * dsa_select_workspace_size(shape): a workspace that holds the score tile
 * runs steps A and B as dsa_indexer_scores + dsa_topk; a smaller one that
 * holds the fused selection's regions runs them as dsa_select does (same
 * selection, less memory, more time); anything smaller is
 * DSA_ERR_WORKSPACE. */
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

/* ---- One sequence's keys over several devices (key-split decode) ----------
 * The pages run DSA on one device; these three calls are the exchange steps
 * that let one long sequence's keys live on P devices (an addition of this
 * library, resting on arithmetic, not on a passage of the pages: exact top-k
 * decomposes over disjoint key ranges -- the whole row's winners are winners
 * of their own range under the same order -- and exact softmax attention
 * decomposes through the log-sum-exp).  Part r holds keys
 * [part_begin_r, part_begin_r + S_r) and runs dsa_indexer_scores and dsa_topk
 * on a shape with S = S_r; then
 *   1. dsa_topk_candidates packs its selection as (score, global index);
 *   2. the caller all-gathers the P candidate lists (NCCL, P x B*T x k pairs);
 *   3. dsa_topk_merge gives the global top-k and this part's share of it as
 *      local indices, which dsa_sparse_attn (shape with S = S_r) consumes;
 *   4. the caller all-gathers the P (out, lse) pairs;
 *   5. dsa_attn_combine merges them.
 * Rows are every query row of the shape (B * T, decode: B). */

/* (score, global index) of each selected key: reads idx [B, T, k] (local
 * indices, -1 = empty) and the score rows [B*T, ld_scores] they index
 * (rows as dsa_indexer_scores writes them for q_begin = 0, q_count = T);
 * writes cand_scores [B*T, k] FP32 and cand_idx [B*T, k] int32 =
 * part_begin + local index (-inf and -1 for empty slots).  An index >= S is
 * reported as DSA_ERR_DEVICE_BOUNDS and written as empty. */
DSA_API dsa_status dsa_topk_candidates(const dsa_shape* shape, const float* scores,
                               int64_t ld_scores, const int32_t* idx,
                               int32_t part_begin, float* cand_scores,
                               int32_t* cand_idx, void* stream);

/* Global top-k of nparts candidate lists: cand_scores / cand_idx
 * [nparts, B*T, k] (part-major, as an all-gather stacks them).  Writes
 * idx [B*T, k]: the k best candidates by (score descending, global index
 * ascending), in no particular order, -1 after the last; and, if idx_local is
 * not NULL, idx_local [B*T, k]: the same selection as indices local to the
 * key range [local_begin, local_begin + local_count), -1 outside it.
 * nparts * k must not exceed 8192 (DSA_ERR_UNSUPPORTED; merge in rounds). */
DSA_API dsa_status dsa_topk_merge(const dsa_shape* shape, int nparts,
                          const float* cand_scores, const int32_t* cand_idx,
                          int32_t* idx, int32_t local_begin, int32_t local_count,
                          int32_t* idx_local, void* stream);

/* Merge of attention results over disjoint key subsets: o_parts
 * [nparts, B, T, H, d_v] BF16 and lse_parts [nparts, B, T, H] FP32 (natural
 * log, -inf = no key) as dsa_sparse_attn writes them, stacked part-major.
 *   out = sum_r e^(lse_r - M) o_r / sum_r e^(lse_r - M),  M = max_r lse_r,
 *   lse = M + ln sum_r e^(lse_r - M)   (lse may be NULL). */
DSA_API dsa_status dsa_attn_combine(const dsa_shape* shape, int nparts,
                            const uint16_t* o_parts, const float* lse_parts,
                            uint16_t* out, float* lse, void* stream);

/* ---- Training the indexer (kernel level) ----------------------------------
 * tenelement.pl, "DeepSeek V3.2-Exp Cuts Long-Context Costs ...", section
 * "Proces Treningu DSA: Od Warm-up do Sparsity": a warm-up in which the
 * indexer learns the dense model's attention distribution through a KL
 * divergence with the main model frozen, then a sparse stage over the top-k
 * set; the indexer's gradients stay apart from the main language loss.
 * Readings (the pages give no formula): the target of query t is the main
 * attention's weights summed over heads and divided by H; the loss is
 * KL(target || softmax(I[t, .])) over the visible keys (idx NULL: warm-up)
 * or over the selected set idx[b, t, :] (sparse stage); the target is a
 * constant.  Rows are queries [q_begin, q_begin + q_count) of every
 * sequence, row r = b * q_count + i of the [rows, ld] FP32 arrays. */

/* target[r, s] = (1/H) sum_h exp(tau q[b,t,h] . kv[b,s] - lse[b,t,h]) for
 * every visible key s (idx NULL) or every key of the set; lse [B, T, H] is
 * the main attention's natural log-sum-exp over the same keys (dsa_dense_attn
 * or dsa_sparse_attn output).  Other entries are left untouched.
 * d_k must be 576 (the MLA row). */
DSA_API dsa_status dsa_kl_target(const dsa_shape* shape, const uint16_t* q,
                         const uint16_t* kv, const float* lse, const int32_t* idx,
                         int q_begin, int q_count, float* target, int64_t ld,
                         void* stream);

/* Per row: loss[r] = KL(target || softmax(I)) over the set, and
 * grad[r, s] = softmax(I)_s - target[r, s] for keys of the set, 0 for other
 * visible keys.  scores: the indexer scores as dsa_indexer_scores writes
 * them for the same rows. */
DSA_API dsa_status dsa_indexer_kl(const dsa_shape* shape, const float* scores,
                          const float* target, int64_t ld, const int32_t* idx,
                          int q_begin, int q_count, float* grad, float* loss,
                          void* stream);

/* Gradients of sum_s grad[r, s] I[t, s] with respect to the dequantised
 * indexer inputs (FP32): dq [B, T, H_I, D_I] and dw [B, T, H_I] (rows of the
 * launch written), dk [B, S, D_I] accumulated into (+=; zero it first; paged
 * caches: the pool layout).  idx: the set whose keys carry gradient (NULL:
 * every visible key).  Supported (H_I, D_I): (64, 128), (32, 128),
 * (16, 128), (64, 64), (32, 64). */
DSA_API dsa_status dsa_indexer_backward(const dsa_shape* shape, const uint8_t* q_I,
                                const float* q_scale, const float* w,
                                const uint8_t* k_I, const float* k_scale,
                                const float* grad, int64_t ld, const int32_t* idx,
                                int q_begin, int q_count, float* dq, float* dw,
                                float* dk, void* stream);

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
