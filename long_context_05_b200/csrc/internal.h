// Internal declarations shared by the host API and the kernel files of
// libdsa.so.  Nothing here is part of the public ABI (include/dsa.h).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "dsa.h"

namespace dsa {

// Device error word: the first error recorded wins; read and cleared by
// dsa_get_device_error().  code is a dsa_status, detail kernel-specific.
struct DevErr {
  unsigned int code;
  unsigned int detail;
};

// Detail codes (low byte: which kernel; the rest: where).
enum : unsigned int {
  ERR_SITE_INDEXER = 0x10,
  ERR_SITE_TOPK = 0x20,
  ERR_SITE_ATTN = 0x30,
  ERR_SITE_COMBINE = 0x40,
};

#ifdef __CUDACC__
__device__ __forceinline__ void report_error(DevErr* e, unsigned int code, unsigned int detail) {
  if (e != nullptr && atomicCAS(&e->code, 0u, code) == 0u) atomicExch(&e->detail, detail);
}

// Order-preserving 32-bit key of a score: a > b as floats iff key(a) >
// key(b) as unsigned integers; -0.0 is folded onto +0.0.
__device__ __forceinline__ unsigned int order_key(float f) {
  unsigned int u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
#endif

// Where the keys of each sequence are: per-sequence lengths and the
// (optionally paged) layout of the key-side caches.
struct KvMap {
  const int32_t* seqlens;      // device int32[B] or null (every sequence has S keys)
  const int32_t* block_table;  // device int32[B, pages_per_seq] (paged only)
  int S;                       // keys per sequence at most; row stride when contiguous
  int T;                       // queries per sequence (a length below T is clamped up)
  int page_size;               // 0: contiguous [B, S, ...] caches
  int pages_per_seq, num_pages;

#ifdef __CUDACC__
  // Keys of sequence b, L_b.  A length outside [T, S] is reported once per
  // calling thread and clamped into that range.
  __device__ __forceinline__ int len(int b, DevErr* err, unsigned site) const {
    if (seqlens == nullptr) return S;
    const int L = seqlens[b];
    if (L < T || L > S) {
      report_error(err, DSA_ERR_DEVICE_BOUNDS, site | (0xB0u << 8));
      return L < T ? T : S;
    }
    return L;
  }
  // Cache row of token s of sequence b in a contiguous [B, S, ...] cache.
  __device__ __forceinline__ long long row_contig(int b, int s) const { return (long long)b * S + s; }
  // Cache row of token s of sequence b, or -1 when its page is not mapped.
  // Kernels instantiate a contiguous form that calls row_contig instead, so
  // that the page lookup stays out of their hot loops.
  template <bool PAGED = true>
  __device__ __forceinline__ long long row(int b, int s) const {
    if (!PAGED || page_size == 0) return (long long)b * S + s;
    const int pg = s / page_size;
    if (pg < 0 || pg >= pages_per_seq) return -1;
    const int e = block_table[(size_t)b * pages_per_seq + pg];
    if (e < 0 || e >= num_pages) return -1;
    return (long long)e * page_size + (s - pg * page_size);
  }
#endif
  // rows in each cache pool (contiguous: B * S)
  long long pool_rows(int B) const {
    return page_size == 0 ? (long long)B * S : (long long)num_pages * page_size;
  }
};

// Everything a launcher needs besides its own arguments.
struct LaunchCtx {
  cudaStream_t stream;
  DevErr* err;            // device address of this device's error word
  long long wait_ns;      // wall-clock limit of a bounded wait
  int num_sms;
  int device;
};

struct IndexerArgs {
  KvMap kv;
  int kstride;              // score every kstride-th key only (a sample; contiguous caches, S % kstride == 0)
  // candidate mode (thr set): instead of writing score rows, every epilogue
  // warp appends (launch row, key index, order key) of each visible score
  // whose key is >= thr[row] to its own list of wl_cap entries (warp w of the
  // launch at w * wl_cap; no atomics), and writes its count to wl_cnt[w];
  // entries past wl_cap are dropped and their rows flagged in row_fail
  const unsigned int* thr;
  int32_t* wl_row;
  int32_t* wl_idx;
  unsigned int* wl_key;
  unsigned int* wl_cnt;
  long long wl_cap;
  int* row_fail;
  // repair mode (row_slot set): score only the rows with row_slot[row] >= 0,
  // into score row row_slot[row]; work items without such a row are skipped
  const int* row_slot;
  const uint8_t* q_I;
  const float* q_scale;
  const float* w;
  const uint8_t* k_I;
  const float* k_scale;
  float* scores;
  int64_t ld;
  int B, T, S, H_I, D_I;
  int q_begin, q_count;
};

struct TopkArgs {
  KvMap kv;                 // only the lengths are used
  const float* scores;
  int64_t ld;
  int32_t* idx;
  int B, T, S, k;
  int q_begin, q_count;
};

struct AttnArgs {
  KvMap map;
  const uint16_t* q;
  const uint16_t* kv;
  const uint16_t* v;   // separate values [.., d_v] or null (V = kv[.., :d_v])
  const int32_t* idx;  // null: dense causal attention over every visible key
  int dense_rows;      // query rows t < dense_rows take all visible keys (idx not read)
  uint16_t* out;
  float* lse;
  float* part;         // split partials [rows, nsplit, H, d_v + 2] or null
  int B, T, S, H, d_k, d_v, k;
  int nsplit;          // key splits per query row (1 = write out directly)
  float tau;
  bool decode;         // decode mode: the split-k memory-bound kernel where it applies
};

// counts every kernel launch (dsa_launch_count)
void note_launches(int n);

// Launch with programmatic stream serialization: the kernel may start while
// the one before it on the stream finishes, and must call pdl_wait
// (sm100.cuh) before it reads anything that kernel writes.
template <class... KArgs, class... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

cudaError_t launch_indexer(const LaunchCtx& c, const IndexerArgs& a);
// ws: optional scratch for the split path (few long rows); see topk.cu
cudaError_t launch_topk(const LaunchCtx& c, const TopkArgs& a, void* ws, size_t ws_bytes);
size_t topk_workspace_bytes(int rows);
// top-k split path into an explicit histogram array of rows * 2048 words
cudaError_t launch_topk_split_into(const LaunchCtx& c, const TopkArgs& a, unsigned int* hist);
constexpr int kTopkHistBins = 2048;
bool topk_uses_workspace(int rows, int S, int num_sms);
cudaError_t launch_sparse_attn(const LaunchCtx& c, const AttnArgs& a);

// key-split rows (one sequence's keys over several parts; split.cu, topk.cu)
cudaError_t launch_topk_merge(const LaunchCtx& c, const float* cand_scores, const int32_t* cand_idx, int rows,
                              int nparts, int k, int32_t* idx, int local_begin, int local_count, int32_t* idx_local);
int topk_merge_max_candidates();

// selection without a score tile (topk.cu; the indexer's sample and
// candidate modes feed it)
int topk_cand_cap();
cudaError_t launch_topk_threshold(const LaunchCtx& c, const TopkArgs& a, const float* sample, long long ld_s,
                                  int kstride, int target, int cap, unsigned int* thr, unsigned int* cnt, int* row_slot,
                                  int* row_fail, unsigned int* nfail, unsigned int* wl_cnt, int nwl);
cudaError_t launch_topk_cand_select(const LaunchCtx& c, const TopkArgs& a, const unsigned int* cand_key,
                                    const int32_t* cand_idx, const unsigned int* cnt, int cap, const int* row_fail,
                                    int* row_slot, int* fail_rows, unsigned int* nfail, int max_fail);
// the warps' candidate lists into per-row lists [rows, cap] (counts in cnt)
cudaError_t launch_topk_scatter(const LaunchCtx& c, const int32_t* wl_row, const int32_t* wl_idx,
                                const unsigned int* wl_key, const unsigned int* wl_cnt, long long wl_cap, int nwarps,
                                unsigned int* cnt, unsigned int* cand_key, int32_t* cand_idx, int cap);
// epilogue warps of one indexer CTA, and the indexer's grid, for sizing its
// candidate lists
int indexer_epilogue_warps(int H_I);
cudaError_t launch_topk_repair(const LaunchCtx& c, const TopkArgs& a, const float* tile, long long ld,
                               const int* fail_rows, const unsigned int* nfail, int max_fail);

// the indexer's backward on tensor cores (indexer_bwd.cu): D_I 128, H_I <= 64
bool indexer_bwd_tc_supported(int H_I, int D_I);
cudaError_t launch_indexer_bwd_tc(const LaunchCtx& c, const KvMap& map, const uint8_t* q_I, const float* q_scale,
                                  const float* w, const uint8_t* k_I, const float* k_scale, const float* grad,
                                  long long ld, const int32_t* idx, int B, int T, int k, int H_I, int q_begin,
                                  int q_count, float* dq, float* dw, float* dk);

cudaError_t launch_wait_timeout_probe(const LaunchCtx& c);

// shape validation and launch context of the public entry points (dsa_api.cu)
dsa_status api_check_shape(const dsa_shape* s);
dsa_status api_make_ctx(void* stream, LaunchCtx* c);
// the key map (lengths, paged or contiguous caches) a shape describes
KvMap api_kv_map(const dsa_shape* s);

// split-k partial buffer size (floats) for a decode attention launch
size_t attn_partial_floats(int rows, int H, int d_v, int nsplit);
int attn_choose_nsplit(int rows, int H, int d_v, int k, int num_sms);

// the decode kernel (sparse_attn_decode.cu): MLA rows (d_k 576, d_v 512, V in
// the key row), splits of 128 selected slots, FP16 partials + FP32 LSE
bool attn_decode_supported(const AttnArgs& a);
int attn_decode_nsplit(int k);
size_t attn_decode_partial_bytes(int rows, int H, int nsplit);
cudaError_t launch_sparse_attn_decode(const LaunchCtx& c, const AttnArgs& a, void* part);

}  // namespace dsa
