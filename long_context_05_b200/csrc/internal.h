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
#endif

// Everything a launcher needs besides its own arguments.
struct LaunchCtx {
  cudaStream_t stream;
  DevErr* err;            // device address of this device's error word
  long long wait_ns;      // wall-clock limit of a bounded wait
  int num_sms;
  int device;
};

struct IndexerArgs {
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
  const float* scores;
  int64_t ld;
  int32_t* idx;
  int B, T, S, k;
  int q_begin, q_count;
};

struct AttnArgs {
  const uint16_t* q;
  const uint16_t* kv;
  const int32_t* idx;
  uint16_t* out;
  float* lse;
  float* part;         // split partials [rows, nsplit, H, d_v + 2] or null
  int B, T, S, H, d_k, d_v, k;
  int nsplit;          // key splits per query row (1 = write out directly)
  float tau;
};

// counts every kernel launch (dsa_launch_count)
void note_launches(int n);

cudaError_t launch_indexer(const LaunchCtx& c, const IndexerArgs& a);
// ws: optional scratch for the split path (few long rows); see topk.cu
cudaError_t launch_topk(const LaunchCtx& c, const TopkArgs& a, void* ws, size_t ws_bytes);
size_t topk_workspace_bytes(int rows);
// top-k split path into an explicit histogram array of rows * 2048 words
cudaError_t launch_topk_split_into(const LaunchCtx& c, const TopkArgs& a, unsigned int* hist);
constexpr int kTopkHistBins = 2048;
bool topk_uses_workspace(int rows, int S, int num_sms);
cudaError_t launch_sparse_attn(const LaunchCtx& c, const AttnArgs& a);

cudaError_t launch_wait_timeout_probe(const LaunchCtx& c);

// shape validation and launch context of the public entry points (dsa_api.cu)
dsa_status api_check_shape(const dsa_shape* s);
dsa_status api_make_ctx(void* stream, LaunchCtx* c);

// split-k partial buffer size (floats) for a decode attention launch
size_t attn_partial_floats(int rows, int H, int d_v, int nsplit);
int attn_choose_nsplit(int rows, int H, int d_v, int k, int num_sms);

}  // namespace dsa
