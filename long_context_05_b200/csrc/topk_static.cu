// dsa_topk_static: the split (several blocks per row) top-k path with its
// per-row histograms in a fixed array in device global memory instead of a
// caller-supplied workspace, so the call allocates nothing, anywhere.
//
// Who needs that: a caller that has no device allocator of its own (a plain C
// host program that was handed device pointers for scores and indices and
// nothing else), or one that reserves all of HBM up front for weights and the
// key cache, where an allocation made later in a decode step could fail for
// lack of memory, and where cudaMalloc / cudaFree can synchronise the device
// and so stall the stream the step runs on.  The fixed array is part of the
// loaded module and costs nothing per call.
//
// Limits and sharing:
//   * at most kStaticRows score rows (B * q_count) per call; larger calls are
//     rejected with DSA_ERR_WORKSPACE before anything is launched;
//   * every call clears the histograms it uses (rows * 2048 words) at its
//     start, in stream order, so a call never sees the previous call's counts;
//   * all calls on a device share the one array: two calls whose launches can
//     run at the same time on the GPU (different streams without an ordering
//     between them, or different host threads) race on it and both may return
//     wrong indices.  Calls issued one after another on one stream are safe.
//   * the first call on each device looks up the array's device address
//     (cudaGetSymbolAddress, with that device current); make that first call
//     before any stream capture begins on the calling thread.
#include <mutex>

#include "internal.h"

namespace dsa {
namespace {

constexpr int kStaticRows = DSA_TOPK_STATIC_MAX_ROWS;
constexpr int kMaxDevices = 64;

// rows x 2048 bins of u32 = 512 KiB for 64 rows
__device__ __align__(256) unsigned int g_topk_static_hist[(size_t)kStaticRows * kTopkHistBins];

struct StaticScratch {
  unsigned int* hist = nullptr;
  bool ready = false;
};
StaticScratch g_scratch[kMaxDevices];
std::mutex g_scratch_mu;

// Address of the array on `device` (the current device).  Looked up once per
// device; later calls only read the cached pointer.
dsa_status static_hist(int device, unsigned int** out) {
  if (device < 0 || device >= kMaxDevices) return DSA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  StaticScratch& s = g_scratch[device];
  if (!s.ready) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_topk_static_hist) != cudaSuccess) return DSA_ERR_CUDA;
    s.hist = static_cast<unsigned int*>(p);
    s.ready = true;
  }
  *out = s.hist;
  return DSA_OK;
}

}  // namespace
}  // namespace dsa

using namespace dsa;

extern "C" dsa_status dsa_topk_static(const dsa_shape* s, const float* scores, int64_t ld_scores, int q_begin,
                                      int q_count, int32_t* idx, void* stream) {
  dsa_status st = api_check_shape(s);
  if (st != DSA_OK) return st;
  if (scores == nullptr || idx == nullptr || (reinterpret_cast<uintptr_t>(scores) & 15u) != 0)
    return DSA_ERR_INVALID_ARG;
  if (q_begin < 0 || q_count < 0 || q_begin + q_count > s->T) return DSA_ERR_INVALID_ARG;
  if (ld_scores < s->S || ld_scores % 4 != 0) return DSA_ERR_INVALID_ARG;
  if ((long long)s->B * q_count > kStaticRows) return DSA_ERR_WORKSPACE;
  LaunchCtx c;
  if ((st = api_make_ctx(stream, &c)) != DSA_OK) return st;
  unsigned int* hist = nullptr;
  if ((st = static_hist(c.device, &hist)) != DSA_OK) return st;
  TopkArgs a = {};
  a.kv = api_kv_map(s);
  a.scores = scores; a.ld = ld_scores; a.idx = idx;
  a.B = s->B; a.T = s->T; a.S = s->S; a.k = s->k;
  a.q_begin = q_begin; a.q_count = q_count;
  return launch_topk_split_into(c, a, hist) == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}
