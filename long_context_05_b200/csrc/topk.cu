// Step B: per-query top-k over the visible part of a score row.
//
// Keep the min(k, n) best of the n = pos(t) + 1 visible scores, ties to the
// lower index (ouchyi thread, "Nasil calisiyor" paragraph: only the top-k
// key/value entries are kept, 2,048 per query; tenelement.pl, section
// "Architektura ...", "Selekcja top-k" bullet).  The selection stays on the
// device and reads the row straight from the score tile (sider.ai blog,
// "Uyarilar": no CPU-GPU ping-pong in candidate selection).
//
// Method: radix select on order-preserving 32-bit keys, one block per row.
// Each pass histograms the next 8 bits of the keys that still match the
// prefix found so far and picks the bucket holding the k-th largest key; after
// four passes the k-th largest key `thr` is known exactly, together with how
// many keys equal to it must be kept.  A last pass in index order writes every
// key above `thr` and the lowest-indexed keys equal to it.
#include "internal.h"

namespace dsa {
namespace {

constexpr int kTopkThreads = 1024;
constexpr int kTopkWarps = kTopkThreads / 32;

// float -> unsigned with the same order; -0.0 is folded onto +0.0
__device__ __forceinline__ unsigned int order_key(float f) {
  unsigned int u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__global__ void __launch_bounds__(kTopkThreads) topk_radix_kernel(TopkArgs a) {
  __shared__ unsigned int hist[256];
  __shared__ unsigned int s_digit, s_krem;
  __shared__ int s_count, s_eq_base;
  __shared__ int warp_eq[kTopkWarps];

  const int r = blockIdx.x;
  const int b = r / a.q_count;
  const int i = r - b * a.q_count;
  const int t = a.q_begin + i;
  const int n = a.S - a.T + t + 1;  // visible keys
  const int k = a.k;
  const float* row = a.scores + (size_t)r * a.ld;
  int32_t* out = a.idx + ((size_t)b * a.T + t) * k;
  const int tid = threadIdx.x;

  if (n <= k) {
    for (int x = tid; x < k; x += kTopkThreads) out[x] = x < n ? x : -1;
    return;
  }

  unsigned int prefix = 0u, mask = 0u;
  unsigned int krem = (unsigned int)k;  // rank of the wanted key among the matching ones
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int x = tid; x < 256; x += kTopkThreads) hist[x] = 0u;
    __syncthreads();
    for (int x = tid; x < n; x += kTopkThreads) {
      const unsigned int key = order_key(row[x]);
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (tid == 0) {
      unsigned int cum = 0u;
      int d = 255;
      for (; d > 0; --d) {
        if (cum + hist[d] >= krem) break;
        cum += hist[d];
      }
      s_digit = (unsigned int)d;
      s_krem = krem - cum;
    }
    __syncthreads();
    prefix |= s_digit << shift;
    mask |= 255u << shift;
    krem = s_krem;
    __syncthreads();
  }
  const unsigned int thr = prefix;  // the k-th largest key; keep krem copies of it

  if (tid == 0) {
    s_count = 0;
    s_eq_base = 0;
  }
  __syncthreads();
  const int lane = tid & 31, warp = tid >> 5;
  for (int base = 0; base < n; base += kTopkThreads) {
    const int x = base + tid;
    const bool valid = x < n;
    const unsigned int key = valid ? order_key(row[x]) : 0u;
    const bool gt = valid && key > thr;
    const bool eq = valid && key == thr;
    if (gt) out[atomicAdd(&s_count, 1)] = x;
    const unsigned int bal = __ballot_sync(0xffffffffu, eq);
    if (lane == 0) warp_eq[warp] = __popc(bal);
    __syncthreads();
    int before = s_eq_base;
    for (int w = 0; w < warp; ++w) before += warp_eq[w];
    before += __popc(bal & ((1u << lane) - 1u));
    if (eq && before < (int)krem) out[atomicAdd(&s_count, 1)] = x;
    __syncthreads();
    if (tid == 0) {
      int tot = 0;
      for (int w = 0; w < kTopkWarps; ++w) tot += warp_eq[w];
      s_eq_base += tot;
    }
    __syncthreads();
  }
}

}  // namespace

cudaError_t launch_topk(const LaunchCtx& c, const TopkArgs& a) {
  const int rows = a.B * a.q_count;
  if (rows <= 0) return cudaSuccess;
  topk_radix_kernel<<<rows, kTopkThreads, 0, c.stream>>>(a);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace dsa
