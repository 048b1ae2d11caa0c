// Step C: sparse MQA/MLA attention over the selected keys.
//
// out[t,h] = sum_{s in idx[t]} softmax_s(tau q[t,h] . kv[s]) kv[s, :d_v]
// (ouchyi thread, "Nasil calisiyor" paragraph: the expensive attention runs
// only over the kept subset; tenelement.pl, section "Architektura ...",
// "Integracja z MLA" bullet: MQA form in decoding, one KV row shared by all
// heads; degnora.com, "MLA - Multi-Latent Attention": keys and values come
// from the one cached latent, so V is the first d_v columns of the row).
#include <cuda_bf16.h>

#include "internal.h"

namespace dsa {
namespace {

__device__ __forceinline__ float bf16_to_float(uint16_t u) {
  return __uint_as_float(((unsigned int)u) << 16);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

constexpr int kHeadsPerBlock = 8;

// One block: one query row, 8 heads, one warp per head; online softmax over
// the selected keys in slot order.
template <int DK, int DV>
__global__ void __launch_bounds__(32 * kHeadsPerBlock) sparse_attn_cuda_core_kernel(AttnArgs a, DevErr* err) {
  constexpr int NQ = (DK + 31) / 32;
  constexpr int NV = DV / 32;
  const int row = blockIdx.x;               // b * T + t
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y * kHeadsPerBlock + warp;
  if (h >= a.H) return;
  const int b = row / a.T;
  const uint16_t* qp = a.q + ((size_t)row * a.H + h) * DK;
  float qr[NQ];
#pragma unroll
  for (int c = 0; c < NQ; ++c) {
    const int d = lane + 32 * c;
    qr[c] = d < DK ? bf16_to_float(qp[d]) * a.tau : 0.f;
  }
  float o[NV];
#pragma unroll
  for (int c = 0; c < NV; ++c) o[c] = 0.f;
  float m = -INFINITY, l = 0.f;
  const int32_t* ir = a.idx + (size_t)row * a.k;
  const uint16_t* kvb = a.kv + (size_t)b * a.S * DK;
  for (int i = 0; i < a.k; ++i) {
    const int s = ir[i];
    if (s < 0) continue;
    if (s >= a.S) {
      if (lane == 0) report_error(err, DSA_ERR_DEVICE_BOUNDS, ERR_SITE_ATTN);
      continue;
    }
    const uint16_t* kr = kvb + (size_t)s * DK;
    float part = 0.f;
#pragma unroll
    for (int c = 0; c < NQ; ++c) {
      const int d = lane + 32 * c;
      if (d < DK) part = fmaf(qr[c], bf16_to_float(kr[d]), part);
    }
    const float z = warp_sum(part);
    const float mn = fmaxf(m, z);
    const float sc = expf(m - mn);
    const float p = expf(z - mn);
    l = l * sc + p;
#pragma unroll
    for (int c = 0; c < NV; ++c) o[c] = fmaf(o[c], sc, p * bf16_to_float(kr[lane + 32 * c]));
    m = mn;
  }
  const float inv = l > 0.f ? 1.f / l : 0.f;
  uint16_t* op = a.out + ((size_t)row * a.H + h) * DV;
#pragma unroll
  for (int c = 0; c < NV; ++c) {
    __nv_bfloat16 v = __float2bfloat16_rn(o[c] * inv);
    op[lane + 32 * c] = *reinterpret_cast<uint16_t*>(&v);
  }
  if (a.lse != nullptr && lane == 0) a.lse[(size_t)row * a.H + h] = l > 0.f ? m + logf(l) : -INFINITY;
}

}  // namespace

size_t attn_partial_floats(int rows, int H, int d_v, int nsplit) {
  return nsplit > 1 ? (size_t)rows * nsplit * H * (d_v + 2) : 0;
}

int attn_choose_nsplit(int rows, int H, int k, int num_sms) {
  (void)rows; (void)H; (void)k; (void)num_sms;
  return 1;
}

cudaError_t launch_sparse_attn(const LaunchCtx& c, const AttnArgs& a) {
  const int rows = a.B * a.T;
  if (rows <= 0) return cudaSuccess;
  dim3 grid(rows, (a.H + kHeadsPerBlock - 1) / kHeadsPerBlock);
  dim3 block(32 * kHeadsPerBlock);
  if (a.d_k == 576 && a.d_v == 512) {
    sparse_attn_cuda_core_kernel<576, 512><<<grid, block, 0, c.stream>>>(a, c.err);
  } else if (a.d_k == 80 && a.d_v == 64) {
    sparse_attn_cuda_core_kernel<80, 64><<<grid, block, 0, c.stream>>>(a, c.err);
  } else {
    return cudaErrorInvalidValue;
  }
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace dsa
