// Step A: lightning indexer scores.
//
// I[t,s] = sum_j w[t,j] * ReLU(q_I[t,j] . k_I[s]) over the dequantised FP8
// operands (ouchyi thread on DeepSeek Sparse Attention, "Nasil calisiyor"
// paragraph: few heads, FP8, cheap; tenelement.pl, "DeepSeek V3.2-Exp Cuts
// Long-Context Costs ...", section "Architektura DeepSeek V3.2-Exp: Od MoE do
// DSA": logits for the context tokens through a ReLU).  Both scales are > 0,
// so ReLU(a b x) = a b ReLU(x): the kernel folds w * q_scale per query head
// and k_scale per key after the ReLU and works on the raw e4m3 values.
#include <cuda_fp8.h>

#include "internal.h"

namespace dsa {
namespace {

__device__ __forceinline__ float e4m3_to_float(uint8_t b) {
  __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(b), __NV_E4M3);
  return __half2float(__half(h));
}

constexpr int kKeysPerBlock = 128;

// One block: one query t of sequence b, 128 consecutive keys; one thread per key.
template <int DI>
__global__ void __launch_bounds__(kKeysPerBlock) indexer_cuda_core_kernel(IndexerArgs a) {
  extern __shared__ float smem[];
  float* qf = smem;                 // [H_I][DI] raw e4m3 values
  float* wq = smem + a.H_I * DI;    // [H_I] w * q_scale
  const int b = blockIdx.z;
  const int i = blockIdx.y;
  const int t = a.q_begin + i;
  const int pos = a.S - a.T + t;
  const int s0 = blockIdx.x * kKeysPerBlock;
  if (s0 > pos) return;

  const size_t qrow = (size_t)b * a.T + t;
  const uint8_t* qp = a.q_I + qrow * a.H_I * DI;
  for (int x = threadIdx.x; x < a.H_I * DI; x += blockDim.x) qf[x] = e4m3_to_float(qp[x]);
  for (int j = threadIdx.x; j < a.H_I; j += blockDim.x)
    wq[j] = a.w[qrow * a.H_I + j] * a.q_scale[qrow * a.H_I + j];
  __syncthreads();

  const int s = s0 + threadIdx.x;
  if (s > pos) return;
  const uint8_t* kp = a.k_I + ((size_t)b * a.S + s) * DI;
  float kf[DI];
#pragma unroll
  for (int d = 0; d < DI; d += 16) {
    uint4 v = *reinterpret_cast<const uint4*>(kp + d);
    const uint8_t* vb = reinterpret_cast<const uint8_t*>(&v);
#pragma unroll
    for (int e = 0; e < 16; ++e) kf[d + e] = e4m3_to_float(vb[e]);
  }
  float acc = 0.f;
  for (int j = 0; j < a.H_I; ++j) {
    const float* qj = qf + j * DI;
    float dot = 0.f;
#pragma unroll
    for (int d = 0; d < DI; ++d) dot = fmaf(qj[d], kf[d], dot);
    acc = fmaf(wq[j], fmaxf(dot, 0.f), acc);
  }
  a.scores[((size_t)b * a.q_count + i) * a.ld + s] = acc * a.k_scale[(size_t)b * a.S + s];
}

}  // namespace

cudaError_t launch_indexer(const LaunchCtx& c, const IndexerArgs& a) {
  if (a.q_count <= 0 || a.B <= 0) return cudaSuccess;
  const int last_pos = a.S - a.T + a.q_begin + a.q_count - 1;
  dim3 grid((last_pos + kKeysPerBlock) / kKeysPerBlock, a.q_count, a.B);
  size_t smem = (size_t)(a.H_I * a.D_I + a.H_I) * sizeof(float);
  switch (a.D_I) {
    case 32: indexer_cuda_core_kernel<32><<<grid, kKeysPerBlock, smem, c.stream>>>(a); break;
    case 64: indexer_cuda_core_kernel<64><<<grid, kKeysPerBlock, smem, c.stream>>>(a); break;
    case 128: indexer_cuda_core_kernel<128><<<grid, kKeysPerBlock, smem, c.stream>>>(a); break;
    default: return cudaErrorInvalidValue;
  }
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace dsa
