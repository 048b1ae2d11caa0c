// One sequence's keys spread over several parts (devices): the exchange
// steps of a key-split decode.
//
// The selection is exact top-k, so it decomposes over disjoint key ranges:
// an entry of the whole row's top-k has fewer than k better entries in the
// row, hence in its own range, so it is among its range's top-k under the
// same order (score descending, index ascending).  Each part therefore runs
// the indexer and the top-k over its own keys, and only k (score, index)
// candidates per part and row travel.  Attention is exact softmax, so it
// decomposes too: each part attends over the selected keys it holds, and the
// parts' results merge through their log-sum-exp (ouchyi thread on DeepSeek
// Sparse Attention, "Nasil calisiyor" paragraph: exact top-k, then attention
// over the kept entries only; the decomposition is arithmetic, not a step the
// pages describe).
//
//   dsa_topk_candidates: a part's selection as (score, global index) pairs;
//   dsa_topk_merge:      the global top-k of all parts' candidates, and the
//                        caller's share of it as local indices;
//   dsa_attn_combine:    O = sum_r e^(LSE_r - M) O_r / sum_r e^(LSE_r - M).
#include <math.h>

#include "internal.h"
#include "sm100.cuh"

namespace dsa {
namespace {

using namespace sm100;

// cand[r, x] = (scores[r, idx[r, x]], idx[r, x] + part_begin), or (-inf, -1)
// for an empty slot.  Row r of the scores holds query row r of the launch.
__global__ void topk_candidates_kernel(const float* scores, long long ld, const int32_t* idx, int rows, int k,
                                       int S, int part_begin, float* cand_scores, int32_t* cand_idx, DevErr* err) {
  const int r = blockIdx.x;
  if (r >= rows) return;
  for (int x = threadIdx.x; x < k; x += blockDim.x) {
    const int i = idx[(size_t)r * k + x];
    float sc = -INFINITY;
    int g = -1;
    if (i >= 0 && i < S) {
      sc = scores[(size_t)r * ld + i];
      g = part_begin + i;
    } else if (i >= S) {
      report_error(err, DSA_ERR_DEVICE_BOUNDS, ERR_SITE_TOPK | (0x30u << 8));
    }
    cand_scores[(size_t)r * k + x] = sc;
    cand_idx[(size_t)r * k + x] = g;
  }
}

// Merge the parts' attention results of each (row, head): d_v / 8 threads
// per (row, head), eight value columns each.
__global__ void __launch_bounds__(256) attn_combine_parts_kernel(const uint16_t* o_parts, const float* lse_parts,
                                                                 uint16_t* out, float* lse, int rows, int H,
                                                                 int dv, int nparts) {
  const int per = dv / 8;                       // threads per (row, head)
  const long long gh = (long long)blockIdx.x * (256 / per) + threadIdx.x / per;
  if (threadIdx.x >= (256 / per) * per || gh >= (long long)rows * H) return;
  const int d0 = (threadIdx.x % per) * 8;
  const size_t rh = (size_t)gh;                 // row * H + h
  const size_t stride = (size_t)rows * H;       // one part's [rows, H]
  float mx = -INFINITY;
  for (int r = 0; r < nparts; ++r) mx = fmaxf(mx, lse_parts[r * stride + rh]);
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  float wsum = 0.f;
  if (mx != -INFINITY) {
    for (int r = 0; r < nparts; ++r) {
      const float l = lse_parts[r * stride + rh];
      if (l == -INFINITY) continue;
      const float w = expf(l - mx);
      wsum += w;
      const uint4 v = *reinterpret_cast<const uint4*>(o_parts + (r * stride + rh) * dv + d0);
      const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        acc[2 * i] = fmaf(w, __uint_as_float(u[i] << 16), acc[2 * i]);
        acc[2 * i + 1] = fmaf(w, __uint_as_float(u[i] & 0xFFFF0000u), acc[2 * i + 1]);
      }
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  uint4 o;
  o.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
  o.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
  o.z = pack_bf16x2(acc[4] * inv, acc[5] * inv);
  o.w = pack_bf16x2(acc[6] * inv, acc[7] * inv);
  *reinterpret_cast<uint4*>(out + rh * dv + d0) = o;
  if (d0 == 0 && lse != nullptr) lse[rh] = wsum > 0.f ? mx + logf(wsum) : -INFINITY;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace dsa

using namespace dsa;

extern "C" dsa_status dsa_topk_candidates(const dsa_shape* s, const float* scores, int64_t ld_scores,
                                          const int32_t* idx, int32_t part_begin, float* cand_scores,
                                          int32_t* cand_idx, void* stream) {
  dsa_status st = api_check_shape(s);
  if (st != DSA_OK) return st;
  if (!scores || !idx || !cand_scores || !cand_idx || ld_scores < s->S || part_begin < 0) return DSA_ERR_INVALID_ARG;
  LaunchCtx c;
  if ((st = api_make_ctx(stream, &c)) != DSA_OK) return st;
  const int rows = s->B * s->T;
  topk_candidates_kernel<<<rows, 256, 0, c.stream>>>(scores, ld_scores, idx, rows, s->k, s->S, part_begin,
                                                     cand_scores, cand_idx, c.err);
  note_launches(1);
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

extern "C" dsa_status dsa_topk_merge(const dsa_shape* s, int nparts, const float* cand_scores,
                                     const int32_t* cand_idx, int32_t* idx, int32_t local_begin,
                                     int32_t local_count, int32_t* idx_local, void* stream) {
  dsa_status st = api_check_shape(s);
  if (st != DSA_OK) return st;
  if (nparts <= 0 || !cand_scores || !cand_idx || !idx || local_begin < 0 || local_count < 0)
    return DSA_ERR_INVALID_ARG;
  if ((long long)nparts * s->k > topk_merge_max_candidates()) return DSA_ERR_UNSUPPORTED;
  LaunchCtx c;
  if ((st = api_make_ctx(stream, &c)) != DSA_OK) return st;
  const cudaError_t e = launch_topk_merge(c, cand_scores, cand_idx, s->B * s->T, nparts, s->k, idx, local_begin,
                                          local_count, idx_local);
  return e == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

extern "C" dsa_status dsa_attn_combine(const dsa_shape* s, int nparts, const uint16_t* o_parts,
                                       const float* lse_parts, uint16_t* out, float* lse, void* stream) {
  dsa_status st = api_check_shape(s);
  if (st != DSA_OK) return st;
  if (nparts <= 0 || !o_parts || !lse_parts || !out || !aligned16(o_parts) || !aligned16(out))
    return DSA_ERR_INVALID_ARG;
  LaunchCtx c;
  if ((st = api_make_ctx(stream, &c)) != DSA_OK) return st;
  const long long rh = (long long)s->B * s->T * s->H;
  const int per = s->d_v / 8;
  const long long blocks = (rh + (256 / per) - 1) / (256 / per);
  attn_combine_parts_kernel<<<(unsigned)blocks, 256, 0, c.stream>>>(o_parts, lse_parts, out, lse, s->B * s->T,
                                                                    s->H, s->d_v, nparts);
  note_launches(1);
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}
