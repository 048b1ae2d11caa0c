// Training the lightning indexer, kernel level (tenelement.pl, "DeepSeek
// V3.2-Exp Cuts Long-Context Costs ...", section "Proces Treningu DSA: Od
// Warm-up do Sparsity": the indexer learns the main attention's distribution
// through a KL divergence, first densely with the main model frozen, then
// over the top-k set; its gradients stay apart from the main loss).
//
// Readings where the pages are silent: the target of query t is the main
// attention's weights summed over heads and divided by H; the loss is
// KL(target || softmax(I[t, .])) over the visible keys (warm-up) or over the
// selected set (sparse stage); the target is a constant.
//
//   dsa_kl_target:         p[t, s] = (1/H) sum_h exp(tau q_h . kv_s - lse_h)
//                          with lse from the main attention (dense: every
//                          visible key; sparse: the selected set, where lse
//                          is the sparse attention's), on tcgen05: one CTA
//                          per query with Q resident in TMEM, Q K^T per
//                          64-key chunk, the head sum in the epilogue;
//   dsa_indexer_kl:        per row, loss and dL/dI = softmax(I) - p;
//   dsa_indexer_backward:  dL/dw, dL/dq_I, dL/dk_I through the ReLU, on the
//                          dequantised operands: on tcgen05 for D_I = 128
//                          (indexer_bwd.cu), FP32 on the CUDA cores here
//                          otherwise.
#include <cuda_fp8.h>
#include <math.h>

#include "internal.h"
#include "sm100.cuh"
#include "tma_host.h"

namespace dsa {
namespace {

using namespace sm100;

// ------------------------------------------------------------------ KL target

// One CTA per query row.  All of the row's Q (128 heads x 576 dims, BF16)
// sits in TMEM for the whole row, so every MMA reads A from TMEM; it gets
// there through the first two ring slots (each thread copies its own head
// row in, swizzled so the read-back is free of bank conflicts) while the
// first chunk of keys lands in the third.  The keys stream through the ring
// of three 64-key slots (128B-swizzled K-major atoms laid out
// [slot][atom][row]); chunk j uses slot (j + 2) mod 3.  Per 64-key chunk: S = Q K^T
// (36 MMAs of 128 x 64 x 16) into one of two TMEM buffers, then the head sum
// of exp(tau S - lse_h) on eight warps: each warp reduces its 32 heads for 32
// keys with one transpose-reduce over the lanes (31 shuffles), the four lane
// quarters meet in shared memory, and one warp per key half writes the row's
// target entries.
constexpr int DK = 576;
constexpr int kChunk = 64, kSlots = 3, kNAtom = DK / 64;
constexpr int kAtomBytes = kChunk * 128, kSlotBytes = kNAtom * kAtomBytes;
constexpr int kKSteps = DK / 16;
constexpr uint32_t kTmemCols = 512, kQCol = 0, kSCol = 384;      // Q [0, 288), S x2 [384, 512)
constexpr int kFirstGather = 1, kGatherWarps = 6, kFirstEpi = 7, kEpiWarps = 8;
constexpr int kThreads = 32 * (kFirstEpi + kEpiWarps);
constexpr int kGatherThreads = 32 * kGatherWarps;
constexpr int OFF_KV = 0;
constexpr int OFF_SUM = OFF_KV + kSlots * kSlotBytes;     // head sums, two chunk buffers (float)
constexpr int OFF_BAR = OFF_SUM + 2 * kChunk * 4;
constexpr int kNumBars = 1 + 2 * kSlots + 2 + 2 + 1;       // q_ready, kv_full[3], kv_empty[3], s_full[2], s_empty[2], mma_done
constexpr int OFF_MISC = OFF_BAR + kNumBars * 8;
constexpr int kSmem = OFF_MISC + 16;
static_assert(kSmem <= 232448, "shared memory per CTA");
static_assert(kGatherThreads == 3 * kChunk, "three gather threads per key row");
static_assert(128 * DK * 2 <= 2 * kSlotBytes, "Q fits the first two slots");

struct TargetParams {
  KvMap map;
  const uint16_t* q;
  const uint16_t* kv;
  const float* lse;       // [rows_all, H] natural log, the main attention's
  const int32_t* idx;     // null: dense (keys 0..pos)
  float* target;
  long long ld;
  int T, H, k, q_begin, q_count, B;
  float scale_log2;
  bool tma_keys;          // every visible key, contiguous cache: chunks by TMA tiles
  long long wait_ns;
  DevErr* err;
};

// v[i] over the warp's lanes, summed: lane l returns sum over lanes of v[l]
__device__ __forceinline__ float transpose_reduce32(float (&v)[32], int lane) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < off; ++i) {
      const float send = upper ? v[i] : v[i + off];
      const float keep = upper ? v[i + off] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
  }
  return v[0];
}

__global__ void __launch_bounds__(kThreads, 1)
    kl_target_kernel(const __grid_constant__ CUtensorMap tm_kv, TargetParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) report_error(p.err, DSA_ERR_DEVICE_BOUNDS, ERR_SITE_ATTN | (0xDu << 8));
    return;
  }
  uint8_t* sKV = smem + OFF_KV;
  float* sSum = reinterpret_cast<float*>(smem + OFF_SUM);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* q_ready = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = kv_full + kSlots;
  uint64_t* s_full = kv_empty + kSlots;
  uint64_t* s_empty = s_full + 2;
  uint64_t* mma_done = s_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int lr = blockIdx.x;                       // row of the launch: b * q_count + i
  const int b = lr / p.q_count, t = p.q_begin + (lr - (lr / p.q_count) * p.q_count);
  const int row = b * p.T + t;                     // query row of the problem
  const int Lb = p.map.len(b, p.err, ERR_SITE_ATTN);
  const int n = Lb - p.T + t + 1;                  // visible keys
  const bool dense = p.idx == nullptr;
  const int m = dense ? n : p.k;                   // key slots of the row
  const int nch = (m + kChunk - 1) / kChunk;

  if (threadIdx.x == 0) {
    mbar_init(q_ready, kEpiWarps);
    for (int i = 0; i < kSlots; ++i) {
      mbar_init(&kv_full[i], p.tma_keys ? 1 : kGatherThreads);
      mbar_init(&kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], kEpiWarps);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  for (int i = threadIdx.x; i < 2 * kChunk; i += kThreads) sSum[i] = 0.f;
  if (warp == 0) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const AbortSources ab{abort_flag, &p.err->code};
  const AbortSources no_abort{nullptr, nullptr};
  auto fail = [&](unsigned where) {
    report_error(p.err, DSA_ERR_TIMEOUT, ERR_SITE_ATTN | ((0x60u + where) << 8));
    *abort_flag = 1;
  };
  auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
    const bool r = mbar_wait(bar, parity, p.wait_ns, ab);
    return __all_sync(0xffffffffu, r);
  };

  if (warp >= kFirstGather && warp < kFirstEpi) {
    const int gt = threadIdx.x - 32 * kFirstGather;
    if (p.tma_keys) {
      // ---------------------------------------------------------- keys 0.. of a contiguous cache: one
      // thread loads each chunk as nine 64 x 64 tiles (rows past the cache read as zero)
      if (gt == 0) {
        prefetch_tmap(&tm_kv);
        const int row0 = (int)p.map.row_contig(b, 0);
        int issued = 0;
        for (int j = 0; j < nch; ++j) {
          const int sl = (j + 2) % kSlots;
          if (j >= kSlots ? !mbar_wait(&kv_empty[sl], ((j / kSlots) - 1) & 1, p.wait_ns, ab)
                          : (j >= 1 && !mbar_wait(q_ready, 0, p.wait_ns, ab))) {
            fail(1);
            break;
          }
          mbar_arrive_expect_tx(&kv_full[sl], kSlotBytes);
          for (int a = 0; a < kNAtom; ++a)
            tma_load_2d(sKV + sl * kSlotBytes + a * kAtomBytes, &tm_kv, &kv_full[sl], a * 64, row0 + j * kChunk);
          issued = j + 1;
        }
        // drain: the last loads of each slot land before the CTA's memory is released
        for (int j = issued > kSlots ? issued - kSlots : 0; j < issued; ++j)
          mbar_wait(&kv_full[(j + 2) % kSlots], (j / kSlots) & 1, p.wait_ns, no_abort);
      }
    } else {
    // ------------------------------------------------------------ gather: three threads per key row
    const int r = gt / 3, part = gt - 3 * (gt / 3);     // row of the slot; 24 of its 72 chunks
    for (int j = 0; j < nch; ++j) {
      const int sl = (j + 2) % kSlots;
      // slots 0 and 1 hold Q until it is in TMEM; later uses wait for the MMAs
      if (j >= kSlots ? !wwait(&kv_empty[sl], ((j / kSlots) - 1) & 1) : (j >= 1 && !wwait(q_ready, 0))) {
        fail(1);
        break;
      }
      const int slot = j * kChunk + r;
      int v = -1;
      if (slot < m) v = dense ? slot : p.idx[(size_t)row * p.k + slot];
      if (v >= Lb) {
        if (part == 0) report_error(p.err, DSA_ERR_DEVICE_BOUNDS, ERR_SITE_ATTN);
        v = -1;
      }
      if (v >= n) v = -1;
      const long long cr = v >= 0 ? p.map.row(b, v) : -1;
      if (v >= 0 && cr < 0) {
        if (part == 0) report_error(p.err, DSA_ERR_DEVICE_BOUNDS, ERR_SITE_ATTN | (1u << 8));
        v = -1;
      }
      const bool valid = v >= 0;
      const uint16_t* src = p.kv + (size_t)(valid ? cr : 0) * DK;
      uint8_t* dst = sKV + sl * kSlotBytes;
#pragma unroll 4
      for (int cc = 0; cc < 24; ++cc) {
        const int c = part * 24 + cc;                   // 16-byte chunk of the row: atom c / 8, chunk c % 8
        const int a = c >> 3, c16 = c & 7;
        cp_async16_zfill(dst + a * kAtomBytes + r * 128 + ((c16 ^ (r & 7)) << 4), src + c * 8, valid ? 16u : 0u);
      }
      cp_async_arrive(&kv_full[sl]);
    }
    cp_async_commit();
    cp_async_wait<0>();                            // every copy landed before the CTA can exit
    }
  } else if (warp == 0) {
    // ------------------------------------------------------------ Q K^T
    if (lane == 0) {
      constexpr uint32_t idesc_qk = make_idesc(kFmtBF16, kFmtBF16, 0, 0, 128, kChunk);
      bool ok = mbar_wait(q_ready, 0, p.wait_ns, ab);
      if (!ok) fail(2);
      for (int j = 0; j < nch && ok; ++j) {
        const int sl = (j + 2) % kSlots;
        if (!mbar_wait(&kv_full[sl], (j / kSlots) & 1, p.wait_ns, ab)) { fail(3); ok = false; break; }
        if (j >= 2 && !mbar_wait(&s_empty[j & 1], ((j - 2) >> 1) & 1, p.wait_ns, ab)) { fail(4); ok = false; break; }
        fence_proxy_async_smem();                   // the gather's cp.async bytes, before the tensor core reads them
        tc_fence_after();
        const uint32_t dS = tmem + kSCol + (j & 1) * kChunk;
        const uint64_t kdesc0 = make_sdesc(smem_u32(sKV + sl * kSlotBytes), 16, 1024, kSwizzle128);
#pragma unroll
        for (int ks = 0; ks < kKSteps; ++ks) {
          const int d = ks * 16;
          const uint64_t bdesc = kdesc0 + (uint64_t)(((d / 64) * kAtomBytes + (d % 64) * 2) >> 4);
          mma_bf16_ts(dS, tmem + kQCol + ks * 8, bdesc, idesc_qk, ks > 0 ? 1u : 0u);
        }
        mma_commit(&s_full[j & 1]);
        mma_commit(&kv_empty[sl]);
      }
      mma_commit(mma_done);
      mbar_wait(mma_done, 0, p.wait_ns, no_abort);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ head sum
    const int side = (warp - kFirstEpi) >> 2;      // key half of each chunk; dims half of Q
    const int quarter = warp & 3;
    const int h = quarter * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
    const bool head_ok = h < p.H;
    {
      // Q dims [288 side, 288 side + 288) of head h: global -> slots 0-1
      // (own row, 16-byte chunk c of the 72 at h * 1152 + (c / 8) * 128 +
      // ((c % 8) ^ (h % 8)) * 16) -> registers -> TMEM as BF16 pairs
      const uint16_t* qrow = p.q + ((size_t)row * p.H + (head_ok ? h : 0)) * DK;
      uint8_t* qs = sKV + h * (DK * 2);
#pragma unroll 4
      for (int cc = 0; cc < 36; ++cc) {
        const int c = side * 36 + cc;
        cp_async16_zfill(qs + (c >> 3) * 128 + (((c & 7) ^ (h & 7)) << 4), qrow + c * 8, head_ok ? 16u : 0u);
      }
      cp_async_commit();
      cp_async_wait<0>();
#pragma unroll 1
      for (int qb = 0; qb < 5; ++qb) {
        const int nv = qb < 4 ? 8 : 4;             // chunks of this block: 64 dims, the last 32
        uint32_t v[32];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          uint4 x = make_uint4(0u, 0u, 0u, 0u);
          const int c = side * 36 + qb * 8 + i;
          if (i < nv) x = *reinterpret_cast<const uint4*>(qs + (c >> 3) * 128 + (((c & 7) ^ (h & 7)) << 4));
          v[4 * i] = x.x; v[4 * i + 1] = x.y; v[4 * i + 2] = x.z; v[4 * i + 3] = x.w;
        }
        const uint32_t col = tmem + lane_addr + kQCol + side * (DK / 4) + qb * 32;
        if (qb < 4) tmem_st32(col, v);
        else tmem_st16(col, v);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(q_ready);
    }
    const float lse2 = head_ok ? p.lse[(size_t)row * p.H + h] * 1.4426950408889634f : INFINITY;
    const float sc = p.scale_log2;
    const float inv_h = 1.0f / (float)p.H;
    float* target = p.target + (size_t)lr * p.ld;
    // every warp takes every iteration (a failed wait only skips the work),
    // so the named barriers below always fill
    bool ok = true;
    for (int j = 0; j < nch; ++j) {
      float part = 0.f;
      if (ok && !wwait(&s_full[j & 1], (j >> 1) & 1)) {
        fail(5);
        ok = false;
      }
      if (ok) {
        tc_fence_after();
        uint32_t s[32];
        tmem_ld32(tmem + lane_addr + kSCol + (j & 1) * kChunk + side * 32, s);
        tmem_wait_ld_dep(s);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_empty[j & 1]);
        float e[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) e[i] = exp2f(fmaf(__uint_as_float(s[i]), sc, -lse2));
        part = transpose_reduce32(e, lane);          // this warp's 32 heads, key side * 32 + lane
      }
      float* sum = sSum + (j & 1) * kChunk + side * 32 + lane;
      if (ok) atomicAdd(sum, part);
      // the four quarters of this key half meet; quarter 0 writes the keys
      asm volatile("bar.sync %0, %1;" ::"r"(1 + side), "n"(128) : "memory");
      if (quarter == 0) {
        // the key of this slot, as the gather read it
        const int slot = j * kChunk + side * 32 + lane;
        int key = -1;
        if (slot < m) key = dense ? slot : p.idx[(size_t)row * p.k + slot];
        if (key >= n || (key >= 0 && p.map.row(b, key) < 0)) key = -1;
        if (ok && key >= 0) target[key] = *sum * inv_h;
        *sum = 0.f;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------ KL and dL/dI

// Block reductions over 256 threads.
__device__ __forceinline__ float block_max(float v, float* red) {
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float r = -INFINITY;
  for (int i = 0; i < 8; ++i) r = fmaxf(r, red[i]);
  __syncthreads();
  return r;
}
__device__ __forceinline__ float block_sum(float v, float* red) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float r = 0.f;
  for (int i = 0; i < 8; ++i) r += red[i];
  __syncthreads();
  return r;
}

// One block per launch row: over the set (keys 0..pos, or the idx row),
// lq = I - max - ln sum exp(I - max), loss = sum p (ln p - lq) over p > 0,
// grad = exp(lq) - p; grad is 0 at visible keys outside the set.
__global__ void __launch_bounds__(256) indexer_kl_kernel(KvMap map, const float* scores, const float* target,
                                                         long long ld, const int32_t* idx, int T, int k, int q_begin,
                                                         int q_count, float* grad, float* loss, DevErr* err) {
  __shared__ float red[8];
  const int lr = blockIdx.x;
  const int b = lr / q_count, t = q_begin + (lr - (lr / q_count) * q_count);
  const int n = map.len(b, err, ERR_SITE_TOPK) - T + t + 1;
  const float* I = scores + (size_t)lr * ld;
  const float* P = target + (size_t)lr * ld;
  float* G = grad + (size_t)lr * ld;
  const int32_t* set = idx ? idx + ((size_t)b * T + t) * k : nullptr;
  const int m = set ? k : n;                       // set entries (idx slots may be -1)
  auto key_of = [&](int i) -> int {
    if (!set) return i;
    const int s = set[i];
    return (s >= 0 && s < n) ? s : -1;
  };
  float mx = -INFINITY;
  for (int i = threadIdx.x; i < m; i += 256) {
    const int s = key_of(i);
    if (s >= 0) mx = fmaxf(mx, I[s]);
  }
  mx = block_max(mx, red);
  float z = 0.f;
  for (int i = threadIdx.x; i < m; i += 256) {
    const int s = key_of(i);
    if (s >= 0) z += expf(I[s] - mx);
  }
  z = block_sum(z, red);
  const float lz = logf(z);
  if (set) {
    for (int s = threadIdx.x; s < n; s += 256) G[s] = 0.f;
    __syncthreads();
  }
  float l = 0.f;
  for (int i = threadIdx.x; i < m; i += 256) {
    const int s = key_of(i);
    if (s < 0) continue;
    const float lq = I[s] - mx - lz;
    const float ps = P[s];
    G[s] = expf(lq) - ps;
    if (ps > 0.f) l += ps * (logf(ps) - lq);
  }
  l = block_sum(l, red);
  if (threadIdx.x == 0) loss[lr] = l;
}

// ------------------------------------------------------------------ backward to the indexer's inputs

constexpr int kBT = 64;   // keys per tile

__device__ __forceinline__ float e4m3_value(uint8_t x) {
  __nv_fp8_e4m3 v;
  v.__x = x;
  return float(v);
}

// One block per launch row t, over its keys (0..pos, or the idx row) in
// tiles of 64; FP32 on the dequantised operands:
//   D[j, s] = q_j . k_s,   M[j, s] = g_s w_j [D > 0]
//   dw_j += sum_s g_s ReLU(D[j, s]),  dq_j += sum_s M[j, s] k_s,
//   dk_s += sum_j M[j, s] q_j  (atomic: every row adds to the shared keys).
template <int HI, int DI>
__global__ void __launch_bounds__(256) indexer_bwd_kernel(KvMap map, const uint8_t* q_I, const float* q_scale,
                                                          const float* w, const uint8_t* k_I, const float* k_scale,
                                                          const float* grad, long long ld, const int32_t* idx,
                                                          int T, int k, int q_begin, int q_count, float* dq,
                                                          float* dw, float* dk, DevErr* err) {
  // shared memory (dynamic): sQ [HI][DI+1] | sK [kBT][DI+1] | sM [HI][kBT+1] |
  // sW [HI] | sG [kBT] | sS [kBT] | sDw [HI]  (the +1 pads keep rows off one bank)
  extern __shared__ float bsm[];
  float (*sQ)[DI + 1] = reinterpret_cast<float (*)[DI + 1]>(bsm);
  float (*sK)[DI + 1] = reinterpret_cast<float (*)[DI + 1]>(bsm + HI * (DI + 1));
  float (*sM)[kBT + 1] = reinterpret_cast<float (*)[kBT + 1]>(bsm + (HI + kBT) * (DI + 1));
  float* sW = bsm + (HI + kBT) * (DI + 1) + HI * (kBT + 1);
  float* sG = sW + HI;
  int* sS = reinterpret_cast<int*>(sG + kBT);
  float* sDw = reinterpret_cast<float*>(sS + kBT);
  const int lr = blockIdx.x;
  const int b = lr / q_count, t = q_begin + (lr - (lr / q_count) * q_count);
  const int n = map.len(b, err, ERR_SITE_INDEXER) - T + t + 1;
  const size_t qrow = ((size_t)b * T + t) * HI;
  for (int x = threadIdx.x; x < HI * DI; x += 256) {
    const int j = x / DI, d = x - (x / DI) * DI;
    sQ[j][d] = e4m3_value(q_I[qrow * DI + x]) * q_scale[qrow + j];
  }
  for (int j = threadIdx.x; j < HI; j += 256) {
    sW[j] = w[qrow + j];
    sDw[j] = 0.f;
  }
  const int32_t* set = idx ? idx + ((size_t)b * T + t) * k : nullptr;
  const int m = set ? k : n;
  const float* G = grad + (size_t)lr * ld;
  // dq accumulators: thread owns heads jq..jq+QJ-1, dims dq0..dq0+7
  constexpr int QJ = HI * DI / (256 * 8);          // heads per thread (>= 1 for HI*DI >= 2048)
  static_assert(QJ >= 1 && HI * DI == QJ * 8 * 256, "dq tiling");
  const int dq_d0 = (threadIdx.x % (DI / 8)) * 8;
  const int dq_j0 = (threadIdx.x / (DI / 8)) * QJ;
  float accq[QJ][8];
#pragma unroll
  for (int a = 0; a < QJ; ++a)
#pragma unroll
    for (int c = 0; c < 8; ++c) accq[a][c] = 0.f;
  __syncthreads();
  for (int i0 = 0; i0 < m; i0 += kBT) {
    // keys of the tile, their gradients and dequantised rows
    for (int i = threadIdx.x; i < kBT; i += 256) {
      int s = -1;
      if (i0 + i < m) {
        s = set ? set[i0 + i] : i0 + i;
        if (s >= n) s = -1;
      }
      sS[i] = s;
      sG[i] = s >= 0 ? G[s] : 0.f;
    }
    __syncthreads();
    for (int x = threadIdx.x; x < kBT * DI; x += 256) {
      const int i = x / DI, d = x - (x / DI) * DI;
      const int s = sS[i];
      const long long kr = s >= 0 ? map.row(b, s) : -1;
      sK[i][d] = kr >= 0 ? e4m3_value(k_I[kr * DI + d]) * k_scale[kr] : 0.f;
    }
    __syncthreads();
    // D and M: thread computes (HI * kBT) / 256 entries
    for (int x = threadIdx.x; x < HI * kBT; x += 256) {
      const int j = x / kBT, i = x - (x / kBT) * kBT;
      float dsum = 0.f;
#pragma unroll 8
      for (int d = 0; d < DI; ++d) dsum = fmaf(sQ[j][d], sK[i][d], dsum);
      const float g = sG[i];
      sM[j][i] = dsum > 0.f ? g * sW[j] : 0.f;
      if (dsum > 0.f && g != 0.f) atomicAdd(&sDw[j], g * dsum);
    }
    __syncthreads();
    // dq_j += sum_i M[j, i] k_i
#pragma unroll
    for (int a = 0; a < QJ; ++a) {
      const int j = dq_j0 + a;
      for (int i = 0; i < kBT; ++i) {
        const float mv = sM[j][i];
#pragma unroll
        for (int c = 0; c < 8; ++c) accq[a][c] = fmaf(mv, sK[i][dq_d0 + c], accq[a][c]);
      }
    }
    // dk_i += sum_j M[j, i] q_j: thread owns key i, dims d0..d0+DI*kBT/256-1
    {
      constexpr int KD = DI * kBT / 256;              // dims per thread
      const int i = threadIdx.x / (DI / KD);
      const int d0 = (threadIdx.x % (DI / KD)) * KD;
      const int s = sS[i];
      if (s >= 0) {
        float acc[KD];
#pragma unroll
        for (int c = 0; c < KD; ++c) acc[c] = 0.f;
        for (int j = 0; j < HI; ++j) {
          const float mv = sM[j][i];
          if (mv == 0.f) continue;
#pragma unroll
          for (int c = 0; c < KD; ++c) acc[c] = fmaf(mv, sQ[j][d0 + c], acc[c]);
        }
        const long long kr = map.row(b, s);
        if (kr >= 0) {
          float* dst = dk + kr * DI + d0;
#pragma unroll
          for (int c = 0; c < KD; ++c)
            if (acc[c] != 0.f) atomicAdd(dst + c, acc[c]);
        }
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int a = 0; a < QJ; ++a)
#pragma unroll
    for (int c = 0; c < 8; ++c) dq[(qrow + dq_j0 + a) * DI + dq_d0 + c] = accq[a][c];
  for (int j = threadIdx.x; j < HI; j += 256) dw[qrow + j] = sDw[j];
}

template <int HI, int DI>
cudaError_t launch_bwd_t(const LaunchCtx& c, const KvMap& map, const uint8_t* q_I, const float* q_scale,
                         const float* w, const uint8_t* k_I, const float* k_scale, const float* grad, long long ld,
                         const int32_t* idx, int B, int T, int k, int q_begin, int q_count, float* dq, float* dw,
                         float* dk) {
  const int smem = ((HI + kBT) * (DI + 1) + HI * (kBT + 1) + 2 * HI + 2 * kBT) * 4;
  cudaError_t e = cudaFuncSetAttribute(indexer_bwd_kernel<HI, DI>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  indexer_bwd_kernel<HI, DI><<<B * q_count, 256, smem, c.stream>>>(map, q_I, q_scale, w, k_I, k_scale, grad, ld, idx,
                                                                   T, k, q_begin, q_count, dq, dw, dk, c.err);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace
}  // namespace dsa

using namespace dsa;

namespace {
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
}  // namespace

extern "C" dsa_status dsa_kl_target(const dsa_shape* s, const uint16_t* q, const uint16_t* kv, const float* lse,
                                    const int32_t* idx, int q_begin, int q_count, float* target, int64_t ld,
                                    void* stream) {
  dsa_status st = api_check_shape(s);
  if (st != DSA_OK) return st;
  if (!q || !kv || !lse || !target || !aligned16(q) || !aligned16(kv)) return DSA_ERR_INVALID_ARG;
  if (q_begin < 0 || q_count < 0 || q_begin + q_count > s->T || ld < s->S) return DSA_ERR_INVALID_ARG;
  if (s->d_k != DK) return DSA_ERR_UNSUPPORTED;
  LaunchCtx c;
  if ((st = api_make_ctx(stream, &c)) != DSA_OK) return st;
  if (q_count == 0) return DSA_OK;
  TargetParams p = {};
  p.map = api_kv_map(s);
  p.q = q; p.kv = kv; p.lse = lse; p.idx = idx; p.target = target; p.ld = ld;
  p.T = s->T; p.H = s->H; p.k = s->k; p.q_begin = q_begin; p.q_count = q_count; p.B = s->B;
  const float tau = s->softmax_scale > 0.f ? s->softmax_scale : 1.0f / sqrtf((float)s->d_k);
  p.scale_log2 = tau * 1.4426950408889634f;
  p.wait_ns = c.wait_ns;
  p.err = c.err;
  CUtensorMap tm_kv = {};
  p.tma_keys = idx == nullptr && p.map.page_size == 0;
  if (p.tma_keys && !make_tmap_2d(&tm_kv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kv, (uint64_t)s->B * s->S, DK,
                                  (uint64_t)DK * 2, kChunk, 64, CU_TENSOR_MAP_SWIZZLE_128B))
    return DSA_ERR_CUDA;
  if (cudaFuncSetAttribute(kl_target_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem) != cudaSuccess)
    return DSA_ERR_CUDA;
  kl_target_kernel<<<(unsigned)((long long)s->B * q_count), kThreads, kSmem, c.stream>>>(tm_kv, p);
  note_launches(1);
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

extern "C" dsa_status dsa_indexer_kl(const dsa_shape* s, const float* scores, const float* target, int64_t ld,
                                     const int32_t* idx, int q_begin, int q_count, float* grad, float* loss,
                                     void* stream) {
  dsa_status st = api_check_shape(s);
  if (st != DSA_OK) return st;
  if (!scores || !target || !grad || !loss || ld < s->S) return DSA_ERR_INVALID_ARG;
  if (q_begin < 0 || q_count < 0 || q_begin + q_count > s->T) return DSA_ERR_INVALID_ARG;
  LaunchCtx c;
  if ((st = api_make_ctx(stream, &c)) != DSA_OK) return st;
  if (q_count == 0) return DSA_OK;
  const KvMap map = api_kv_map(s);
  indexer_kl_kernel<<<s->B * q_count, 256, 0, c.stream>>>(map, scores, target, ld, idx, s->T, s->k, q_begin, q_count,
                                                          grad, loss, c.err);
  note_launches(1);
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

extern "C" dsa_status dsa_indexer_backward(const dsa_shape* s, const uint8_t* q_I, const float* q_scale,
                                           const float* w, const uint8_t* k_I, const float* k_scale,
                                           const float* grad, int64_t ld, const int32_t* idx, int q_begin,
                                           int q_count, float* dq, float* dw, float* dk, void* stream) {
  dsa_status st = api_check_shape(s);
  if (st != DSA_OK) return st;
  if (!q_I || !q_scale || !w || !k_I || !k_scale || !grad || !dq || !dw || !dk || ld < s->S) return DSA_ERR_INVALID_ARG;
  if (q_begin < 0 || q_count < 0 || q_begin + q_count > s->T) return DSA_ERR_INVALID_ARG;
  LaunchCtx c;
  if ((st = api_make_ctx(stream, &c)) != DSA_OK) return st;
  if (q_count == 0) return DSA_OK;
  const KvMap map = api_kv_map(s);
  // tensor-core form where it applies (16-byte aligned rows, cache rows that
  // fit an int); the CUDA-core form otherwise
  if (indexer_bwd_tc_supported(s->H_I, s->D_I) && aligned16(q_I) && aligned16(k_I) && aligned16(dq) &&
      aligned16(dk) && map.pool_rows(s->B) < (1ll << 31)) {
    const cudaError_t e = launch_indexer_bwd_tc(c, map, q_I, q_scale, w, k_I, k_scale, grad, ld, idx, s->B, s->T,
                                                s->k, s->H_I, q_begin, q_count, dq, dw, dk);
    return e == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
  }
  cudaError_t e = cudaErrorInvalidValue;
#define DSA_BWD(HI_, DI_)                                                                                          \
  if (s->H_I == HI_ && s->D_I == DI_)                                                                              \
    e = launch_bwd_t<HI_, DI_>(c, map, q_I, q_scale, w, k_I, k_scale, grad, ld, idx, s->B, s->T, s->k, q_begin, \
                               q_count, dq, dw, dk);
  DSA_BWD(64, 128)
  DSA_BWD(32, 128)
  DSA_BWD(16, 128)
  DSA_BWD(64, 64)
  DSA_BWD(32, 64)
#undef DSA_BWD
  if (e == cudaErrorInvalidValue) return DSA_ERR_UNSUPPORTED;
  return e == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}
