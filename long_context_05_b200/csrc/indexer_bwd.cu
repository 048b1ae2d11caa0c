// Backward of the lightning indexer on tcgen05 tensor cores (training the
// indexer: tenelement.pl, "DeepSeek V3.2-Exp Cuts Long-Context Costs ...",
// section "Proces Treningu DSA: Od Warm-up do Sparsity"; the score is the
// indexer formula of the ouchyi thread on DeepSeek Sparse Attention, "Nasil
// calisiyor" paragraph).
//
// For query row t with score gradient g_s = dL/dI[t, s] over its keys s
// (the selected set, or every visible key), I[t, s] = sum_j w_j ReLU(D_js)
// with D_js = q_j . k_s on the dequantised operands q_j = qs_j q8_j,
// k_s = ks_s k8_s.  With the mask M_js = [D_js > 0]:
//
//   R_j  = sum_s g_s M_js k_s            (a vector of D_I per head)
//   dq_j = w_j R_j,   dw_j = q_j . R_j   (= sum_s g_s ReLU(D_js))
//   dk_s += g_s sum_j M_js w_j q_j       (every row adds into the shared keys)
//
// so one pass over a row's keys in tiles of 128 needs three contractions per
// tile and no reduction across keys on the CUDA cores:
//
//   D^T  [128 keys x 64 heads]  = K8 Q8^T                  (kind::f8f6f4, the
//        FP8 bytes as stored; the scales are positive, so [D > 0] = [K8 Q8^T > 0])
//   dk   [128 keys x 128 dims]  = P (Q'hi + Q'lo)          (kind::f16)
//        P = M^T as BF16 0/1, Q'_j = w_j qs_j q8_j split into BF16 hi + lo
//   R    [64 heads x 128 dims] += (G_hi + G_lo)^T K16      (kind::f16, M = 128:
//        the hi rows of G^T stacked over the lo rows, summed at the end)
//        G_sj = g_s ks_s M_js split into BF16 hi + lo, K16 = k8 as BF16 (exact)
//
// The hi + lo splits keep about 16 bits of every FP32 factor, so the
// gradients carry FP32-like error although the tensor cores read BF16.
//
// Warp roles (672 threads, one query row per CTA): warp 0 issues the MMAs;
// warps 1-4 gather the tile's key rows (k_I bytes, by cp.async) and g_s ks_s
// into a 3-stage ring; warps 5-12 read D^T from TMEM and build P, G^T and K16
// in shared memory (and finish dq, dw at the row's end); warps 13-20 add each
// tile's dk into global memory while the next tile is being built.
#include <cuda_fp8.h>
#include <math.h>

#include "internal.h"
#include "sm100.cuh"

namespace dsa {
namespace {

using namespace sm100;

namespace ib {
constexpr int kKeys = 128;      // keys per tile: TMEM lanes of D^T and dk
constexpr int kHeads = 64;      // indexer heads, zero-padded up to 64
constexpr int kDim = 128;       // D_I
constexpr int kStages = 3;      // key-row ring
constexpr int kFirstGather = 1, kGatherWarps = 4, kFirstEpi = 5, kEpiWarps = 8, kFirstRd = 13, kRdWarps = 8;
constexpr int kThreads = 32 * (kFirstRd + kRdWarps);
constexpr int kK8Bytes = kKeys * 128;                       // FP8 key rows, 128B-swizzled K-major
constexpr int OFF_K8 = 0;
constexpr int OFF_GT = OFF_K8 + kStages * kK8Bytes;         // G^T: 2 atoms (keys 0-63, 64-127) of 128 rows x 128 B
constexpr int OFF_K16 = OFF_GT + 2 * 128 * 128;             // K16: 2 atoms (dims 0-63, 64-127) of 128 keys x 128 B
constexpr int OFF_P = OFF_K16 + 2 * 128 * 128;              // P: 128 keys x 64 heads BF16, one atom
constexpr int OFF_Q8 = OFF_P + 128 * 128;                   // Q8: 64 heads x 128 B
constexpr int OFF_QH = OFF_Q8 + kHeads * 128;               // Q'hi: 2 atoms (dims) of 64 heads x 128 B
constexpr int OFF_QL = OFF_QH + 2 * kHeads * 128;           // Q'lo
constexpr int OFF_C = OFF_QL + 2 * kHeads * 128;            // per stage: g_s ks_s of each key
constexpr int OFF_HEAD = OFF_C + kStages * kKeys * 4;       // w[64], qs[64], dw halves [2][64]
constexpr int kStageStride = 144;                           // dk staging: 32 floats per key + 16 B pad
constexpr int OFF_STAGE = OFF_HEAD + 4 * kHeads * 4;        // per dk reader warp: 32 keys x kStageStride
constexpr int OFF_BAR = OFF_STAGE + kRdWarps * 32 * kStageStride;
// q_full, k8_full[3], k8_empty[3], d_full[2], d_empty[2], p_full, p_empty,
// dk_full[2], dk_empty[2], mma_done
constexpr int kNumBars = 1 + 2 * kStages + 2 + 2 + 1 + 1 + 2 + 2 + 1;
constexpr int OFF_MISC = OFF_BAR + kNumBars * 8;
constexpr int kSmem = OFF_MISC + 16;
static_assert(kSmem <= 232448, "shared memory per CTA");
static_assert(OFF_GT % 1024 == 0 && OFF_K16 % 1024 == 0 && OFF_P % 1024 == 0 && OFF_Q8 % 1024 == 0 &&
                  OFF_QH % 1024 == 0 && OFF_QL % 1024 == 0,
              "swizzled operands start on 1024-byte boundaries");
// the row-end exchange of R's lo rows (64 x 132 floats) reuses K16 and P
static_assert(64 * 132 * 4 <= OFF_Q8 - OFF_K16, "exchange buffer");
// TMEM columns: D^T x2 [0, 128), dk x2 [128, 384), R [384, 512)
constexpr uint32_t kTmemCols = 512, kColD = 0, kColDk = 128, kColR = 384;
}  // namespace ib

struct BwdParams {
  KvMap map;
  const uint8_t* q_I;
  const float* q_scale;
  const float* w;
  const uint8_t* k_I;
  const float* k_scale;
  const float* grad;
  long long ld;
  const int32_t* idx;     // null: every visible key
  float* dq;
  float* dw;
  float* dk;
  int T, k, H_I, q_begin, q_count;
  long long wait_ns;
  DevErr* err;
};

// two e4m3 bytes (low byte first) as two floats (exact)
__device__ __forceinline__ float2 e4m3x2_float2(uint32_t v) {
  const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(v & 0xFFFFu), __NV_E4M3);
  return __half22float2(*reinterpret_cast<const __half2*>(&hr));
}

// x as BF16 hi + lo (round to nearest even both times): hi + lo carries
// about 16 significant bits of x
__device__ __forceinline__ void split_bf16(float x, float y, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(x, y);
  const float2 hf = __bfloat1622float2(h);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = pack_bf16x2(x - hf.x, y - hf.y);
}

__device__ __forceinline__ void st_shared_v4(uint8_t* p, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(smem_u32(p)), "r"(a), "r"(b), "r"(c), "r"(d)
               : "memory");
}

__device__ __forceinline__ uint4 ld_shared_v4(const uint8_t* p) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(smem_u32(p))
               : "memory");
  return v;
}

// byte offset of 16-byte chunk c of row r in a 128B-swizzled atom
__device__ __forceinline__ int swz(int r, int c) { return r * 128 + ((c ^ (r & 7)) << 4); }

__global__ void __launch_bounds__(ib::kThreads, 1) indexer_bwd_tc_kernel(BwdParams p) {
  using namespace ib;
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) report_error(p.err, DSA_ERR_DEVICE_BOUNDS, ERR_SITE_INDEXER | (0xE0u << 8));
    return;
  }
  uint8_t* sK8 = smem + OFF_K8;
  uint8_t* sGT = smem + OFF_GT;
  uint8_t* sK16 = smem + OFF_K16;
  uint8_t* sP = smem + OFF_P;
  uint8_t* sQ8 = smem + OFF_Q8;
  uint8_t* sQH = smem + OFF_QH;
  uint8_t* sQL = smem + OFF_QL;
  float* sC = reinterpret_cast<float*>(smem + OFF_C);
  float* sW = reinterpret_cast<float*>(smem + OFF_HEAD);
  float* sQs = sW + kHeads;
  float* sDw = sQs + kHeads;                       // [2][64]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* k8_full = bars + 1;
  uint64_t* k8_empty = k8_full + kStages;
  uint64_t* d_full = k8_empty + kStages;
  uint64_t* d_empty = d_full + 2;
  uint64_t* p_full = d_empty + 2;
  uint64_t* p_empty = p_full + 1;
  uint64_t* dk_full = p_empty + 1;
  uint64_t* dk_empty = dk_full + 2;
  uint64_t* mma_done = dk_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int lr = blockIdx.x;                       // row of the launch: b * q_count + i
  const int b = lr / p.q_count, t = p.q_begin + (lr - (lr / p.q_count) * p.q_count);
  const size_t qrow = ((size_t)b * p.T + t) * p.H_I;   // first (token, head) of this query
  const int n = p.map.len(b, p.err, ERR_SITE_INDEXER) - p.T + t + 1;   // visible keys
  const int32_t* set = p.idx ? p.idx + ((size_t)b * p.T + t) * p.k : nullptr;
  const int m = set ? p.k : n;                     // key slots of the row
  const int nt = (m + kKeys - 1) / kKeys;          // tiles

  if (threadIdx.x == 0) {
    mbar_init(q_full, 32 * kEpiWarps);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&k8_full[i], 32 * kGatherWarps);
      mbar_init(&k8_empty[i], kEpiWarps);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&d_full[i], 1);
      mbar_init(&d_empty[i], kEpiWarps);
      mbar_init(&dk_full[i], 1);
      mbar_init(&dk_empty[i], kRdWarps);
    }
    mbar_init(p_full, kEpiWarps);
    mbar_init(p_empty, 1);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
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
    report_error(p.err, DSA_ERR_TIMEOUT, ERR_SITE_INDEXER | ((0xE0u + where) << 8));
    *abort_flag = 1;
  };
  auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
    const bool r = mbar_wait(bar, parity, p.wait_ns, ab);
    return __all_sync(0xffffffffu, r);
  };

  if (warp >= kFirstGather && warp < kFirstEpi) {
    // ------------------------------------------------------------ gather
    const int kk = threadIdx.x - 32 * kFirstGather;        // key of the tile, 0..127
    const float* G = p.grad + (size_t)lr * p.ld;
    bool ok = true;
    for (int i = 0; i < nt && ok; ++i) {
      const int st = i % kStages;
      if (i >= kStages && !wwait(&k8_empty[st], ((i / kStages) - 1) & 1)) {
        fail(1);
        ok = false;
        break;
      }
      const int slot = i * kKeys + kk;
      int s = -1;
      if (slot < m) s = set ? set[slot] : slot;
      long long row = -1;
      if (s >= 0 && s < n) row = p.map.row(b, s);
      const bool valid = row >= 0;
      const float g = valid ? G[s] : 0.f;
      const float ks = valid ? p.k_scale[row] : 0.f;
      sC[st * kKeys + kk] = g * ks;
      const uint8_t* src = p.k_I + (size_t)(valid ? row : 0) * kDim;
      uint8_t* dst = sK8 + st * kK8Bytes;
#pragma unroll
      for (int c = 0; c < 8; ++c) cp_async16_zfill(dst + swz(kk, c), src + c * 16, valid ? 16u : 0u);
      cp_async_commit();
      if (i >= 1) {
        cp_async_wait<1>();
        fence_proxy_async_smem();
        mbar_arrive(&k8_full[(i - 1) % kStages]);
      }
    }
    cp_async_wait<0>();
    if (ok && nt >= 1) {
      fence_proxy_async_smem();
      mbar_arrive(&k8_full[(nt - 1) % kStages]);
    }
  } else if (warp == 0) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      constexpr uint32_t idesc_d = make_idesc(kFmtE4M3, kFmtE4M3, 0, 0, 128, kHeads);
      constexpr uint32_t idesc_dk = make_idesc(kFmtBF16, kFmtBF16, 0, 1, 128, kDim);
      constexpr uint32_t idesc_r = make_idesc(kFmtBF16, kFmtBF16, 0, 1, 128, kDim);
      const uint64_t q8desc = make_sdesc(smem_u32(sQ8), 16, 1024, kSwizzle128);
      const uint64_t pdesc = make_sdesc(smem_u32(sP), 16, 1024, kSwizzle128);
      const uint64_t qhdesc = make_sdesc(smem_u32(sQH), kHeads * 128, 1024, kSwizzle128);
      const uint64_t qldesc = make_sdesc(smem_u32(sQL), kHeads * 128, 1024, kSwizzle128);
      const uint64_t gtdesc = make_sdesc(smem_u32(sGT), 16, 1024, kSwizzle128);
      const uint64_t k16desc = make_sdesc(smem_u32(sK16), 128 * 128, 1024, kSwizzle128);
      bool ok = mbar_wait(q_full, 0, p.wait_ns, ab);
      if (!ok) fail(2);
      for (int i = 0; i <= nt && ok; ++i) {
        if (i < nt) {
          // D^T of tile i
          const int st = i % kStages;
          if (!mbar_wait(&k8_full[st], (i / kStages) & 1, p.wait_ns, ab)) { fail(3); ok = false; break; }
          if (i >= 2 && !mbar_wait(&d_empty[i & 1], ((i - 2) >> 1) & 1, p.wait_ns, ab)) {
            fail(4);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t kdesc = make_sdesc(smem_u32(sK8 + st * kK8Bytes), 16, 1024, kSwizzle128);
#pragma unroll
          for (int ks = 0; ks < kDim / 32; ++ks)
            mma_f8(tmem + kColD + (i & 1) * kHeads, kdesc + (uint64_t)(ks * 2), q8desc + (uint64_t)(ks * 2), idesc_d,
                   ks > 0 ? 1u : 0u);
          mma_commit(&d_full[i & 1]);
        }
        if (i >= 1) {
          // R and dk of tile j = i - 1
          const int j = i - 1;
          if (!mbar_wait(p_full, j & 1, p.wait_ns, ab)) { fail(5); ok = false; break; }
          if (j >= 2 && !mbar_wait(&dk_empty[j & 1], ((j - 2) >> 1) & 1, p.wait_ns, ab)) {
            fail(6);
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int ks = 0; ks < kKeys / 16; ++ks) {
            const uint32_t aoff = (uint32_t)((ks * 16 / 64) * (128 * 128) + (ks * 16 % 64) * 2);
            mma_bf16(tmem + kColR, gtdesc + (uint64_t)(aoff >> 4), k16desc + (uint64_t)((ks * 16 * 128) >> 4),
                     idesc_r, (j > 0 || ks > 0) ? 1u : 0u);
          }
          const uint32_t dk_col = tmem + kColDk + (j & 1) * kDim;
#pragma unroll
          for (int ks = 0; ks < kHeads / 16; ++ks)
            mma_bf16(dk_col, pdesc + (uint64_t)(ks * 2), qhdesc + (uint64_t)((ks * 16 * 128) >> 4), idesc_dk,
                     ks > 0 ? 1u : 0u);
#pragma unroll
          for (int ks = 0; ks < kHeads / 16; ++ks)
            mma_bf16(dk_col, pdesc + (uint64_t)(ks * 2), qldesc + (uint64_t)((ks * 16 * 128) >> 4), idesc_dk, 1u);
          mma_commit(&dk_full[j & 1]);
          mma_commit(p_empty);
        }
      }
      mma_commit(mma_done);
      mbar_wait(mma_done, 0, p.wait_ns, no_abort);
    }
    __syncwarp();
  } else if (warp >= kFirstRd) {
    // ------------------------------------------------------------ dk reader
    // dk of each tile: TMEM -> registers, times g_s, through this warp's
    // staging rows so that each red.v4 of the warp covers four keys' 128
    // contiguous bytes (8 rounds for the warp's 32 keys), added into dk
    // (global).  The key's cache row and g_s are read again from global
    // memory (before the wait), so nothing is shared with the other roles.
    const int h = (warp - kFirstRd) >> 2;          // dims 64h .. 64h + 63
    const int q = warp & 3;
    const int sl = q * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
    uint8_t* stage = smem + OFF_STAGE + (warp - kFirstRd) * 32 * kStageStride;
    const float* G = p.grad + (size_t)lr * p.ld;
    for (int i = 0; i < nt; ++i) {
      const int slot = i * kKeys + sl;
      int s = -1;
      if (slot < m) s = set ? set[slot] : slot;
      int row = -1;
      float g = 0.f;
      if (s >= 0 && s < n) {
        const long long r = p.map.row(b, s);
        if (r >= 0) {
          row = (int)r;
          g = G[s];
        }
      }
      if (!wwait(&dk_full[i & 1], (i >> 1) & 1)) {
        fail(7);
        break;
      }
      tc_fence_after();
      uint32_t a[2][32];
      const uint32_t col = tmem + lane_addr + kColDk + (i & 1) * kDim + h * 64;
      tmem_ld32(col, a[0]);
      tmem_ld32(col + 32, a[1]);
      tmem_wait_ld_dep(a[0]);
      tmem_wait_ld_dep(a[1]);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&dk_empty[i & 1]);
      const float gs = row >= 0 ? g : 0.f;
#pragma unroll
      for (int ps = 0; ps < 2; ++ps) {
#pragma unroll
        for (int c = 0; c < 8; ++c)
          st_shared_v4(stage + lane * kStageStride + c * 16, __float_as_uint(gs * __uint_as_float(a[ps][4 * c])),
                       __float_as_uint(gs * __uint_as_float(a[ps][4 * c + 1])),
                       __float_as_uint(gs * __uint_as_float(a[ps][4 * c + 2])),
                       __float_as_uint(gs * __uint_as_float(a[ps][4 * c + 3])));
        __syncwarp();
#pragma unroll
        for (int it = 0; it < 8; ++it) {
          const int kl = it * 4 + (lane >> 3), c = lane & 7;   // key of the warp, float4 of its 32 floats
          const int rw = __shfl_sync(0xffffffffu, row, kl);
          const float gk = __shfl_sync(0xffffffffu, gs, kl);
          const uint4 v = ld_shared_v4(stage + kl * kStageStride + c * 16);
          if (rw >= 0 && gk != 0.f)
            atomicAdd(reinterpret_cast<float4*>(p.dk + (size_t)rw * kDim + h * 64 + ps * 32 + c * 4),
                      make_float4(__uint_as_float(v.x), __uint_as_float(v.y), __uint_as_float(v.z),
                                  __uint_as_float(v.w)));
        }
        __syncwarp();
      }
    }
  } else if (warp >= kFirstEpi) {
    // ------------------------------------------------------------ epilogue
    const int e = warp - kFirstEpi;
    const int h = e >> 2;                          // heads 32h.. of D^T / P / G^T; dims 64h.. of K16 / dk / R
    const int q = warp & 3;                        // TMEM lane quarter
    const int sl = q * 32 + lane;                  // key of the tile == TMEM lane
    const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
    bool ok = true;
    {
      // Q8 and Q'hi / Q'lo of this query (heads past H_I are zero)
      const int te = threadIdx.x - 32 * kFirstEpi;       // 0..255
      const int j = te >> 2, part = te & 3;              // head, 32 dims
      uint4 x0 = make_uint4(0u, 0u, 0u, 0u), x1 = x0;
      float wj = 0.f, qs = 0.f;
      if (j < p.H_I) {
        const uint4* src = reinterpret_cast<const uint4*>(p.q_I + (qrow + j) * kDim + part * 32);
        x0 = src[0];
        x1 = src[1];
        wj = p.w[qrow + j];
        qs = p.q_scale[qrow + j];
      }
      if (part == 0) {
        sW[j] = wj;
        sQs[j] = qs;
      }
      st_shared_v4(sQ8 + swz(j, 2 * part), x0.x, x0.y, x0.z, x0.w);
      st_shared_v4(sQ8 + swz(j, 2 * part + 1), x1.x, x1.y, x1.z, x1.w);
      const float f = wj * qs;
      const uint32_t wd[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
      const int atom = part >> 1, c0 = (part & 1) * 4;
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const uint32_t v = wd[2 * cc + u];
          const float2 a = e4m3x2_float2(v), bq = e4m3x2_float2(v >> 16);
          split_bf16(f * a.x, f * a.y, hi[2 * u], lo[2 * u]);
          split_bf16(f * bq.x, f * bq.y, hi[2 * u + 1], lo[2 * u + 1]);
        }
        st_shared_v4(sQH + atom * kHeads * 128 + swz(j, c0 + cc), hi[0], hi[1], hi[2], hi[3]);
        st_shared_v4(sQL + atom * kHeads * 128 + swz(j, c0 + cc), lo[0], lo[1], lo[2], lo[3]);
      }
      fence_proxy_async_smem();
      mbar_arrive(q_full);
    }
    for (int i = 0; i < nt && ok; ++i) {
      const int st = i % kStages;
      if (!wwait(&k8_full[st], (i / kStages) & 1)) { fail(8); ok = false; break; }
      if (!wwait(&d_full[i & 1], (i >> 1) & 1)) { fail(9); ok = false; break; }
      tc_fence_after();
      uint32_t r[32];
      tmem_ld32(tmem + lane_addr + kColD + (i & 1) * kHeads + h * 32, r);
      tmem_wait_ld_dep(r);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&d_empty[i & 1]);
      uint32_t mbits = 0;
#pragma unroll
      for (int jj = 0; jj < 32; ++jj) mbits |= (__uint_as_float(r[jj]) > 0.f ? 1u : 0u) << jj;
      // transpose the warp's 32 x 32 mask: lane l gets head 32h + l over the
      // warp's keys 32q .. 32q + 31
      uint32_t tb = 0;
#pragma unroll
      for (int jj = 0; jj < 32; ++jj) {
        const uint32_t bal = __ballot_sync(0xffffffffu, (mbits >> jj) & 1u);
        if (lane == jj) tb = bal;
      }
      if (i >= 1 && !wwait(p_empty, (i - 1) & 1)) { fail(10); ok = false; break; }
      // P row sl: heads 32h .. 32h + 31 as BF16 0 / 1
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint32_t bits = mbits >> (8 * cc + 2 * u);
          v[u] = ((bits & 1u) ? 0x3F80u : 0u) | ((bits & 2u) ? 0x3F800000u : 0u);
        }
        st_shared_v4(sP + swz(sl, 4 * h + cc), v[0], v[1], v[2], v[3]);
      }
      // G^T rows 32h + l (hi) and 64 + 32h + l (lo): keys 32q .. 32q + 31
      {
        const float* cst = sC + st * kKeys + q * 32;
        const int rhi = 32 * h + lane, rlo = 64 + 32 * h + lane;
        uint8_t* atom = sGT + (q >> 1) * (128 * 128);
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t hi[4], lo[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int k0 = 8 * cc + 2 * u;
            const float x = ((tb >> k0) & 1u) ? cst[k0] : 0.f;
            const float y = ((tb >> (k0 + 1)) & 1u) ? cst[k0 + 1] : 0.f;
            split_bf16(x, y, hi[u], lo[u]);
          }
          st_shared_v4(atom + swz(rhi, (q & 1) * 4 + cc), hi[0], hi[1], hi[2], hi[3]);
          st_shared_v4(atom + swz(rlo, (q & 1) * 4 + cc), lo[0], lo[1], lo[2], lo[3]);
        }
      }
      // K16 row sl, dims 64h .. 64h + 63, from the key's FP8 bytes
      {
        const uint8_t* k8 = sK8 + st * kK8Bytes;
        uint8_t* atom = sK16 + h * (128 * 128);
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          const uint4 x = ld_shared_v4(k8 + swz(sl, 4 * h + cc));
          const uint32_t wd[4] = {x.x, x.y, x.z, x.w};
          uint32_t o[8];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float2 a = e4m3x2_float2(wd[u]), bq = e4m3x2_float2(wd[u] >> 16);
            o[2 * u] = pack_bf16x2(a.x, a.y);
            o[2 * u + 1] = pack_bf16x2(bq.x, bq.y);
          }
          st_shared_v4(atom + swz(sl, 2 * cc), o[0], o[1], o[2], o[3]);
          st_shared_v4(atom + swz(sl, 2 * cc + 1), o[4], o[5], o[6], o[7]);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(p_full);
        mbar_arrive(&k8_empty[st]);
      }
    }
    // R: lo rows (lanes 64..127) through shared memory onto the hi rows
    if (ok && nt >= 1 && !wwait(p_empty, (nt - 1) & 1)) { fail(11); ok = false; }
    float* X = reinterpret_cast<float*>(sK16);           // [64][132]
    if (ok && nt >= 1 && q >= 2) {
      tc_fence_after();
      uint32_t a[32], c[32];
      const uint32_t col = tmem + lane_addr + kColR + h * 64;
      tmem_ld32(col, a);
      tmem_ld32(col + 32, c);
      tmem_wait_ld_dep(a);
      tmem_wait_ld_dep(c);
      float4* dst = reinterpret_cast<float4*>(X + (32 * (q - 2) + lane) * 132 + h * 64);
#pragma unroll
      for (int v = 0; v < 8; ++v)
        dst[v] = make_float4(__uint_as_float(a[4 * v]), __uint_as_float(a[4 * v + 1]), __uint_as_float(a[4 * v + 2]),
                             __uint_as_float(a[4 * v + 3]));
#pragma unroll
      for (int v = 0; v < 8; ++v)
        dst[8 + v] = make_float4(__uint_as_float(c[4 * v]), __uint_as_float(c[4 * v + 1]),
                                 __uint_as_float(c[4 * v + 2]), __uint_as_float(c[4 * v + 3]));
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kEpiWarps * 32) : "memory");
    if (q < 2) {
      // head j: R_j = hi + lo, dq_j = w_j R_j, and this half's part of dw_j
      // (tcgen05.ld runs on the whole warp; heads past H_I write nothing)
      const int j = 32 * q + lane;
      const bool have = ok && nt >= 1;
      const float wj = sW[j];
      float dwp = 0.f;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t a[32];
        if (have) {
          tc_fence_after();
          tmem_ld32(tmem + lane_addr + kColR + h * 64 + hh * 32, a);
          tmem_wait_ld_dep(a);
        }
        const float* xr = X + j * 132 + h * 64 + hh * 32;
        float Rv[32];
#pragma unroll
        for (int d = 0; d < 32; ++d) Rv[d] = have ? __uint_as_float(a[d]) + xr[d] : 0.f;
        if (j < p.H_I) {
          float4* dq = reinterpret_cast<float4*>(p.dq + (qrow + j) * kDim + h * 64 + hh * 32);
#pragma unroll
          for (int v = 0; v < 8; ++v)
            dq[v] = make_float4(wj * Rv[4 * v], wj * Rv[4 * v + 1], wj * Rv[4 * v + 2], wj * Rv[4 * v + 3]);
        }
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const uint4 x = ld_shared_v4(sQ8 + swz(j, 4 * h + 2 * hh + cc));
          const uint32_t wd[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float2 a2 = e4m3x2_float2(wd[u]), b2 = e4m3x2_float2(wd[u] >> 16);
            const int d = 16 * cc + 4 * u;
            dwp = fmaf(a2.x, Rv[d], dwp);
            dwp = fmaf(a2.y, Rv[d + 1], dwp);
            dwp = fmaf(b2.x, Rv[d + 2], dwp);
            dwp = fmaf(b2.y, Rv[d + 3], dwp);
          }
        }
      }
      sDw[h * kHeads + j] = dwp * sQs[j];
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kEpiWarps * 32) : "memory");
    if (q < 2 && h == 0) {
      const int j = 32 * q + lane;
      if (j < p.H_I) p.dw[qrow + j] = sDw[j] + sDw[kHeads + j];
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, ib::kTmemCols);
  }
}

}  // namespace

bool indexer_bwd_tc_supported(int H_I, int D_I) { return D_I == ib::kDim && H_I >= 1 && H_I <= ib::kHeads; }

cudaError_t launch_indexer_bwd_tc(const LaunchCtx& c, const KvMap& map, const uint8_t* q_I, const float* q_scale,
                                  const float* w, const uint8_t* k_I, const float* k_scale, const float* grad,
                                  long long ld, const int32_t* idx, int B, int T, int k, int H_I, int q_begin,
                                  int q_count, float* dq, float* dw, float* dk) {
  BwdParams p = {};
  p.map = map;
  p.q_I = q_I; p.q_scale = q_scale; p.w = w; p.k_I = k_I; p.k_scale = k_scale; p.grad = grad; p.ld = ld;
  p.idx = idx; p.dq = dq; p.dw = dw; p.dk = dk;
  p.T = T; p.k = k; p.H_I = H_I; p.q_begin = q_begin; p.q_count = q_count;
  p.wait_ns = c.wait_ns;
  p.err = c.err;
  cudaError_t e = cudaFuncSetAttribute(indexer_bwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, ib::kSmem);
  if (e != cudaSuccess) return e;
  indexer_bwd_tc_kernel<<<(unsigned)((long long)B * q_count), ib::kThreads, ib::kSmem, c.stream>>>(p);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace dsa
