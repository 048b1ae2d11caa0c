// Step C: sparse MQA/MLA attention over the selected keys, on tcgen05.
//
// out[t,h] = sum_{s in idx[t]} softmax_s(tau q[t,h] . kv[s]) kv[s, :d_v]
// (ouchyi thread, "Nasil calisiyor" paragraph: the expensive attention runs
// only over the kept subset; tenelement.pl, section "Architektura ...",
// "Integracja z MLA" bullet: MQA form, one KV row shared by all heads;
// degnora.com, "MLA - Multi-Latent Attention": keys and values come from the
// one cached latent, so V is the first d_v columns of the row).
//
// Work split.  All heads of one query form the MMA M dimension (128 rows;
// fewer heads leave zero-weight rows).  A 128 x 512 FP32 output accumulator
// would fill all of TMEM, so each query is handled by two independent CTAs,
// one per half of the value columns; each computes the full logit tile
// (Q K^T over the 576-wide key) and its 128 x 256 half of the output.
//
// Per CTA: Q (128 x 576 BF16, 144 KB) is loaded once by TMA into shared
// memory (128B swizzle); selected KV rows arrive in chunks of 32 through a
// 2-stage ring filled with 16-byte cp.async by two gather warps that take
// alternate chunks; both MMAs read their operands from shared memory
// (S = Q K^T into a double-buffered TMEM tile, O += P V with P written by the
// softmax warps in a 64B-swizzled tile and V read as the MN-major view of the
// same gathered rows).  Online softmax in base 2 with a lazy rescale: the
// running maximum moves only when a chunk exceeds it by more than 8 (so
// p <= 256), and then the TMEM accumulator is rescaled once.
//
// Warp roles (224 threads): warps 0-1 gather (warp w fills stage w), warp 2
// owns TMEM and issues the MMAs, warps 3-6 run the softmax (thread = head
// row) and write the output.  Decode splits the selected keys of each query
// over several CTAs and merges the partial results with a combine kernel.
// Every barrier that receives an asynchronous arrival is waited on before
// the CTA exits.
#include <cuda_bf16.h>

#include "internal.h"
#include "sm100.cuh"
#include "tma_host.h"

namespace dsa {
namespace {

using namespace sm100;

constexpr int kN = 32;          // selected keys per chunk
constexpr int kStages = 2;      // one per gather warp
constexpr int kThreads = 224;
constexpr int kMmaWarp = 2;
constexpr uint32_t kOCol = 0, kSCol = 256, kTmemCols = 512;  // S: two buffers of kN columns
constexpr float kRescaleThreshold = 8.f;                     // log2 units

template <int DK, int DV>
struct Cfg {
  static constexpr int KSTEPS = DK / 16;            // 16-wide MMA K steps over the key dim
  static constexpr int NATOM = (DK + 63) / 64;      // 64-column (128-byte) atoms of a row
  static constexpr bool SPLIT_V = DV >= 128;        // value columns split over two CTAs
  static constexpr int NHALF = SPLIT_V ? 2 : 1;
  static constexpr int DVH = DV / NHALF;
  static constexpr int Q_ATOM = 128 * 128;          // 128 head rows x 128 bytes
  static constexpr int KV_ATOM = kN * 128;          // kN key rows x 128 bytes
  static constexpr int STAGE = NATOM * KV_ATOM;
  static constexpr int P_BYTES = 128 * kN * 2;      // 128 rows x 64 bytes, 64B swizzle
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = OFF_Q + NATOM * Q_ATOM;
  static constexpr int OFF_P = OFF_KV + kStages * STAGE;
  static constexpr int OFF_META = OFF_P + P_BYTES;  // valid flag per slot, kStages x kN bytes
  static constexpr int OFF_BAR = OFF_META + kStages * kN;
  static constexpr int NBARS = 1 + 2 * kStages + 2 + 2 + 1 + 1 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBARS * 8;
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int ALLOC = BYTES + 1024;        // room to align the base to 1024
  static_assert(DVH <= 256 && DVH % 16 == 0, "value columns per CTA");
  static_assert(kSCol + 2 * kN <= kTmemCols && DVH <= kSCol, "TMEM layout");
  static_assert(ALLOC <= 232448, "shared memory per CTA");
};

struct AttnParams {
  const uint16_t* kv;
  const int32_t* idx;
  uint16_t* out;
  float* lse;
  float* part_o;    // [rows, nsplit, H, d_v] (split mode)
  float* part_lse;  // [rows, nsplit, H], log2 units
  int T, S, H, k;
  int rows;         // B * T query rows
  int nsplit, kc;   // splits per row and selected slots per split
  float scale_log2; // tau * log2(e)
  long long wait_ns;
  DevErr* err;
};

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

template <int DK, int DV>
__global__ void __launch_bounds__(kThreads, 1)
    sparse_attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, AttnParams p) {
  using C = Cfg<DK, DV>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sKV = smem + C::OFF_KV;
  uint8_t* sP = smem + C::OFF_P;
  uint8_t* sMeta = smem + C::OFF_META;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;                // [kStages]
  uint64_t* kv_empty = kv_full + kStages;      // [kStages]
  uint64_t* s_full = kv_empty + kStages;       // [2]
  uint64_t* s_free = s_full + 2;               // [2]
  uint64_t* p_full = s_free + 2;
  uint64_t* pv_done = p_full + 1;
  uint64_t* mma_done = pv_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int half = blockIdx.x % C::NHALF;
  const int rest = blockIdx.x / C::NHALF;
  const int row = rest / p.nsplit;  // b * T + t
  const int split = rest - row * p.nsplit;
  const int b = row / p.T;
  const int slot0 = split * p.kc;
  const int slot1 = min(p.k, slot0 + p.kc);
  // self-check: a CTA outside the launch's rows does no work
  const bool row_ok = row >= 0 && row < p.rows && split >= 0 && split < p.nsplit && slot0 >= 0;
  const int nchunks = row_ok && slot1 > slot0 ? (slot1 - slot0 + kN - 1) / kN : 0;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&kv_full[i], 32);  // the 32 lanes of the gather warp that owns the stage
      mbar_init(&kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 4);
    }
    mbar_init(p_full, 4);
    mbar_init(pv_done, 1);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const AbortSources ab{abort_flag, &p.err->code};
  const AbortSources no_abort{nullptr, nullptr};  // drains of this CTA's own async work
  auto fail = [&](unsigned where) {
    report_error(p.err, DSA_ERR_TIMEOUT, ERR_SITE_ATTN | (where << 8));
    *abort_flag = 1;
  };

  if (warp < 2) {
    // ------------------------------------------------------------ gather (warp w fills stage w)
    const int w = warp;
    bool q_issued = false;
    if (w == 0 && lane == 0 && nchunks > 0) {
      prefetch_tmap(&tm_q);
      mbar_arrive_expect_tx(q_full, C::NATOM * C::Q_ATOM);
      for (int a = 0; a < C::NATOM; ++a) tma_load_2d(sQ + a * C::Q_ATOM, &tm_q, q_full, a * 64, row * p.H);
      q_issued = true;
    }
    const int c16 = lane & 7, rg = lane >> 3;  // 16-byte column chunk, row group
    const int32_t* irow = p.idx + (size_t)row * p.k;
    const uint16_t* kvb = p.kv + (size_t)b * p.S * DK;
    uint8_t* stage = sKV + w * C::STAGE;
    // the indices of a chunk are loaded one chunk ahead, while the previous
    // chunk's rows are in flight
    int ivn[kN / 4];
    auto load_idx = [&](int j) {
#pragma unroll
      for (int m = 0; m < kN / 4; ++m) {
        const int slot = slot0 + j * kN + rg + 4 * m;
        ivn[m] = (j < nchunks && slot < slot1) ? irow[slot] : -1;
      }
    };
    load_idx(w);
    for (int j = w, use = 0; j < nchunks; j += kStages, ++use) {
      int iv[kN / 4];
#pragma unroll
      for (int m = 0; m < kN / 4; ++m) iv[m] = ivn[m];
      if (!mbar_wait(&kv_empty[w], (use & 1) ^ 1, p.wait_ns, ab)) { fail(1); break; }
#pragma unroll
      for (int m = 0; m < kN / 4; ++m) {
        const int r = rg + 4 * m;
        int v = iv[m];
        if (v >= p.S) {
          if (c16 == 0) report_error(p.err, DSA_ERR_DEVICE_BOUNDS, ERR_SITE_ATTN);
          v = -1;
        }
        const bool valid = v >= 0;
        if (c16 == 0) sMeta[w * kN + r] = valid ? 1 : 0;
        const uint16_t* src = kvb + (size_t)(valid ? v : 0) * DK;
#pragma unroll
        for (int a = 0; a < C::NATOM; ++a) {
          if (a * 128 + c16 * 16 < DK * 2)
            cp_async16(stage + a * C::KV_ATOM + r * 128 + ((c16 ^ (r & 7)) << 4), src + a * 64 + c16 * 8);
        }
      }
      cp_async_commit();
      load_idx(j + kStages);
      cp_async_wait<0>();
      fence_proxy_async_smem();
      mbar_arrive(&kv_full[w]);
    }
    cp_async_wait<0>();
    // drain: the Q load must have landed before this CTA's memory is reused
    if (q_issued) mbar_wait(q_full, 0, p.wait_ns, no_abort);
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      constexpr uint32_t idesc_qk = make_idesc(kFmtBF16, kFmtBF16, 0, 0, 128, kN);
      constexpr uint32_t idesc_pv = make_idesc(kFmtBF16, kFmtBF16, 0, 1, 128, C::DVH);
      const uint32_t q_base = smem_u32(sQ), kv_base = smem_u32(sKV), p_base = smem_u32(sP);
      const uint32_t v_atom = (uint32_t)(half * C::DVH / 64);
      int pv_issued = 0;
      auto issue_pv = [&](int i) {
        tc_fence_after();
        const int st = i & 1;
        const uint32_t vbase = kv_base + st * C::STAGE + v_atom * C::KV_ATOM;
        const uint64_t pdesc = make_sdesc(p_base, 16, 512, kSwizzle64);
#pragma unroll
        for (int ks = 0; ks < kN / 16; ++ks) {
          const uint64_t vdesc = make_sdesc(vbase + ks * 16 * 128, C::KV_ATOM, 1024, kSwizzle128);
          mma_bf16(tmem + kOCol, pdesc + 2 * ks, vdesc, idesc_pv, (i > 0 || ks > 0) ? 1u : 0u);
        }
        mma_commit(pv_done);
        mma_commit(&kv_empty[st]);
        pv_issued = i + 1;
      };
      bool ok = nchunks == 0 || mbar_wait(q_full, 0, p.wait_ns, ab);
      if (!ok) fail(3);
      // Issue whichever MMA is ready: Q K^T of chunk qk once its rows have
      // landed (and its S buffer is free), P V of chunk pv once its
      // probabilities are written.  P V never waits behind a later chunk's
      // gather, so a stage is handed back to its gather warp as early as the
      // data dependencies allow.
      int qk = 0, pv = 0;
      uint64_t t_idle = 0;
      uint32_t spins = 0;
      while (ok && pv < nchunks) {
        bool progressed = false;
        if (qk < nchunks && qk <= pv + 1) {
          const int st = qk & 1;
          if (mbar_test_wait(&kv_full[st], (qk >> 1) & 1) &&
              (qk < 2 || mbar_test_wait(&s_free[st], ((qk >> 1) - 1) & 1))) {
            fence_proxy_async_smem();
            tc_fence_after();
            const uint32_t sbase = kv_base + st * C::STAGE;
#pragma unroll 4
            for (int ks = 0; ks < C::KSTEPS; ++ks) {
              const int d = ks * 16;
              const uint32_t off = (uint32_t)((d % 64) * 2);
              const uint64_t adesc = make_sdesc(q_base + (d / 64) * C::Q_ATOM + off, 16, 1024, kSwizzle128);
              const uint64_t bdesc = make_sdesc(sbase + (d / 64) * C::KV_ATOM + off, 16, 1024, kSwizzle128);
              mma_bf16(tmem + kSCol + st * kN, adesc, bdesc, idesc_qk, ks > 0 ? 1u : 0u);
            }
            mma_commit(&s_full[st]);
            ++qk;
            progressed = true;
          }
        }
        if (pv < qk && mbar_test_wait(p_full, pv & 1)) {
          issue_pv(pv);
          ++pv;
          progressed = true;
        }
        if (progressed) {
          spins = 0;
          continue;
        }
        // nothing ready: doze briefly on the event most likely next, with
        // bounded idle time, and abort when another role failed
        if (pv < qk)
          mbar_try_wait_hint(p_full, pv & 1, 200);
        else
          mbar_try_wait_hint(&kv_full[qk & 1], (qk >> 1) & 1, 200);
        if (++spins == 1) t_idle = global_ns();
        if ((spins & 1023u) == 0u) {
          if (*abort_flag != 0) { ok = false; break; }
          const long long dt = (long long)(global_ns() - t_idle);
          if (dt > p.wait_ns || (dt > 1000000 && (spins & 65535u) == 0u && p.err->code != 0u)) {
            fail(4);
            ok = false;
          }
        }
      }
      mma_commit(mma_done);
      mbar_wait(mma_done, 0, p.wait_ns, no_abort);
      // drain: the last releases of each stage are never waited by the gather
      // warps; make sure they have landed before this CTA's memory is reused
      for (int i = max(0, pv_issued - kStages); i < pv_issued; ++i)
        mbar_wait(&kv_empty[i & 1], (i >> 1) & 1, p.wait_ns, no_abort);
    }
  } else {
    // ------------------------------------------------------------ softmax + output
    const int quarter = warp & 3;
    const int h = quarter * 32 + lane;              // head row == TMEM lane
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
    // every lane polls; the warp proceeds only if all lanes saw the phase
    auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
      const bool r = mbar_wait(bar, parity, p.wait_ns, ab);
      return __all_sync(0xffffffffu, r);
    };
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nchunks && ok; ++j) {
      const int sb = j & 1, st = j & 1;
      // 1. logits of this chunk
      if (!wwait(&s_full[sb], (j >> 1) & 1)) { fail(6); ok = false; break; }
      tc_fence_after();
      uint32_t sr[32];
      tmem_ld32(tmem + lane_addr + kSCol + sb * kN, sr);
      tmem_wait_ld_dep(sr);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[sb]);
      // 2. mask the empty slots, update the running maximum
      if (!wwait(&kv_full[st], (j >> 1) & 1)) { fail(7); ok = false; break; }
      const uint4* meta = reinterpret_cast<const uint4*>(sMeta + st * kN);
      float s[kN];
      float mc = -INFINITY;
#pragma unroll
      for (int c = 0; c < kN / 16; ++c) {
        const uint4 mv = meta[c];
        const uint32_t words[4] = {mv.x, mv.y, mv.z, mv.w};
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const bool valid = (words[q >> 2] >> ((q & 3) * 8)) & 0xffu;
          const float x = valid ? __uint_as_float(sr[c * 16 + q]) * p.scale_log2 : -INFINITY;
          s[c * 16 + q] = x;
          mc = fmaxf(mc, x);
        }
      }
      float alpha = 1.f;
      bool rescale = false;
      if (m_used == -INFINITY) {
        m_used = mc;
      } else if (mc > m_used + kRescaleThreshold) {
        alpha = exp2f(m_used - mc);
        m_used = mc;
        rescale = true;
      }
      // 3. the previous P.V is done: P buffer free, accumulator stable
      if (j >= 1 && !wwait(pv_done, (j - 1) & 1)) { fail(8); ok = false; break; }
      // 4. rescale the output accumulator when the maximum moved (warp-wide)
      if (__any_sync(0xffffffffu, rescale)) {
        tc_fence_after();
        for (int c = 0; c < C::DVH / 32; ++c) {
          uint32_t o[32];
          __syncwarp();
          tmem_ld32(tmem + lane_addr + kOCol + c * 32, o);
          tmem_wait_ld_dep(o);
#pragma unroll
          for (int q = 0; q < 32; ++q) o[q] = __float_as_uint(__uint_as_float(o[q]) * alpha);
          tmem_st32(tmem + lane_addr + kOCol + c * 32, o);
        }
        tmem_wait_st();
      }
      // 5. probabilities (bf16) into P with the 64-byte swizzle: 16-byte
      //    chunk c of row h lands at h*64 + ((c ^ ((h >> 1) & 3)) * 16)
      float rs = 0.f;
      uint8_t* prow = sP + h * 64;
      const bool any = m_used != -INFINITY;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float e[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          e[q] = any ? exp2f(s[c * 8 + q] - m_used) : 0.f;
          rs += e[q];
        }
        uint4 pk;
        pk.x = pack_bf16x2(e[0], e[1]);
        pk.y = pack_bf16x2(e[2], e[3]);
        pk.z = pack_bf16x2(e[4], e[5]);
        pk.w = pack_bf16x2(e[6], e[7]);
        *reinterpret_cast<uint4*>(prow + ((c ^ ((h >> 1) & 3)) << 4)) = pk;
      }
      l = l * alpha + rs;
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    // 6. output
    if (ok && nchunks > 0 && !wwait(pv_done, (nchunks - 1) & 1)) {
      fail(9);
      ok = false;
    }
    if (ok && nchunks > 0) {
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const float lse2 = l > 0.f ? m_used + log2f(l) : -INFINITY;
      const bool write_o = h < p.H;
      const int vlo = half * C::DVH;
      for (int c = 0; c < C::DVH / 32; ++c) {
        uint32_t o[32];
        __syncwarp();
        tmem_ld32(tmem + lane_addr + kOCol + c * 32, o);
        tmem_wait_ld_dep(o);
        if (!write_o) continue;
        if (p.nsplit == 1) {
          uint4* dst = reinterpret_cast<uint4*>(p.out + ((size_t)row * p.H + h) * DV + vlo + c * 32);
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(o[8 * g + 0]) * inv, __uint_as_float(o[8 * g + 1]) * inv);
            v.y = pack_bf16x2(__uint_as_float(o[8 * g + 2]) * inv, __uint_as_float(o[8 * g + 3]) * inv);
            v.z = pack_bf16x2(__uint_as_float(o[8 * g + 4]) * inv, __uint_as_float(o[8 * g + 5]) * inv);
            v.w = pack_bf16x2(__uint_as_float(o[8 * g + 6]) * inv, __uint_as_float(o[8 * g + 7]) * inv);
            dst[g] = v;
          }
        } else {
          float4* dst = reinterpret_cast<float4*>(p.part_o + (((size_t)row * p.nsplit + split) * p.H + h) * DV +
                                                  vlo + c * 32);
#pragma unroll
          for (int g = 0; g < 8; ++g)
            dst[g] = make_float4(__uint_as_float(o[4 * g]) * inv, __uint_as_float(o[4 * g + 1]) * inv,
                                 __uint_as_float(o[4 * g + 2]) * inv, __uint_as_float(o[4 * g + 3]) * inv);
        }
      }
      if (half == 0 && h < p.H) {
        if (p.nsplit == 1) {
          if (p.lse != nullptr) p.lse[(size_t)row * p.H + h] = lse2 * 0.6931471805599453f;
        } else {
          p.part_lse[((size_t)row * p.nsplit + split) * p.H + h] = lse2;
        }
      }
    } else if (ok && h < p.H && row_ok && half == 0) {
      // no selected slots in this split: empty result
      if (p.nsplit > 1) p.part_lse[((size_t)row * p.nsplit + split) * p.H + h] = -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Merge the per-split results of one (row, head): weights 2^(lse_s - max).
template <int DV>
__global__ void __launch_bounds__(128) attn_combine_kernel(const float* part_o, const float* part_lse, uint16_t* out,
                                                            float* lse, int H, int nsplit) {
  const int row = blockIdx.x / H;
  const int h = blockIdx.x - row * H;
  float mx = -INFINITY;
  for (int s = 0; s < nsplit; ++s) mx = fmaxf(mx, part_lse[((size_t)row * nsplit + s) * H + h]);
  constexpr int PER = (DV + 127) / 128;
  float acc[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) acc[i] = 0.f;
  float wsum = 0.f;
  if (mx != -INFINITY) {
    for (int s = 0; s < nsplit; ++s) {
      const float ls = part_lse[((size_t)row * nsplit + s) * H + h];
      if (ls == -INFINITY) continue;
      const float w = exp2f(ls - mx);
      wsum += w;
      const float* src = part_o + (((size_t)row * nsplit + s) * H + h) * DV;
#pragma unroll
      for (int i = 0; i < PER; ++i)
        if (threadIdx.x + 128 * i < DV) acc[i] = fmaf(w, src[threadIdx.x + 128 * i], acc[i]);
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  uint16_t* dst = out + ((size_t)row * H + h) * DV;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    if (threadIdx.x + 128 * i >= DV) continue;
    __nv_bfloat16 v = __float2bfloat16_rn(acc[i] * inv);
    dst[threadIdx.x + 128 * i] = *reinterpret_cast<uint16_t*>(&v);
  }
  if (threadIdx.x == 0 && lse != nullptr)
    lse[(size_t)row * H + h] = wsum > 0.f ? (mx + log2f(wsum)) * 0.6931471805599453f : -INFINITY;
}

template <int DK, int DV>
cudaError_t launch_tc(const LaunchCtx& c, const AttnArgs& a) {
  using Cf = Cfg<DK, DV>;
  AttnParams p;
  p.kv = a.kv;
  p.idx = a.idx;
  p.out = a.out;
  p.lse = a.lse;
  p.T = a.T;
  p.S = a.S;
  p.H = a.H;
  p.k = a.k;
  p.rows = a.B * a.T;
  p.nsplit = a.nsplit;
  p.kc = ((a.k + a.nsplit - 1) / a.nsplit + kN - 1) / kN * kN;
  p.scale_log2 = a.tau * 1.4426950408889634f;
  p.wait_ns = c.wait_ns;
  p.err = c.err;
  const long long rows = (long long)a.B * a.T;
  p.part_o = a.part;
  p.part_lse = a.part ? a.part + (size_t)rows * a.nsplit * a.H * DV : nullptr;
  // Q as a [rows * H, DK] BF16 matrix read in 128-row x 64-column boxes
  CUtensorMap tm_q;
  if (!make_tmap_2d(&tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.q, (uint64_t)rows * a.H, DK, (uint64_t)DK * 2, 128,
                    64, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(sparse_attn_tc_kernel<DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       Cf::ALLOC);
  if (e != cudaSuccess) return e;
  const long long ctas = rows * a.nsplit * Cf::NHALF;
  sparse_attn_tc_kernel<DK, DV><<<(unsigned)ctas, kThreads, Cf::ALLOC, c.stream>>>(tm_q, p);
  note_launches(1);
  e = cudaGetLastError();
  if (e != cudaSuccess || a.nsplit == 1) return e;
  attn_combine_kernel<DV><<<(unsigned)(rows * a.H), 128, 0, c.stream>>>(p.part_o, p.part_lse, a.out, a.lse, a.H,
                                                                         a.nsplit);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace

size_t attn_partial_floats(int rows, int H, int d_v, int nsplit) {
  return nsplit > 1 ? (size_t)rows * nsplit * H * (d_v + 1) : 0;
}

int attn_choose_nsplit(int rows, int H, int k, int num_sms) {
  (void)H;
  const int chunks = (k + kN - 1) / kN;
  int target = rows > 0 ? (num_sms + rows - 1) / rows : 1;
  if (target < 1) target = 1;
  if (target > chunks) target = chunks;
  const int kc = ((k + target - 1) / target + kN - 1) / kN * kN;
  return (k + kc - 1) / kc;
}

cudaError_t launch_sparse_attn(const LaunchCtx& c, const AttnArgs& a) {
  if ((long long)a.B * a.T <= 0) return cudaSuccess;
  if (a.nsplit > 1 && a.part == nullptr) return cudaErrorInvalidValue;
  if (a.d_k == 576 && a.d_v == 512) return launch_tc<576, 512>(c, a);
  if (a.d_k == 80 && a.d_v == 64) return launch_tc<80, 64>(c, a);
  return cudaErrorInvalidValue;
}

}  // namespace dsa
