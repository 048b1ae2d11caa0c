// Step C in decode: split-k sparse MQA/MLA attention, the memory-bound form.
//
// out[t,h] = sum_{s in idx[t]} softmax_s(tau q[t,h] . kv[s]) kv[s, :512]
// (ouchyi thread on DeepSeek Sparse Attention, "Nasil calisiyor" paragraph:
// at 128K a decode step attends over the 2,048 kept keys only; tenelement.pl,
// "DeepSeek V3.2-Exp Cuts Long-Context Costs ...", section "Architektura
// ...", "Integracja z MLA" bullet: in decoding the MLA latent is shared by
// all heads, MQA form).
//
// A decode row is one query of 128 heads over k selected rows of 1152 bytes:
// per selected key it moves 1152 B and computes 2 x 128 x (576 + 512) FLOP,
// about 240 FLOP per byte, so the step sits at the ridge of B200 and must
// stream the gathered rows at HBM rate while keeping the tensor cores busy.
// Work split: one CTA per (row, split of 128 selected slots), all 512 value
// columns in the one CTA, so every gathered byte is read once and Q K^T is
// computed once (the prefill kernel's two value-half CTAs would double both).
//
// Per CTA:
//   * shared memory: the 5 Q atoms of key dims 256..575 (80 KB, one TMA
//     load each) and the 128 gathered rows as 9 atoms of 128 keys x 128 B
//     (144 KB, 128B-swizzled K-major); no ring: every row of the split is in
//     flight at once;
//   * TMEM (512 columns): [0, 256) O quarters 0 and 1 | [256, 384) S, two
//     64-key chunks, then P as BF16 pairs over [256, 320) | [384, 512) Q key
//     dims 0..255 as BF16 pairs.  After Q K^T and the softmax, [320, 448) is
//     free and takes O quarter 2; quarter 3 reuses [0, 128) once quarter 0
//     has been read out;
//   * warp 0 issues the MMAs; warps 1-6 gather (three per 64-key half, each
//     copying three of the nine atoms of every row with 16-byte cp.async);
//     warps 7-14 run the softmax (two per TMEM lane quarter, one per half,
//     exchanging partial maxima and sums through shared memory) and drain O.
// Q K^T runs once both 64-key halves have landed, as one N = 128 pass over
// the split's keys; P V runs in four 128-column quarters (N = 128, K = the
// 128 keys) so the read-out of one quarter overlaps the MMAs of the next.  Each split writes its output
// normalised by its own row sum, as FP16 (|O| is bounded by the largest |V|,
// far inside FP16's range, and FP16 keeps 11 significant bits), with its
// log2-sum-exp in FP32; a combine kernel, launched as a programmatic
// dependent of this one, merges the splits:
//   O = sum_i 2^(lse_i - M) O_i / sum_i 2^(lse_i - M),  M = max_i lse_i.
#include "internal.h"
#include "sm100.cuh"
#include "tma_host.h"

namespace dsa {
namespace {

using namespace sm100;

constexpr int DK = 576, DV = 512;
constexpr int kKeys = 128;                     // selected slots per CTA
constexpr int kChunk = 64;                     // keys per Q K^T chunk (N)
constexpr int kNAtom = DK / 64;                // 128-byte atoms per key row
constexpr int kAtomBytes = kKeys * 128;        // one atom of the split's rows
constexpr int kQT = 256;                       // key dims of Q in TMEM
constexpr int kQSAtoms = (DK - kQT) / 64;      // Q atoms in shared memory
constexpr int kQAtomBytes = 128 * 128;         // 128 head rows x 128 bytes
constexpr int kKSteps = DK / 16;
constexpr int kQTSteps = kQT / 16;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSCol = 256, kQCol = 384;
__device__ __forceinline__ uint32_t ocol(int q) { return q == 2 ? 320u : (q == 3 ? 0u : (uint32_t)q * 128u); }

constexpr int kMmaWarp = 0, kFirstGather = 1, kGatherWarps = 6, kFirstSoftmax = 7, kSoftmaxWarps = 8;
constexpr int kThreads = 32 * (kFirstSoftmax + kSoftmaxWarps);

constexpr int OFF_Q = 0;
constexpr int OFF_KV = OFF_Q + kQSAtoms * kQAtomBytes;
constexpr int OFF_MASK = OFF_KV + kNAtom * kAtomBytes;      // 2 x uint64 valid-key masks
constexpr int OFF_XM = OFF_MASK + 16;                        // [2 sides][128] partial maxima
constexpr int OFF_XL = OFF_XM + 2 * 128 * 4;                 // [2 sides][128] partial sums
constexpr int OFF_BAR = OFF_XL + 2 * 128 * 4;
// q_full, q_ready, kv_full[2], s_full[2], p_full, pv_done[4], o_free, mma_done, mx[4], lx[4]
constexpr int kNumBars = 2 + 2 + 2 + 1 + 4 + 1 + 1 + 4 + 4;
constexpr int OFF_MISC = OFF_BAR + kNumBars * 8;
constexpr int kSmem = OFF_MISC + 16;
static_assert(kSmem <= 232448, "shared memory per CTA");
static_assert(OFF_KV % 1024 == 0 && OFF_BAR % 8 == 0, "alignment");

struct DecParams {
  KvMap map;
  const uint16_t* q;
  const uint16_t* kv;
  const int32_t* idx;
  int dense_rows;       // rows with t < dense_rows take keys 0..pos(t), idx unread
  uint16_t* out;
  float* lse;
  __half* part_o;       // [rows, nsplit, H, DV] (nsplit > 1)
  float* part_lse;      // [rows, nsplit, H], log2 units
  int T, H, k;
  int rows, nsplit;
  float scale_log2;     // tau * log2(e)
  long long wait_ns;
  DevErr* err;
};

template <bool PAGED>
__global__ void __launch_bounds__(kThreads, 1)
    sparse_attn_decode_kernel(const __grid_constant__ CUtensorMap tm_q, DecParams p) {
  extern __shared__ uint8_t smem[];
  if (smem_u32(smem) & 1023u) {
    // self-check: the swizzled layouts need a 1024-byte aligned base
    if (threadIdx.x == 0) report_error(p.err, DSA_ERR_DEVICE_BOUNDS, ERR_SITE_ATTN | (0xCu << 8));
    return;
  }
  // the combine kernel may be scheduled now; it waits for this grid's results
  pdl_launch_dependents();
  uint8_t* sQ = smem + OFF_Q;
  uint8_t* sKV = smem + OFF_KV;
  uint64_t* sMask = reinterpret_cast<uint64_t*>(smem + OFF_MASK);
  float* sXM = reinterpret_cast<float*>(smem + OFF_XM);
  float* sXL = reinterpret_cast<float*>(smem + OFF_XL);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* q_full = bars;           // Q atoms in shared memory (TMA)
  uint64_t* q_ready = bars + 1;      // Q rows in TMEM (8 softmax warps)
  uint64_t* kv_full = bars + 2;      // [2] a 64-key half gathered (3 warps x 32 lanes)
  uint64_t* s_full = bars + 4;       // [2] Q K^T of a half complete (commit)
  uint64_t* p_full = bars + 6;       // P written (8 softmax warps)
  uint64_t* pv_done = bars + 7;      // [4] P V of an O quarter complete (commit)
  uint64_t* o_free = bars + 11;      // O quarter 0 read out (8 softmax warps)
  uint64_t* mma_done = bars + 12;
  uint64_t* mx_bar = bars + 13;      // [4 quarters] both partial maxima written
  uint64_t* lx_bar = bars + 17;      // [4 quarters] both partial sums written
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x / p.nsplit;        // b * T + t
  const int split = blockIdx.x - row * p.nsplit;
  const bool row_ok = row >= 0 && row < p.rows;
  const int b = row / p.T, t = row - (row / p.T) * p.T;
  const int Lb = row_ok ? p.map.len(b, p.err, ERR_SITE_ATTN) : 0;
  const int pos = Lb - p.T + t;
  const bool dense = p.idx == nullptr || t < p.dense_rows;
  const int slot0 = split * kKeys;
  const int slot1 = min(dense ? pos + 1 : p.k, slot0 + kKeys);

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_ready, kSoftmaxWarps);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&kv_full[i], 32 * (kGatherWarps / 2));
      mbar_init(&s_full[i], 1);
    }
    mbar_init(p_full, kSoftmaxWarps);
    for (int i = 0; i < 4; ++i) mbar_init(&pv_done[i], 1);
    mbar_init(o_free, kSoftmaxWarps);
    mbar_init(mma_done, 1);
    for (int i = 0; i < 8; ++i) mbar_init(&mx_bar[i], 2);
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
  const AbortSources no_abort{nullptr, nullptr};
  auto fail = [&](unsigned where) {
    report_error(p.err, DSA_ERR_TIMEOUT, ERR_SITE_ATTN | ((0x40u + where) << 8));
    *abort_flag = 1;
  };
  auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
    const bool r = mbar_wait(bar, parity, p.wait_ns, ab);
    return __all_sync(0xffffffffu, r);
  };

  if (warp >= kFirstGather && warp < kFirstSoftmax) {
    // ------------------------------------------------------------ gather
    const int g = warp - kFirstGather;
    const int half = g / 3, sub = g - 3 * (g / 3);   // keys [64 half, +64); atoms sub, sub+3, sub+6
    bool q_issued = false;
    if (g == 0 && lane == 0 && row_ok) {
      prefetch_tmap(&tm_q);
      mbar_arrive_expect_tx(q_full, kQSAtoms * kQAtomBytes);
      for (int a = 0; a < kQSAtoms; ++a)
        tma_load_2d(sQ + a * kQAtomBytes, &tm_q, q_full, kQT + a * 64, row * p.H);
      q_issued = true;
    }
    // the selection is the kernel before this one's output (this kernel is
    // its programmatic dependent: barrier set-up, TMEM allocation and the Q
    // loads above overlap its tail)
    pdl_wait();
    // the 64 indices of this half: lane l holds slots l and l + 32
    int iv2[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int slot = slot0 + half * kChunk + lane + 32 * u;
      iv2[u] = (row_ok && slot < slot1) ? (dense ? slot : p.idx[(size_t)row * p.k + slot]) : -1;
    }
    const int c16 = lane & 7, rg = lane >> 3;     // 16-byte column chunk, row group
    uint64_t mask = 0;
#pragma unroll
    for (int u = 0; u < 2; ++u)
#pragma unroll 2
    for (int mm = 0; mm < 8; ++mm) {
      const int m = 8 * u + mm;
      const int r = rg + 4 * m;                    // row within the half (32 u + rg + 4 mm)
      int v = __shfl_sync(0xffffffffu, iv2[u], rg + 4 * mm);
      if (v >= Lb) {
        if (c16 == 0 && sub == 0) report_error(p.err, DSA_ERR_DEVICE_BOUNDS, ERR_SITE_ATTN);
        v = -1;
      }
      const long long cr = v >= 0 ? p.map.row<PAGED>(b, v) : -1;
      if (v >= 0 && cr < 0) {
        if (c16 == 0 && sub == 0) report_error(p.err, DSA_ERR_DEVICE_BOUNDS, ERR_SITE_ATTN | (1u << 8));
        v = -1;
      }
      const bool valid = v >= 0;
      // lanes 0, 8, 16, 24 hold rows 4m .. 4m+3
      const uint32_t bal = __ballot_sync(0xffffffffu, valid);
      mask |= (uint64_t)((bal & 1u) | ((bal >> 7) & 2u) | ((bal >> 14) & 4u) | ((bal >> 21) & 8u)) << (4 * m);
      const int kr = half * kChunk + r;            // key row within the split
      const uint16_t* src = p.kv + (size_t)(valid ? cr : 0) * DK + c16 * 8;
#pragma unroll
      for (int i = 0; i < 3; ++i) {
        const int a = sub + 3 * i;
        uint8_t* dst = sKV + a * kAtomBytes + kr * 128 + ((c16 ^ (kr & 7)) << 4);
        // an empty or invalid slot is zero-filled: no stale shared memory
        // meets its zero probability in P V
        cp_async16_zfill(dst, src + a * 64, valid ? 16u : 0u);
      }
    }
    if (sub == 0 && lane == 0) sMask[half] = mask;
    cp_async_commit();
    cp_async_wait<0>();
    fence_proxy_async_smem();
    mbar_arrive(&kv_full[half]);
    // drain: the Q load must have landed before this CTA's memory is reused
    if (q_issued) mbar_wait(q_full, 0, p.wait_ns, no_abort);
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      constexpr uint32_t idesc_qk = make_idesc(kFmtBF16, kFmtBF16, 0, 0, 128, 2 * kChunk);
      constexpr uint32_t idesc_pv = make_idesc(kFmtBF16, kFmtBF16, 0, 1, 128, 128);
      const uint64_t kdesc0 = make_sdesc(smem_u32(sKV), 16, 1024, kSwizzle128);
      const uint64_t qdesc0 = make_sdesc(smem_u32(sQ), 16, 1024, kSwizzle128);
      bool ok = row_ok && mbar_wait(q_full, 0, p.wait_ns, ab) && mbar_wait(q_ready, 0, p.wait_ns, ab);
      if (!ok && row_ok) fail(1);
      int issued_qk = 0, issued_pv = 0;
      // Q K^T over all 128 keys of the split as one N = 128 pass (36 MMAs
      // instead of two N = 64 passes of 36: an N = 64 MMA costs the issuing
      // thread nearly as much as an N = 128 one); both halves land together
      if (ok && (!mbar_wait(&kv_full[0], 0, p.wait_ns, ab) || !mbar_wait(&kv_full[1], 0, p.wait_ns, ab))) {
        fail(2);
        ok = false;
      }
      if (ok) {
        fence_proxy_async_smem();
        tc_fence_after();
        const uint32_t dS = tmem + kSCol;
#pragma unroll
        for (int ks = 0; ks < kKSteps; ++ks) {
          const int d = ks * 16;
          const uint64_t bdesc = kdesc0 + (uint64_t)(((d / 64) * kAtomBytes + (d % 64) * 2) >> 4);
          if (ks < kQTSteps) {
            mma_bf16_ts(dS, tmem + kQCol + ks * 8, bdesc, idesc_qk, ks > 0 ? 1u : 0u);
          } else {
            const int dq = d - kQT;
            const uint64_t adesc = qdesc0 + (uint64_t)(((dq / 64) * kQAtomBytes + (dq % 64) * 2) >> 4);
            mma_bf16(dS, adesc, bdesc, idesc_qk, ks > 0 ? 1u : 0u);
          }
        }
        // one commit per softmax side (each waits for its half's logits)
        mma_commit(&s_full[0]);
        mma_commit(&s_full[1]);
        issued_qk = 2;
      }
      if (ok && !mbar_wait(p_full, 0, p.wait_ns, ab)) { fail(3); ok = false; }
      for (int q = 0; q < 4 && ok; ++q) {
        if (q == 3 && !mbar_wait(o_free, 0, p.wait_ns, ab)) { fail(4); ok = false; break; }
        tc_fence_after();
        // O[:, 128q .. 128q + 127] = P V: V atoms 2q, 2q+1 as the MN-major B operand
        const uint64_t vdesc = make_sdesc(smem_u32(sKV) + (uint32_t)(2 * q) * kAtomBytes, kAtomBytes, 1024,
                                          kSwizzle128);
#pragma unroll
        for (int ks = 0; ks < kKeys / 16; ++ks)
          mma_bf16_ts(tmem + ocol(q), tmem + kSCol + ks * 8, vdesc + (uint64_t)((ks * 16 * 128) >> 4), idesc_pv,
                      ks > 0 ? 1u : 0u);
        mma_commit(&pv_done[q]);
        ++issued_pv;
      }
      mma_commit(mma_done);
      mbar_wait(mma_done, 0, p.wait_ns, no_abort);
      // drain the commit-fed barriers nobody else is left to wait on
      for (int c = 0; c < issued_qk; ++c) mbar_wait(&s_full[c], 0, p.wait_ns, no_abort);
      for (int q = 0; q < issued_pv; ++q) mbar_wait(&pv_done[q], 0, p.wait_ns, no_abort);
    }
  } else {
    // ------------------------------------------------------------ softmax + output
    const int side = (warp - kFirstSoftmax) >> 2;   // 64-key half of the logits; 64 columns of each O quarter
    const int quarter = warp & 3;
    const int h = quarter * 32 + lane;              // head row == TMEM lane
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
    const bool head_ok = row_ok && h < p.H;
    // Q dims [0, 256) of row h into TMEM as BF16 pairs; side s writes the
    // 64-dim blocks s and s + 2
    {
      const uint16_t* qrow = p.q + ((size_t)(head_ok ? row : 0) * p.H + (head_ok ? h : 0)) * DK;
      for (int qb = side; qb < kQT / 64; qb += 2) {
        uint32_t v[32];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          uint4 x = make_uint4(0u, 0u, 0u, 0u);
          if (head_ok) x = *reinterpret_cast<const uint4*>(qrow + qb * 64 + i * 8);
          v[4 * i] = x.x;
          v[4 * i + 1] = x.y;
          v[4 * i + 2] = x.z;
          v[4 * i + 3] = x.w;
        }
        tmem_st32(tmem + lane_addr + kQCol + qb * 32, v);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(q_ready);
    }
    bool ok = row_ok;
    const float sc = p.scale_log2;
    float m_all = -INFINITY, l = 0.f;
    // 1. this side's 64 logits and valid keys; partial maximum
    if (ok && !wwait(&s_full[side], 0)) { fail(5); ok = false; }
    if (ok && !wwait(&kv_full[side], 0)) { fail(6); ok = false; }
    if (ok) {
      tc_fence_after();
      const uint64_t mask = sMask[side];
      const uint32_t saddr = tmem + lane_addr + kSCol + side * kChunk;
      uint32_t s0[32], s1[32];
      tmem_ld32(saddr, s0);
      tmem_ld32(saddr + 32, s1);
      tmem_wait_ld_dep(s0);
      tmem_wait_ld_dep(s1);
      const uint32_t m0 = (uint32_t)mask, m1 = (uint32_t)(mask >> 32);
      float pm = -INFINITY;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        if ((m0 >> i) & 1u) pm = fmaxf(pm, __uint_as_float(s0[i]));
        if ((m1 >> i) & 1u) pm = fmaxf(pm, __uint_as_float(s1[i]));
      }
      // 2. exchange the partial maxima with the other side of this quarter
      sXM[side * 128 + h] = pm;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&mx_bar[quarter]);
      if (!wwait(&mx_bar[quarter], 0)) { fail(7); ok = false; }
      if (ok) {
        tc_fence_after();   // the other side's logits were read before its maximum was published
        m_all = fmaxf(pm, sXM[(side ^ 1) * 128 + h]);
        // 3. probabilities of this side's keys as BF16 pairs over P columns
        //    [32 side, 32 side + 32) of the S region
        uint32_t pk[32];
        float rs = 0.f;
        if (m_all == -INFINITY) {
#pragma unroll
          for (int i = 0; i < 32; ++i) pk[i] = 0u;
        } else {
          const float neg_m = -m_all * sc;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float e0 = ex2_approx(fmaf(__uint_as_float(s0[2 * i]), sc, neg_m));
            float e1 = ex2_approx(fmaf(__uint_as_float(s0[2 * i + 1]), sc, neg_m));
            if (!((m0 >> (2 * i)) & 1u)) e0 = 0.f;
            if (!((m0 >> (2 * i + 1)) & 1u)) e1 = 0.f;
            rs += e0 + e1;
            pk[i] = pack_bf16x2(e0, e1);
          }
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float e0 = ex2_approx(fmaf(__uint_as_float(s1[2 * i]), sc, neg_m));
            float e1 = ex2_approx(fmaf(__uint_as_float(s1[2 * i + 1]), sc, neg_m));
            if (!((m1 >> (2 * i)) & 1u)) e0 = 0.f;
            if (!((m1 >> (2 * i + 1)) & 1u)) e1 = 0.f;
            rs += e0 + e1;
            pk[16 + i] = pack_bf16x2(e0, e1);
          }
        }
        tmem_st32(tmem + lane_addr + kSCol + side * 32, pk);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full);
        // 4. the row sum over both sides
        sXL[side * 128 + h] = rs;
        __syncwarp();
        if (lane == 0) mbar_arrive(&lx_bar[quarter]);
        if (!wwait(&lx_bar[quarter], 0)) {
          fail(8);
          ok = false;
        } else {
          l = rs + sXL[(side ^ 1) * 128 + h];
        }
      }
    }
    // 5. read out the four O quarters (this side: 64 of each quarter's 128
    //    columns), normalised by the split's row sum
    const float inv = l > 0.f ? 1.f / l : 0.f;
    for (int q = 0; q < 4 && ok; ++q) {
      if (!wwait(&pv_done[q], 0)) { fail(9); ok = false; break; }
      tc_fence_after();
      uint32_t o0[32], o1[32];
      const uint32_t oaddr = tmem + lane_addr + ocol(q) + side * 64;
      tmem_ld32(oaddr, o0);
      tmem_ld32(oaddr + 32, o1);
      tmem_wait_ld_dep(o0);
      tmem_wait_ld_dep(o1);
      if (q == 0) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(o_free);
      }
      if (!head_ok) continue;
      const int c0 = q * 128 + side * 64;
      if (p.nsplit == 1) {
        uint4* dst = reinterpret_cast<uint4*>(p.out + ((size_t)row * p.H + h) * DV + c0);
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          const uint32_t* x = g < 4 ? &o0[8 * g] : &o1[8 * (g - 4)];
          uint4 v;
          v.x = pack_bf16x2(__uint_as_float(x[0]) * inv, __uint_as_float(x[1]) * inv);
          v.y = pack_bf16x2(__uint_as_float(x[2]) * inv, __uint_as_float(x[3]) * inv);
          v.z = pack_bf16x2(__uint_as_float(x[4]) * inv, __uint_as_float(x[5]) * inv);
          v.w = pack_bf16x2(__uint_as_float(x[6]) * inv, __uint_as_float(x[7]) * inv);
          dst[g] = v;
        }
      } else {
        uint4* dst = reinterpret_cast<uint4*>(p.part_o + (((size_t)row * p.nsplit + split) * p.H + h) * DV + c0);
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          const uint32_t* x = g < 4 ? &o0[8 * g] : &o1[8 * (g - 4)];
          uint4 v;
          v.x = pack_f16x2(__uint_as_float(x[0]) * inv, __uint_as_float(x[1]) * inv);
          v.y = pack_f16x2(__uint_as_float(x[2]) * inv, __uint_as_float(x[3]) * inv);
          v.z = pack_f16x2(__uint_as_float(x[4]) * inv, __uint_as_float(x[5]) * inv);
          v.w = pack_f16x2(__uint_as_float(x[6]) * inv, __uint_as_float(x[7]) * inv);
          dst[g] = v;
        }
      }
    }
    if (ok && head_ok && side == 0) {
      const float lse2 = l > 0.f ? m_all * sc + log2f(l) : -INFINITY;
      if (p.nsplit == 1) {
        if (p.lse != nullptr) p.lse[(size_t)row * p.H + h] = lse2 * 0.6931471805599453f;
      } else {
        p.part_lse[((size_t)row * p.nsplit + split) * p.H + h] = lse2;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Merge the splits of each (row, head): 64 threads per (row, head), eight
// value columns each (one 16-byte load of FP16 per split).  The splits are
// taken 16 at a time with every load of a batch issued before the first is
// used, so a thread waits for memory once per batch, not once per split.
__global__ void __launch_bounds__(256) attn_combine_f16_kernel(const __half* part_o, const float* part_lse,
                                                               uint16_t* out, float* lse, int rows, int H,
                                                               int nsplit) {
  constexpr int kBatch = 16;
  // results of the attention grid are visible after this
  pdl_wait();
  const long long gh = (long long)blockIdx.x * 4 + (threadIdx.x >> 6);
  if (gh >= (long long)rows * H) return;
  const int row = (int)(gh / H), h = (int)(gh - (long long)(gh / H) * H);
  const int d0 = (threadIdx.x & 63) * 8;
  const float* ls = part_lse + (size_t)row * nsplit * H + h;
  const __half* po = part_o + ((size_t)row * nsplit * H + h) * DV + d0;   // split s at + s * H * DV
  float mx = -INFINITY;
  if (nsplit > kBatch)
    for (int s = 0; s < nsplit; ++s) mx = fmaxf(mx, ls[(size_t)s * H]);
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  float wsum = 0.f;
  for (int s0 = 0; s0 < nsplit; s0 += kBatch) {
    // every load of the batch is issued at once (one memory latency): an
    // empty split's partial was never written, so its value is read and
    // then replaced by zero rather than fetched only when its lse is finite
    float l[kBatch];
    uint4 v[kBatch];
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const int s = s0 + i;
      l[i] = s < nsplit ? ls[(size_t)s * H] : -INFINITY;
      v[i] = s < nsplit ? *reinterpret_cast<const uint4*>(po + (size_t)s * H * DV) : make_uint4(0u, 0u, 0u, 0u);
    }
    if (nsplit <= kBatch) {
#pragma unroll
      for (int i = 0; i < kBatch; ++i) mx = fmaxf(mx, l[i]);
    }
    if (mx == -INFINITY) break;
    float w[kBatch];
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      w[i] = l[i] == -INFINITY ? 0.f : exp2f(l[i] - mx);
      if (l[i] == -INFINITY) v[i] = make_uint4(0u, 0u, 0u, 0u);
    }
    {
#pragma unroll
      for (int i = 0; i < kBatch; ++i) {
        wsum += w[i];
        const uint32_t u[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&u[c]));
          acc[2 * c] = fmaf(w[i], f.x, acc[2 * c]);
          acc[2 * c + 1] = fmaf(w[i], f.y, acc[2 * c + 1]);
        }
      }
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  uint4 o;
  o.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
  o.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
  o.z = pack_bf16x2(acc[4] * inv, acc[5] * inv);
  o.w = pack_bf16x2(acc[6] * inv, acc[7] * inv);
  *reinterpret_cast<uint4*>(out + ((size_t)row * H + h) * DV + d0) = o;
  if (d0 == 0 && lse != nullptr)
    lse[(size_t)row * H + h] = wsum > 0.f ? (mx + log2f(wsum)) * 0.6931471805599453f : -INFINITY;
}

}  // namespace

int attn_decode_nsplit(int k) { return (k + kKeys - 1) / kKeys; }

size_t attn_decode_partial_bytes(int rows, int H, int nsplit) {
  return nsplit > 1 ? (size_t)rows * nsplit * H * (DV * sizeof(__half) + sizeof(float)) : 0;
}

bool attn_decode_supported(const AttnArgs& a) {
  return a.d_k == DK && a.d_v == DV && a.v == nullptr && a.idx != nullptr && a.H <= 128;
}

cudaError_t launch_sparse_attn_decode(const LaunchCtx& c, const AttnArgs& a, void* part) {
  const long long rows = (long long)a.B * a.T;
  if (rows <= 0) return cudaSuccess;
  DecParams p = {};
  p.map = a.map;
  p.q = a.q;
  p.kv = a.kv;
  p.idx = a.idx;
  p.dense_rows = a.dense_rows;
  p.out = a.out;
  p.lse = a.lse;
  p.T = a.T;
  p.H = a.H;
  p.k = a.k;
  p.rows = (int)rows;
  p.nsplit = attn_decode_nsplit(a.k);
  p.scale_log2 = a.tau * 1.4426950408889634f;
  p.wait_ns = c.wait_ns;
  p.err = c.err;
  p.part_o = static_cast<__half*>(part);
  p.part_lse = part ? reinterpret_cast<float*>(static_cast<char*>(part) +
                                              (size_t)rows * p.nsplit * a.H * DV * sizeof(__half))
                    : nullptr;
  if (p.nsplit > 1 && part == nullptr) return cudaErrorInvalidValue;
  CUtensorMap tm_q;
  if (!make_tmap_2d(&tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.q, (uint64_t)rows * a.H, DK, (uint64_t)DK * 2, 128,
                    64, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  auto kern = a.map.page_size != 0 ? sparse_attn_decode_kernel<true> : sparse_attn_decode_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (e != cudaSuccess) return e;
  // a programmatic dependent of the top-k: its prologue overlaps the
  // selection's last launch, which runs only one block per row
  e = launch_pdl(kern, dim3((unsigned)(rows * p.nsplit)), dim3(kThreads), kSmem, c.stream, tm_q, p);
  if (e != cudaSuccess) return e;
  note_launches(1);
  e = cudaGetLastError();
  if (e != cudaSuccess || p.nsplit == 1) return e;
  // the merge, as a programmatic dependent launch: its blocks may start while
  // the attention grid drains and wait (griddepcontrol.wait) for its results
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((rows * a.H + 3) / 4));
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = c.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, attn_combine_f16_kernel, (const __half*)p.part_o, (const float*)p.part_lse, a.out,
                         a.lse, (int)rows, a.H, p.nsplit);
  note_launches(1);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace dsa
