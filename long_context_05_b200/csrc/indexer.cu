// Step A: lightning indexer scores on the tcgen05 tensor cores (FP8).
//
// I[t,s] = sum_j w[t,j] * ReLU(q_I[t,j] . k_I[s]) over the dequantised FP8
// operands (ouchyi thread on DeepSeek Sparse Attention, "Nasil calisiyor"
// paragraph: few heads, FP8, cheap; tenelement.pl, "DeepSeek V3.2-Exp Cuts
// Long-Context Costs ...", section "Architektura DeepSeek V3.2-Exp: Od MoE do
// DSA": logits for the context tokens through a ReLU).  Both scales are > 0,
// so ReLU(a b x) = a b ReLU(x): the MMA runs on the raw e4m3 bytes and the
// epilogue applies w * q_scale per (query, head) and k_scale per key.
//
// Tiling.  One MMA tile is M = 128 keys (A = k_I rows, K-major) by N = 128
// (query, head) rows of q_I (B, K-major), K = D_I; putting the keys on M makes
// the sum over the indexer heads a sum along one TMEM lane, i.e. inside one
// epilogue thread.  A work item is a group of up to 8 such B sub-tiles (16
// queries at 64 heads) kept in shared memory, times a run of up to 32 key
// tiles streamed through a 4-stage TMA ring; every key tile feeds all
// sub-tiles, so each byte of k_I fetched serves 8 MMAs.  Tiles entirely
// above the causal diagonal are skipped.
//
// Warp roles (one CTA per SM, persistent over the work items):
//   warp 0      TMA producer (one elected lane)
//   warp 1      TMEM allocator and MMA issuer (one elected lane)
//   warps 2..   epilogue: groups of four warps (one per TMEM lane quarter);
//               group g drains accumulator groups u with u % NGRP == g
// Four TMEM accumulators of 128 columns each.  With 32 or more indexer heads
// two consecutive key tiles share one accumulator group (two accumulators,
// one commit), so every head-weight load in the epilogue serves both; two
// epilogue groups then drain the two groups in flight (320 threads).  With
// fewer heads each key tile has its own accumulator and three epilogue
// groups run (448 threads), the MMA up to three sub-tiles ahead.  Items with
// at most half of the B sub-tiles in use (decode) double-buffer B, so the
// next item's loads overlap the current item's MMAs.
#include "internal.h"
#include "sm100.cuh"
#include "tma_host.h"

namespace dsa {
namespace {

using namespace sm100;

constexpr int kBM = 128;       // keys per tile (MMA M)
constexpr int kNSub = 128;     // MMA N: (query, head) rows per sub-tile (64 in the one-query form)
constexpr int kKC = 32;        // key tiles per work item (at most; fewer when items are scarce)
constexpr int kStages = 4;     // depth of the k_I ring
constexpr int kNAcc = 4;       // TMEM accumulators (kNAcc * NS columns)
static_assert((kNAcc & (kNAcc - 1)) == 0, "accumulator index is taken with a mask");
// Key tiles per accumulator group: with many heads (HI >= 32) two
// consecutive key tiles share one pass of the epilogue over a sub-tile, so
// every head-weight load from shared memory serves two accumulators.  The
// one-query form (NS = 64) runs one epilogue group and a small shared
// memory layout, so that two CTAs (two MMA-issuing threads) share an SM.
template <int HI, int NS>
struct EpiCfg {
  static constexpr int G = HI >= 32 ? 2 : 1;                     // key tiles per group
  static constexpr int NSLOT = kNAcc / G;                        // accumulator groups in flight
  static constexpr int NGRP = NS == 64 ? 1 : (G == 2 ? 2 : 3);   // epilogue groups of four warps
  static constexpr int EPI_THREADS = 128 * NGRP;
  static constexpr int THREADS = 64 + EPI_THREADS;
  static constexpr int CTAS_PER_SM = NS == 64 ? 2 : 1;
};

struct IdxParams {
  KvMap kv;            // per-sequence lengths, paged or contiguous key cache
  long long pool_rows; // rows of the k_I / k_scale pools
  int box_rows;        // key rows per TMA load (a key tile takes kBM / box_rows)
  int kstride;         // column s of a score row is key s * kstride (1: every key)
  const unsigned int* thr;   // candidate mode: per launch row, the smallest order key kept
  int32_t* wl_row;           // candidate lists, one per epilogue warp of the launch
  int32_t* wl_idx;
  unsigned int* wl_key;
  unsigned int* wl_cnt;
  long long wl_cap;
  int* row_fail;
  const int* row_slot;       // repair mode: score row of each launch row (-1: skip)
  const float* w;
  const float* q_scale;
  const float* k_scale;
  float* scores;
  long long ld;
  int B, T, S, q_begin, q_count;
  int nb;              // B sub-tiles per item
  int kc;              // key tiles per item
  int groups_per_seq;  // query groups per sequence
  long long wait_ns;
  DevErr* err;
};

template <int DI, int NS>
struct Layout {
  static constexpr int kMaxNB = NS == 64 ? 2 : 8;   // sub-tiles per work item
  static constexpr int kABytes = kBM * DI;
  static constexpr int kBSubBytes = NS * DI;
  static constexpr int kBOff = 0;
  static constexpr int kAOff = kBOff + kMaxNB * kBSubBytes;
  static constexpr int kWOff = kAOff + kStages * kABytes;            // wM, two item buffers
  static constexpr int kWFloats = kMaxNB * NS;
  static constexpr int kThrOff = kWOff + 2 * kWFloats * 4;           // thresholds, two item buffers
  static constexpr int kThrWords = kMaxNB * NS / 4;                  // queries per item at most (4 heads)
  static constexpr int kBarOff = kThrOff + 2 * kThrWords * 4;
  static constexpr int kNumBars = 2 * kStages + 4 + 2 * kNAcc + 1 + 2;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr int kAlloc = kBytes + 1024;  // room to align the base to 1024
  static constexpr uint32_t kSwizzleLayout = DI == 128 ? kSwizzle128 : DI == 64 ? kSwizzle64 : kSwizzle32;
  static constexpr uint32_t kSBO = 8 * DI;   // 8 rows per swizzle atom
};

// Work enumeration shared by all roles: items are (sequence, query group,
// key chunk); CTA `cta` takes every item whose flat index is cta mod grid.
struct Item {
  int b, t0, tend, c, ntiles;
  int L;    // keys of sequence b
  int off;  // L - T: pos(t) = off + t
};

template <int HI, int NS, bool PLAIN, class F>
__device__ __forceinline__ void for_each_item(const IdxParams& p, F&& f) {
  const int KS = PLAIN ? 1 : p.kstride;
  const int* const SLOT = PLAIN ? nullptr : p.row_slot;
  constexpr int QPS = NS / HI;
  const int per_group = p.nb * QPS;
  const int grid = gridDim.x, cta = blockIdx.x;
  long long flat = 0;
  const int q_end = p.q_begin + p.q_count;
  for (int gid = 0; gid < p.B * p.groups_per_seq; ++gid) {
    const int b = gid / p.groups_per_seq;
    const int g = gid - b * p.groups_per_seq;
    Item it;
    it.b = b;
    it.L = PLAIN ? p.S : p.kv.len(b, p.err, ERR_SITE_INDEXER);
    it.off = it.L - p.T;
    it.t0 = p.q_begin + g * per_group;
    it.tend = min(it.t0 + per_group, q_end);
    const int pos_last = it.off + it.tend - 1;
    it.ntiles = pos_last / KS / kBM + 1;
    const int nch = (it.ntiles + p.kc - 1) / p.kc;
    if (SLOT != nullptr) {
      // repair mode: only query groups holding a listed row are scored
      bool any = false;
      for (int t = it.t0; t < it.tend && !any; ++t) any = SLOT[(size_t)b * p.q_count + (t - p.q_begin)] >= 0;
      if (!any) continue;
    }
    int c0 = (int)(((long long)cta - flat) % grid);
    if (c0 < 0) c0 += grid;
    for (int c = c0; c < nch; c += grid) {
      it.c = c;
      if (!f(it)) return;
    }
    flat += nch;
  }
}

// Sub-tile j of an item covers queries [t0 + j*QPS, min(t0 + (j+1)*QPS, tend)).
// nsub: sub-tiles holding at least one query of the item.  For key tile kt
// the active sub-tiles (some query sees a key of the tile) are [jlo, nsub):
// the last query of sub-tile j grows with j, and the item's last query sees
// every key tile the item covers.
template <int HI, int NS>
__device__ __forceinline__ int item_nsub(const IdxParams& p, const Item& it) {
  constexpr int QPS = NS / HI;
  return min(p.nb, (it.tend - it.t0 + QPS - 1) / QPS);
}
template <int HI, int NS, bool PLAIN>
__device__ __forceinline__ int first_active(const IdxParams& p, const Item& it, int kt, int nsub) {
  constexpr int QPS = NS / HI;
  // smallest j with t0 + (j + 1) * QPS - 1 >= kt * kBM * kstride - off
  const int x = kt * kBM * (PLAIN ? 1 : p.kstride) - it.off - it.t0 + QPS;
  const int j = x > 0 ? x / QPS - 1 : 0;
  return j < 0 ? 0 : (j < nsub - 1 ? j : nsub - 1);
}

// PLAIN: every key of a contiguous cache of S keys per sequence scored into
// score rows (no per-sequence lengths, stride 1, no thresholds, no repair
// list); the general form adds lengths, paged caches, the key sample, the
// candidate and the repair modes, whose checks the plain form must not pay.
// CAND: candidate mode (thr set).  With PLAIN it keeps the contiguous
// fast paths while appending candidates instead of storing scores.
// NS: MMA N, the (query, head) rows of a sub-tile: 128, or 64 where every
// sequence has one query (decode), so that no half of a sub-tile is padding.
template <int DI, int HI, bool PLAIN, bool CAND, int NS>
__global__ void __launch_bounds__(EpiCfg<HI, NS>::THREADS, EpiCfg<HI, NS>::CTAS_PER_SM)
    indexer_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
                      IdxParams p) {
  using L = Layout<DI, NS>;
  constexpr int QPS = NS / HI;
  // the plain form sees constants: no sample stride, no candidates, no repair
  const int KS = PLAIN ? 1 : p.kstride;
  const unsigned int* const THR = CAND ? p.thr : nullptr;
  const int* const SLOT = PLAIN ? nullptr : p.row_slot;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sB = smem + L::kBOff;
  uint8_t* sA = smem + L::kAOff;
  float* sW = reinterpret_cast<float*>(smem + L::kWOff);
  unsigned int* sThr = reinterpret_cast<unsigned int*>(smem + L::kThrOff);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* a_full = bars;
  uint64_t* a_empty = bars + kStages;
  uint64_t* b_full = bars + 2 * kStages;       // [2] B buffer loaded (TMA)
  uint64_t* b_empty = b_full + 2;              // [2] B buffer free (MMA commit)
  uint64_t* acc_full = b_empty + 2;
  uint64_t* acc_empty = acc_full + kNAcc;
  uint64_t* mma_done = acc_empty + kNAcc;
  uint64_t* w_ready = mma_done + 1;  // [2]: epilogue threads finished filling wM buffer
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // a programmatically dependent kernel (the decode top-k) may be scheduled
  // now; it waits for this grid's scores before reading them
  pdl_launch_dependents();
  // With at most half of the B sub-tiles in use (few queries per item, as in
  // decode), the B region holds two item buffers, so the next item's B and
  // its first key tiles load while the current item's MMAs run.
  const int nbbuf = p.nb * 2 <= L::kMaxNB ? 2 : 1;
  constexpr int kBBufBytes = L::kMaxNB / 2 * L::kBSubBytes;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&a_full[i], 1);
      mbar_init(&a_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&b_full[i], 1);
      mbar_init(&b_empty[i], 1);
    }
    for (int i = 0; i < kNAcc; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);  // one arrive per epilogue warp of the owning group
    }
    mbar_init(mma_done, 1);
    mbar_init(&w_ready[0], EpiCfg<HI, NS>::EPI_THREADS);
    mbar_init(&w_ready[1], EpiCfg<HI, NS>::EPI_THREADS);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kNAcc * NS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const AbortSources ab{abort_flag, &p.err->code};
  const AbortSources no_abort{nullptr, nullptr};  // drains of this CTA's own async work
  auto fail = [&](unsigned where) {
    report_error(p.err, DSA_ERR_TIMEOUT, ERR_SITE_INDEXER | (where << 8));
    *abort_flag = 1;
  };

  if (warp == 0) {
    // ---------------------------------------------------------- TMA producer
    if (lane == 0) {
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_q);
      uint32_t a_cnt = 0, items = 0;
      uint32_t last_phase[kStages];
      bool issued[kStages];
      for (int i = 0; i < kStages; ++i) issued[i] = false;
      bool ok = true;
      for_each_item<HI, NS, PLAIN>(p, [&](const Item& it) {
        const int bb = nbbuf == 2 ? (int)(items & 1) : 0;
        const uint32_t use = nbbuf == 2 ? items >> 1 : items;
        if (!mbar_wait(&b_empty[bb], (use & 1) ^ 1, p.wait_ns, ab)) { fail(1); ok = false; return false; }
        int nsub = 0;
        for (int j = 0; j < p.nb; ++j)
          if (it.t0 + j * QPS < it.tend) nsub = j + 1;
        mbar_arrive_expect_tx(&b_full[bb], nsub * L::kBSubBytes);
        for (int j = 0; j < nsub; ++j)
          tma_load_2d(sB + bb * kBBufBytes + j * L::kBSubBytes, &tm_q, &b_full[bb], 0, (it.b * p.T + it.t0 + j * QPS) * HI);
        ++items;
        const int kt0 = it.c * p.kc, kt1 = min(kt0 + p.kc, it.ntiles);
        for (int kt = kt0; kt < kt1; ++kt, ++a_cnt) {
          const int st = a_cnt % kStages;
          if (!mbar_wait(&a_empty[st], ((a_cnt / kStages) & 1) ^ 1, p.wait_ns, ab)) {
            fail(2); ok = false; return false;
          }
          mbar_arrive_expect_tx(&a_full[st], L::kABytes);
          // the tile's keys in runs of box_rows cache rows (a whole tile when
          // the cache is contiguous); a run at or past L_b, or on an unmapped
          // page, reads the fill value from past the end of the pool
          if constexpr (PLAIN) {
            tma_load_2d(sA + st * L::kABytes, &tm_k, &a_full[st], 0, it.b * p.S + kt * kBM);
          } else {
          for (int r0 = 0; r0 < kBM; r0 += p.box_rows) {
            const int s = (kt * kBM + r0) * KS;
            // a key sample is a contiguous cache read every kstride-th row:
            // row b * (S / kstride) + sample index of the strided map
            long long y = s >= it.L ? -1
                          : KS == 1 ? p.kv.row<!PLAIN>(it.b, s)
                                           : (long long)it.b * (p.S / KS) + kt * kBM + r0;
            if (y < 0) {
              if (s < it.L) report_error(p.err, DSA_ERR_DEVICE_BOUNDS, ERR_SITE_INDEXER | (2u << 8));
              y = p.pool_rows;
            }
            tma_load_2d(sA + st * L::kABytes + r0 * DI, &tm_k, &a_full[st], 0, (int)y);
          }
          }
          issued[st] = true;
          last_phase[st] = (a_cnt / kStages) & 1;
        }
        return true;
      });
      // let every load this CTA started land before it exits
      for (int st = 0; st < kStages; ++st)
        if (issued[st]) mbar_wait(&a_full[st], last_phase[st], p.wait_ns, no_abort);
      for (uint32_t i = items > 2 ? items - 2 : 0; i < items; ++i) {
        const int bb = nbbuf == 2 ? (int)(i & 1) : 0;
        const uint32_t use = nbbuf == 2 ? i >> 1 : i;
        if (nbbuf == 2 || i + 1 == items) mbar_wait(&b_full[bb], use & 1, p.wait_ns, no_abort);
      }
      (void)ok;
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = make_idesc(kFmtE4M3, kFmtE4M3, 0, 0, kBM, NS);
      using E = EpiCfg<HI, NS>;
      uint32_t a_cnt = 0, items = 0, u = 0;
      // descriptors built once; a stage or sub-tile only adds its offset >> 4
      const uint64_t adesc0 = make_sdesc(smem_u32(sA), 16, L::kSBO, L::kSwizzleLayout);
      const uint64_t bdesc0 = make_sdesc(smem_u32(sB), 16, L::kSBO, L::kSwizzleLayout);
      for_each_item<HI, NS, PLAIN>(p, [&](const Item& it) {
        const int bb = nbbuf == 2 ? (int)(items & 1) : 0;
        const uint32_t use = nbbuf == 2 ? items >> 1 : items;
        if (!mbar_wait(&b_full[bb], use & 1, p.wait_ns, ab)) { fail(3); return false; }
        ++items;
        const uint64_t bdesc_it = bdesc0 + (uint64_t)((bb * kBBufBytes) >> 4);
        const int nsub = item_nsub<HI, NS>(p, it);
        const int kt0 = it.c * p.kc, kt1 = min(kt0 + p.kc, it.ntiles);
        for (int kt = kt0; kt < kt1; kt += E::G) {
          // key tiles kt .. kt + ng - 1 of this group, each in its ring stage
          const int ng = min(E::G, kt1 - kt);
          uint64_t adesc[E::G];
#pragma unroll
          for (int g = 0; g < E::G; ++g) {
            if (g >= ng) break;
            const uint32_t c = a_cnt + (uint32_t)g;
            const int st = c % kStages;
            if (!mbar_wait(&a_full[st], (c / kStages) & 1, p.wait_ns, ab)) { fail(4); return false; }
            adesc[g] = adesc0 + (uint64_t)((st * L::kABytes) >> 4);
          }
          tc_fence_after();
          // the first active sub-tile of kt also covers kt + 1 (later keys
          // need later queries); masked pairs are computed and dropped
          for (int j = first_active<HI, NS, PLAIN>(p, it, kt, nsub); j < nsub; ++j) {
            const int slot = u % E::NSLOT;
            if (!mbar_test_wait(&acc_empty[slot], ((u / E::NSLOT) & 1) ^ 1) &&
                !mbar_wait(&acc_empty[slot], ((u / E::NSLOT) & 1) ^ 1, p.wait_ns, ab)) {
              fail(5);
              return false;
            }
            tc_fence_after();
            const uint64_t bdesc = bdesc_it + (uint64_t)((j * L::kBSubBytes) >> 4);
#pragma unroll
            for (int g = 0; g < E::G; ++g) {
              if (g >= ng) break;
              const uint32_t dacc = tmem_base + (slot * E::G + g) * NS;
#pragma unroll
              for (int ks = 0; ks < DI / 32; ++ks)
                mma_f8(dacc, adesc[g] + 2 * ks, bdesc + 2 * ks, idesc, ks > 0 ? 1u : 0u);
            }
            mma_commit(&acc_full[slot]);
            ++u;
          }
#pragma unroll
          for (int g = 0; g < E::G; ++g) {
            if (g >= ng) break;
            mma_commit(&a_empty[(a_cnt + (uint32_t)g) % kStages]);
          }
          a_cnt += (uint32_t)ng;
        }
        mma_commit(&b_empty[bb]);
        return true;
      });
      mma_commit(mma_done);
      mbar_wait(mma_done, 0, p.wait_ns, no_abort);
    }
  } else {
    // ---------------------------------------------------------- epilogue
    using E = EpiCfg<HI, NS>;
    const int ew = warp - 2;             // 0 .. 4 * NGRP - 1
    const int grp = ew >> 2;             // drains groups u with u % NGRP == grp
    const int quarter = warp & 3;        // TMEM lane quarter this warp may access
    const int r = quarter * 32 + lane;   // key row within a tile
    const int etid = threadIdx.x - 64;
    uint32_t u = 0, items = 0;
    // candidate mode: this warp's list and its length (warp-uniform)
    const long long wl0 = ((long long)blockIdx.x * (E::EPI_THREADS / 32) + ew) * p.wl_cap;
    long long wpos = 0;
    for_each_item<HI, NS, PLAIN>(p, [&](const Item& it) {
      // per-item head weights  wM[(query, head)] = w * q_scale  (0 past the end)
      float* wbuf = sW + (items & 1) * L::kWFloats;
      for (int x = etid; x < p.nb * NS; x += E::EPI_THREADS) {
        const int t = it.t0 + x / HI;
        float v = 0.f;
        if (t < it.tend) {
          const size_t o = ((size_t)it.b * p.T + t) * HI + (x % HI);
          v = p.w[o] * p.q_scale[o];
        }
        wbuf[x] = v;
      }
      if (THR != nullptr) {
        unsigned int* tbuf = sThr + (items & 1) * L::kThrWords;
        for (int x = etid; x < p.nb * QPS; x += E::EPI_THREADS) {
          const int t = it.t0 + x;
          tbuf[x] = t < it.tend ? THR[(size_t)it.b * p.q_count + (t - p.q_begin)] : 0xFFFFFFFFu;
        }
      }
      mbar_arrive(&w_ready[items & 1]);
      if (!mbar_wait(&w_ready[items & 1], (items >> 1) & 1, p.wait_ns, ab)) { fail(7); return false; }
      const unsigned int* tq = sThr + (items & 1) * L::kThrWords;
      ++items;
      const int nsub = item_nsub<HI, NS>(p, it);
      const int kt0 = it.c * p.kc, kt1 = min(kt0 + p.kc, it.ntiles);
      for (int kt = kt0; kt < kt1; kt += E::G) {
        const int ng = min(E::G, kt1 - kt);
        int sg[E::G], spos[E::G];
        float ksg[E::G];
#pragma unroll
        for (int g = 0; g < E::G; ++g) {
          sg[g] = (kt + g) * kBM + r;
          // 1/2: the head sum below accumulates 2 ReLU(x)
          spos[g] = sg[g] * KS;   // key position of column sg[g]
          if constexpr (PLAIN) {
            ksg[g] = (g < ng && sg[g] < p.S) ? 0.5f * p.k_scale[(size_t)it.b * p.S + sg[g]] : 0.f;
          } else {
            const long long kr = (g < ng && spos[g] < it.L) ? p.kv.row<true>(it.b, spos[g]) : -1;
            ksg[g] = kr >= 0 ? 0.5f * p.k_scale[kr] : 0.f;
          }
        }
        const int jlo = first_active<HI, NS, PLAIN>(p, it, kt, nsub);
        const uint32_t u0 = u;
        u += (uint32_t)(nsub - jlo);
        // this group's sub-tiles: my = u0 + (j - jlo) == grp (mod NGRP)
        const int skip = (int)((grp + E::NGRP - (int)(u0 % E::NGRP)) % E::NGRP);
        for (int j = jlo + skip; j < nsub; j += E::NGRP) {
          const uint32_t my = u0 + (uint32_t)(j - jlo);
          const int slot = my % E::NSLOT;
          const bool got = mbar_wait(&acc_full[slot], (my / E::NSLOT) & 1, p.wait_ns, ab);
          if (!__all_sync(0xffffffffu, got)) { fail(6); return false; }
          tc_fence_after();
          const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + slot * E::G * NS;
          const float* wq = wbuf + j * NS;
          // w * ReLU(x) summed over the heads of each query, for each key tile
          // of the group; four independent packed-pair partial sums per
          // (tile, query) keep the FMA chains short.  ReLU is formed as
          // x + |x| = 2 ReLU(x) (exact in floating point: 2x or +0) with one
          // packed add, on the FMA pipe instead of two ALU max operations;
          // the factor 2 is removed exactly by folding 1/2 into k_scale
          constexpr int NP = HI >= 8 ? 4 : 2;
          constexpr int CW = 16;                      // TMEM columns per load
          float2 part[E::G][QPS][NP];
#pragma unroll
          for (int g = 0; g < E::G; ++g)
#pragma unroll
            for (int q = 0; q < QPS; ++q)
#pragma unroll
              for (int i = 0; i < NP; ++i) part[g][q][i] = make_float2(0.f, 0.f);
          uint32_t v[2][E::G][CW];
#pragma unroll
          for (int g = 0; g < E::G; ++g) tmem_ld16(taddr + g * NS, v[0][g]);
#pragma unroll
          for (int g = 0; g < E::G; ++g) tmem_wait_ld_dep(v[0][g]);
#pragma unroll
          for (int c = 0; c < NS / CW; ++c) {
            if (c + 1 < NS / CW) {
#pragma unroll
              for (int g = 0; g < E::G; ++g) tmem_ld16(taddr + g * NS + (c + 1) * CW, v[(c + 1) & 1][g]);
            } else {
              // every column of the group's accumulators is in registers
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&acc_empty[slot]);
            }
#pragma unroll
            for (int e = 0; e < CW; e += 2 * NP) {
              const int q = (c * CW + e) / HI;
#pragma unroll
              for (int i = 0; i < NP; i += 2) {
                const float4 w4 = *reinterpret_cast<const float4*>(wq + c * CW + e + 2 * i);
#pragma unroll
                for (int g = 0; g < E::G; ++g) {
                  const uint32_t* x = &v[c & 1][g][e + 2 * i];
                  const float2 a0 = make_float2(__uint_as_float(x[0]), __uint_as_float(x[1]));
                  const float2 a1 = make_float2(__uint_as_float(x[2]), __uint_as_float(x[3]));
                  const float2 r0 = __fadd2_rn(a0, make_float2(fabsf(a0.x), fabsf(a0.y)));
                  const float2 r1 = __fadd2_rn(a1, make_float2(fabsf(a1.x), fabsf(a1.y)));
                  part[g][q][i] = __ffma2_rn(make_float2(w4.x, w4.y), r0, part[g][q][i]);
                  part[g][q][i + 1] = __ffma2_rn(make_float2(w4.z, w4.w), r1, part[g][q][i + 1]);
                }
              }
            }
            if (c + 1 < NS / CW) {
#pragma unroll
              for (int g = 0; g < E::G; ++g) tmem_wait_ld_dep(v[(c + 1) & 1][g]);
            }
          }
#pragma unroll
          for (int g = 0; g < E::G; ++g) {
            if (g >= ng) break;
            const int s = sg[g];
            const int sp = spos[g];
#pragma unroll
            for (int q = 0; q < QPS; ++q) {
              float a = 0.f;
#pragma unroll
              for (int i = 0; i < NP; ++i) a += part[g][q][i].x + part[g][q][i].y;
              const int t = it.t0 + j * QPS + q;
              const bool vis = t < it.tend && sp <= it.off + t;
              if constexpr (PLAIN && !CAND) {
                if (vis) {
                  // self-check: the score slot lies inside this launch's tile
                  const long long ri = (long long)it.b * p.q_count + (t - p.q_begin);
                  if (ri >= 0 && ri < (long long)p.B * p.q_count && s >= 0 && s < p.ld)
                    p.scores[ri * p.ld + s] = a * ksg[g];
                  else
                    report_error(p.err, DSA_ERR_DEVICE_BOUNDS, ERR_SITE_INDEXER | (1u << 8));
                }
              } else if constexpr (!CAND) {
                if (vis) {
                  // self-check: the score slot lies inside this launch's tile
                  const long long ri = (long long)it.b * p.q_count + (t - p.q_begin);
                  const bool in_tile = ri >= 0 && ri < (long long)p.B * p.q_count && s >= 0 && s < p.ld;
                  const long long so = !in_tile ? -1 : (SLOT != nullptr ? SLOT[ri] : ri);
                  if (so >= 0)
                    p.scores[so * p.ld + s] = a * ksg[g];
                  else if (!in_tile)
                    report_error(p.err, DSA_ERR_DEVICE_BOUNDS, ERR_SITE_INDEXER | (1u << 8));
                }
              } else {
                const long long ri = (long long)it.b * p.q_count + (t - p.q_begin);
                // candidate mode: append the scores at or above the row's
                // threshold to this warp's own list (the 32 lanes hold 32
                // consecutive keys of the same query: a ballot gives each
                // taking lane its slot, with no atomic)
                const unsigned int key = order_key(a * ksg[g]);
                const bool take = vis && key >= tq[j * QPS + q];
                const unsigned int m = __ballot_sync(0xffffffffu, take);
                if (take) {
                  const long long o = wpos + __popc(m & ((1u << lane) - 1u));
                  if (ri >= 0 && ri < (long long)p.B * p.q_count) {
                    if (o < p.wl_cap) {
                      p.wl_row[wl0 + o] = (int32_t)ri;
                      p.wl_idx[wl0 + o] = sp;
                      p.wl_key[wl0 + o] = key;
                    } else {
                      p.row_fail[ri] = 1;   // dropped: the row is repaired later
                    }
                  } else {
                    report_error(p.err, DSA_ERR_DEVICE_BOUNDS, ERR_SITE_INDEXER | (3u << 8));
                  }
                }
                wpos += __popc(m);
              }
            }
          }
        }
      }
      return true;
    });
    if (THR != nullptr && lane == 0)
      p.wl_cnt[blockIdx.x * (E::EPI_THREADS / 32) + ew] = (unsigned int)(wpos < p.wl_cap ? wpos : p.wl_cap);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kNAcc * NS);
  }
}

template <int DI, int HI, int NS>
cudaError_t launch_tc(const LaunchCtx& c, const IndexerArgs& a) {
  using L = Layout<DI, NS>;
  constexpr int QPS = NS / HI;
  CUtensorMap tm_k, tm_q;
  const CUtensorMapSwizzle sw = DI == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                : DI == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                           : CU_TENSOR_MAP_SWIZZLE_32B;
  // key rows per TMA load: a whole tile, or the largest power of two that
  // divides the page size (every load then stays inside one page)
  int box_rows = kBM;
  if (a.kv.page_size > 0)
    while (a.kv.page_size % box_rows != 0) box_rows >>= 1;
  const long long pool_rows = a.kv.pool_rows(a.B);
  if (box_rows < 16 || pool_rows <= 0 || pool_rows >= (1LL << 31)) return cudaErrorInvalidValue;
  // a key sample (kstride > 1) reads every kstride-th row of a contiguous
  // cache: a tensor map whose row pitch is kstride rows
  const int ks = a.kstride > 1 ? a.kstride : 1;
  if (ks > 1 && (a.kv.page_size != 0 || a.S % ks != 0)) return cudaErrorInvalidValue;
  if (!make_tmap_2d(&tm_k, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.k_I, (uint64_t)(pool_rows / ks), DI,
                    (uint64_t)DI * ks, box_rows, DI, sw))
    return cudaErrorInvalidValue;
  if (!make_tmap_2d(&tm_q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.q_I, (uint64_t)a.B * a.T * HI, DI, DI, NS, DI, sw))
    return cudaErrorInvalidValue;
  IdxParams p = {};
  p.kv = a.kv;
  p.pool_rows = pool_rows;
  p.box_rows = box_rows;
  p.kstride = ks;
  p.thr = a.thr;
  p.wl_row = a.wl_row;
  p.wl_idx = a.wl_idx;
  p.wl_key = a.wl_key;
  p.wl_cnt = a.wl_cnt;
  p.wl_cap = a.wl_cap;
  p.row_fail = a.row_fail;
  p.row_slot = a.row_slot;
  p.w = a.w;
  p.q_scale = a.q_scale;
  p.k_scale = a.k_scale;
  p.scores = a.scores;
  p.ld = a.ld;
  p.B = a.B;
  p.T = a.T;
  p.S = a.S;
  p.q_begin = a.q_begin;
  p.q_count = a.q_count;
  p.nb = (a.q_count + QPS - 1) / QPS;
  if (p.nb > L::kMaxNB) p.nb = L::kMaxNB;
  const int per_group = p.nb * QPS;
  p.groups_per_seq = (a.q_count + per_group - 1) / per_group;
  p.wait_ns = c.wait_ns;
  p.err = c.err;
  // count the items to size the grid; with few query groups (decode) use
  // shorter key runs so that every SM gets several items
  auto count_items = [&](int kc) {
    long long n = 0;
    for (int g = 0; g < p.groups_per_seq; ++g) {
      const int t0 = a.q_begin + g * per_group;
      const int tend = t0 + per_group < a.q_begin + a.q_count ? t0 + per_group : a.q_begin + a.q_count;
      const int ntiles = (a.S - a.T + tend - 1) / ks / kBM + 1;
      n += (ntiles + kc - 1) / kc;
    }
    return n * a.B;
  };
  // CTA slots of the grid (the one-query form runs two CTAs per SM)
  const int slots = EpiCfg<HI, NS>::CTAS_PER_SM * c.num_sms;
  p.kc = kKC;
  long long items = count_items(p.kc);
  if (items < 4LL * slots) {
    // few items (decode: one query group per sequence): the key-run length
    // that gives the busiest CTA the fewest key tiles, then the fewest items
    // (each item reloads its queries and weights)
    long long best = -1;
    for (int kc = kKC; kc >= 4; --kc) {
      const long long n = count_items(kc);
      const long long load = (n + slots - 1) / slots * kc;
      if (best < 0 || load < best) {
        best = load;
        p.kc = kc;
        items = n;
      }
    }
  }
  const int grid = (int)(items < slots ? items : slots);
  if (grid <= 0) return cudaSuccess;
  // the contiguous fast paths (no lengths, no paging, stride 1, no repair
  // list), with score rows or candidate lists as the output
  const bool plain = ks == 1 && p.row_slot == nullptr && a.kv.page_size == 0 && a.kv.seqlens == nullptr;
  const bool cand = p.thr != nullptr;
  auto kern = cand ? (plain ? indexer_tc_kernel<DI, HI, true, true, NS> : indexer_tc_kernel<DI, HI, false, true, NS>)
                   : (plain ? indexer_tc_kernel<DI, HI, true, false, NS>
                            : indexer_tc_kernel<DI, HI, false, false, NS>);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
  if (e != cudaSuccess) return e;
  kern<<<grid, EpiCfg<HI, NS>::THREADS, L::kAlloc, c.stream>>>(tm_k, tm_q, p);
  note_launches(1);
  return cudaGetLastError();
}

template <int DI>
cudaError_t launch_di(const LaunchCtx& c, const IndexerArgs& a) {
  switch (a.H_I) {
    case 4: return launch_tc<DI, 4, kNSub>(c, a);
    case 8: return launch_tc<DI, 8, kNSub>(c, a);
    case 16: return launch_tc<DI, 16, kNSub>(c, a);
    case 32: return launch_tc<DI, 32, kNSub>(c, a);
    // one query per sequence (decode, scores out): sub-tiles of one query's
    // 64 heads, two CTAs per SM
    case 64:
      return a.q_count == 1 && a.thr == nullptr ? launch_tc<DI, 64, 64>(c, a) : launch_tc<DI, 64, kNSub>(c, a);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

int indexer_epilogue_warps(int H_I) {
  return (H_I >= 32 ? EpiCfg<64, kNSub>::EPI_THREADS : EpiCfg<4, kNSub>::EPI_THREADS) / 32;
}

cudaError_t launch_indexer(const LaunchCtx& c, const IndexerArgs& a) {
  if (a.q_count <= 0 || a.B <= 0) return cudaSuccess;
  switch (a.D_I) {
    case 32: return launch_di<32>(c, a);
    case 64: return launch_di<64>(c, a);
    case 128: return launch_di<128>(c, a);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace dsa
