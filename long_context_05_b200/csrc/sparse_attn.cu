// Step C: sparse MQA/MLA attention over the selected keys, on tcgen05.
//
// out[t,h] = sum_{s in idx[t]} softmax_s(tau q[t,h] . kv[s]) kv[s, :d_v]
// (ouchyi thread, "Nasil calisiyor" paragraph: the expensive attention runs
// only over the kept subset; tenelement.pl, section "Architektura ...",
// "Integracja z MLA" bullet: MQA form, one KV row shared by all heads;
// degnora.com, "MLA - Multi-Latent Attention": keys and values come from the
// one cached latent, so V is the first d_v columns of the row).
//
// One query row is handled by a cluster of two CTAs.  All heads of the query
// form the MMA M dimension (128 rows; fewer heads are padded with zero rows).
// A 128 x 512 FP32 output accumulator would fill all of TMEM, so the work is
// split across the pair without duplicating any MMA:
//   * the key dimension of Q.K^T is halved: CTA r keeps its half of Q in TMEM
//     (the A operand) and computes a partial logit tile S_r = Q_r K_r^T;
//   * the two partial tiles are exchanged through distributed shared memory
//     (plain shared::cluster stores published by a release arrive on the
//     peer's mbarrier) and both CTAs form the same S = S_0 + S_1, so both take
//     identical softmax decisions;
//   * each CTA multiplies P by its half of V (256 of the 512 value columns)
//     and owns that half of the output.
// Keys arrive in chunks of 64 selected rows gathered with 16-byte cp.async
// into a 3-stage ring (each CTA fetches only the 64-column atoms it uses).
// Online softmax in base 2 with a lazy rescale: the running maximum moves
// only when a chunk exceeds it by more than 8 (so p <= 256), and then the
// output accumulator in TMEM is rescaled once.
//
// Warp roles (224 threads): warps 0-1 gather, warp 2 issues MMAs and owns
// TMEM, warps 3-6 run the softmax (thread = head row) and the output.
// Decode splits the selected keys of each query over several clusters and
// merges the partial results with a combine kernel (LSE weighting).
#include <cuda_bf16.h>

#include "internal.h"
#include "sm100.cuh"

namespace dsa {
namespace {

using namespace sm100;

constexpr int kN = 64;          // selected keys per chunk (MMA N of Q.K^T, K of P.V)
constexpr int kStages = 3;
constexpr int kThreads = 224;
constexpr int kProducers = 64;  // warps 0-1
constexpr int kMmaWarp = 2;
constexpr int kSoftWarp0 = 3;   // warps 3-6
constexpr uint32_t kOCol = 0, kSCol = 256, kQCol = 320, kTmemCols = 512;
constexpr float kRescaleThreshold = 8.f;  // log2 units

template <int DK, int DV>
struct Cfg {
  static constexpr int KSTEPS = DK / 16;           // 16-wide MMA K steps over the key dim
  static constexpr int KS0 = (KSTEPS + 1) / 2;     // steps of rank 0; rank 1 takes the rest
  static constexpr bool SPLIT_V = DV >= 128;       // value columns split across the pair
  static constexpr int DVH = SPLIT_V ? DV / 2 : DV;
  __host__ __device__ static constexpr int qk_lo(int r) { return r == 0 ? 0 : KS0 * 16; }
  __host__ __device__ static constexpr int qk_hi(int r) { return r == 0 ? KS0 * 16 : DK; }
  __host__ __device__ static constexpr int ks_of(int r) { return r == 0 ? KS0 : KSTEPS - KS0; }
  __host__ __device__ static constexpr int v_lo(int r) { return SPLIT_V ? r * DVH : 0; }
  __host__ __device__ static constexpr int cmin(int a, int b) { return a < b ? a : b; }
  __host__ __device__ static constexpr int cmax(int a, int b) { return a > b ? a : b; }
  __host__ __device__ static constexpr int atom_lo(int r) { return cmin(qk_lo(r), v_lo(r)) / 64; }
  __host__ __device__ static constexpr int atom_hi(int r) { return (cmax(qk_hi(r), v_lo(r) + DVH) + 63) / 64; }
  static constexpr int NATOM = cmax(atom_hi(0) - atom_lo(0), atom_hi(1) - atom_lo(1));
  static constexpr int ATOM_BYTES = kN * 128;
  static constexpr int STAGE_BYTES = NATOM * ATOM_BYTES;
  static constexpr int P_BYTES = 128 * kN * 2;
  static constexpr int X_BYTES = 128 * kN * 4;
  static constexpr int OFF_KV = 0;
  static constexpr int OFF_P = OFF_KV + kStages * STAGE_BYTES;
  static constexpr int OFF_X = OFF_P + 2 * P_BYTES;
  static constexpr int OFF_META = OFF_X + 2 * X_BYTES;         // valid flags, kStages x kN bytes
  static constexpr int OFF_BAR = OFF_META + kStages * kN;
  static constexpr int NBARS = 2 * kStages + 1 + 2 + 2 + 2 + 2 + 2 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBARS * 8;
  static constexpr int BYTES = OFF_MISC + 32;
  static constexpr int ALLOC = BYTES + 1024;
  static_assert(DVH <= 256 && DVH % 16 == 0, "value columns per CTA");
  static_assert(KS0 * 8 + kQCol <= kTmemCols, "Q half must fit in TMEM");
};

struct AttnParams {
  const uint16_t* q;
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
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    sparse_attn_tc_kernel(AttnParams p) {
  using C = Cfg<DK, DV>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sKV = smem + C::OFF_KV;
  uint8_t* sP = smem + C::OFF_P;
  float* sX = reinterpret_cast<float*>(smem + C::OFF_X);
  uint8_t* sMeta = smem + C::OFF_META;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = bars + kStages;
  uint64_t* q_ready = bars + 2 * kStages;
  uint64_t* s_full = q_ready + 1;       // [2]: index 0 used; 1 spare
  uint64_t* s_free = s_full + 2;        // [2]: index 0 used
  uint64_t* p_full = s_free + 2;        // [2]
  uint64_t* pv_done = p_full + 2;       // [2]
  uint64_t* x_full = pv_done + 2;       // [2]: peer's partial logits landed (128 remote arrivals)
  uint64_t* peer_free = x_full + 2;     // [2]: peer consumed what we wrote
  uint64_t* mma_done = peer_free + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  // chunk each role is on (diagnostics for a timeout): producer, MMA, softmax
  volatile int* prog = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 8);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const uint32_t peer = rank ^ 1u;
  const int cid = blockIdx.x >> 1;
  const int row = cid / p.nsplit;          // b * T + t
  const int split = cid - row * p.nsplit;
  const int b = row / p.T;
  const int slot0 = split * p.kc;
  const int slot1 = min(p.k, slot0 + p.kc);
  // self-check: a cluster outside the launch's rows does no work
  const bool row_ok = row >= 0 && row < p.rows && split >= 0 && split < p.nsplit && slot0 >= 0;
  const int nchunks = row_ok ? (slot1 - slot0 + kN - 1) / kN : 0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&kv_full[i], kProducers);
      mbar_init(&kv_empty[i], 1);
    }
    mbar_init(q_ready, 4);
    mbar_init(&s_full[0], 1);
    mbar_init(&s_free[0], 4);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&p_full[i], 4);
      mbar_init(&pv_done[i], 1);
      mbar_init(&x_full[i], 128);
      mbar_init(&peer_free[i], 128);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    prog[0] = prog[1] = prog[2] = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  cluster_sync_all();  // barriers of both CTAs initialised and armed
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const AbortSources ab{abort_flag, &p.err->code};
  const AbortSources no_abort{nullptr, nullptr};  // drains of this CTA's own async work
  // detail: site | where << 8 | rank << 12 | producer, MMA, softmax chunk (6 bits each)
  auto fail = [&](unsigned where) {
    const unsigned d = ERR_SITE_ATTN | ((where & 15u) << 8) | (rank << 12) | ((unsigned)(prog[0] & 63) << 13) |
                       ((unsigned)(prog[1] & 63) << 19) | ((unsigned)(prog[2] & 63) << 25);
    report_error(p.err, DSA_ERR_TIMEOUT, d);
    *abort_flag = 1;
  };
  const int atom_lo = C::atom_lo(rank);
  const int atom_hi = C::atom_hi(rank);

  if (warp < 2) {
    // ------------------------------------------------------------ gather
    const int pt = threadIdx.x;        // 0..63
    const int c16 = pt & 7, rg = pt >> 3;
    const int32_t* irow = p.idx + (size_t)row * p.k;
    const uint16_t* kvb = p.kv + (size_t)b * p.S * DK;
    bool ok = true;
    for (int j = 0; j < nchunks && ok; ++j) {
      const int st = j % kStages;
      if (pt == 0) prog[0] = j;
      if (!mbar_wait(&kv_empty[st], ((j / kStages) & 1) ^ 1, p.wait_ns, ab)) { fail(1); ok = false; break; }
      uint8_t* stage = sKV + st * C::STAGE_BYTES;
#pragma unroll
      for (int m = 0; m < kN / 8; ++m) {
        const int r = rg + 8 * m;
        const int slot = slot0 + j * kN + r;
        int iv = slot < slot1 ? irow[slot] : -1;
        if (iv >= p.S) {
          if (c16 == 0) report_error(p.err, DSA_ERR_DEVICE_BOUNDS, ERR_SITE_ATTN);
          iv = -1;
        }
        const bool valid = iv >= 0;
        if (c16 == 0) sMeta[st * kN + r] = valid ? 1 : 0;
        const uint16_t* src = kvb + (size_t)(valid ? iv : 0) * DK;
        for (int a = atom_lo; a < atom_hi; ++a) {
          const int doff = (a - atom_lo) * C::ATOM_BYTES + r * 128 + ((c16 ^ (r & 7)) << 4);
          if (a * 128 + c16 * 16 < DK * 2) {
            if (doff >= 0 && doff + 16 <= C::STAGE_BYTES)  // self-check: inside the stage
              cp_async16(stage + doff, src + a * 64 + c16 * 8);
            else
              report_error(p.err, DSA_ERR_DEVICE_BOUNDS, ERR_SITE_ATTN | (13u << 8));
          }
        }
      }
      cp_async_commit();
      if (j >= 1) {
        cp_async_wait<1>();
        fence_proxy_async_smem();
        mbar_arrive(&kv_full[(j - 1) % kStages]);
      }
    }
    cp_async_wait<0>();
    if (ok && nchunks > 0) {
      fence_proxy_async_smem();
      mbar_arrive(&kv_full[(nchunks - 1) % kStages]);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      constexpr uint32_t idesc_qk = make_idesc(kFmtBF16, kFmtBF16, 0, 0, 128, kN);
      constexpr uint32_t idesc_pv = make_idesc(kFmtBF16, kFmtBF16, 0, 1, 128, C::DVH);
      const int qk0 = C::qk_lo(rank);
      const int nks = C::ks_of(rank);
      const uint32_t kv_base = smem_u32(sKV), p_base = smem_u32(sP);
      auto do_pv = [&](int i) -> bool {
        if (!mbar_wait(&p_full[i & 1], (i >> 1) & 1, p.wait_ns, ab)) { fail(2); return false; }
        tc_fence_after();
        const int st = i % kStages;
        const uint64_t pdesc = make_sdesc(p_base + (i & 1) * C::P_BYTES, 16, 1024, kSwizzle128);
        const uint32_t vbase = kv_base + st * C::STAGE_BYTES + (C::v_lo(rank) / 64 - atom_lo) * C::ATOM_BYTES;
#pragma unroll
        for (int ks = 0; ks < kN / 16; ++ks) {
          const uint64_t vdesc = make_sdesc(vbase + ks * 16 * 128, C::ATOM_BYTES, 1024, kSwizzle128);
          mma_bf16(tmem + kOCol, pdesc + 2 * ks, vdesc, idesc_pv, (i > 0 || ks > 0) ? 1u : 0u);
        }
        mma_commit(&pv_done[i & 1]);
        mma_commit(&kv_empty[st]);
        return true;
      };
      bool ok = mbar_wait(q_ready, 0, p.wait_ns, ab);
      if (!ok) fail(3);
      tc_fence_after();
      for (int j = 0; j < nchunks && ok; ++j) {
        const int st = j % kStages;
        prog[1] = j;
        if (!mbar_wait(&kv_full[st], (j / kStages) & 1, p.wait_ns, ab)) { fail(4); ok = false; break; }
        fence_proxy_async_smem();
        if (j >= 1 && !mbar_wait(&s_free[0], (j - 1) & 1, p.wait_ns, ab)) { fail(5); ok = false; break; }
        tc_fence_after();
        const uint32_t sbase = kv_base + st * C::STAGE_BYTES;
        for (int ks = 0; ks < nks; ++ks) {
          const int d = qk0 + ks * 16;
          const uint32_t a_loc = (uint32_t)(d / 64 - atom_lo);
          const uint64_t bdesc = make_sdesc(sbase + a_loc * C::ATOM_BYTES + (d % 64) * 2, 16, 1024, kSwizzle128);
          mma_bf16_ts(tmem + kSCol, tmem + kQCol + ks * 8, bdesc, idesc_qk, ks > 0 ? 1u : 0u);
        }
        mma_commit(&s_full[0]);
        if (j >= 1 && !do_pv(j - 1)) { ok = false; break; }
      }
      if (ok && nchunks > 0) do_pv(nchunks - 1);
      mma_commit(mma_done);
      mbar_wait(mma_done, 0, p.wait_ns, no_abort);
    }
  } else {
    // ------------------------------------------------------------ softmax + output
    const int quarter = warp & 3;
    const int h = quarter * 32 + lane;              // head row == TMEM lane
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
    // Q half -> TMEM (A operand of Q.K^T): two bf16 per 32-bit column
    {
      const int d0 = C::qk_lo(rank), d1 = C::qk_hi(rank);
      const uint4* qsrc = reinterpret_cast<const uint4*>(p.q + ((size_t)row * p.H + h) * DK + d0);
      for (int g = 0; g < (d1 - d0) / 16; ++g) {
        uint4 a = make_uint4(0, 0, 0, 0), c = make_uint4(0, 0, 0, 0);
        if (h < p.H) {
          a = qsrc[2 * g];
          c = qsrc[2 * g + 1];
        }
        const uint32_t w[8] = {a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w};
        __syncwarp();
        tmem_st8(tmem + lane_addr + kQCol + g * 8, w);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(q_ready);
    }
    const uint32_t xpeer = map_to_rank(sX, peer);
    const uint32_t xfull_peer = map_to_rank(x_full, peer);
    const uint32_t pfree_peer = map_to_rank(peer_free, peer);
    const int hs = h & 15;
    // every lane polls; the warp proceeds only if all lanes saw the phase
    auto wwait = [&](uint64_t* bar, uint32_t parity, bool cluster) -> bool {
      const bool r = cluster ? mbar_wait_cluster(bar, parity, p.wait_ns, ab)
                             : mbar_wait(bar, parity, p.wait_ns, ab);
      return __all_sync(0xffffffffu, r);
    };
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nchunks && ok; ++j) {
      const int bsel = j & 1;
      if (threadIdx.x == kSoftWarp0 * 32) prog[2] = j;
      // 1. partial logits of this CTA
      if (!wwait(&s_full[0], j & 1, false)) { fail(6); ok = false; break; }
      tc_fence_after();
      uint32_t sr[2][32];
      tmem_ld32(tmem + lane_addr + kSCol, sr[0]);
      tmem_ld32(tmem + lane_addr + kSCol + 32, sr[1]);
      tmem_wait_ld_dep(sr[0]);
      tmem_wait_ld_dep(sr[1]);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[0]);
      // 2. send them to the peer
      if (j >= 2 && !wwait(&peer_free[bsel], ((j - 2) >> 1) & 1, true)) {
        fail(7); ok = false; break;
      }
      const uint32_t xrow = xpeer + (uint32_t)(bsel * C::X_BYTES + h * kN * 4);
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const int v = (c < 8) ? 0 : 1;
        const int e = (c & 7) * 4;
        st_cluster_v4(xrow + (uint32_t)((c ^ hs) * 16), __uint_as_float(sr[v][e]), __uint_as_float(sr[v][e + 1]),
                      __uint_as_float(sr[v][e + 2]), __uint_as_float(sr[v][e + 3]));
      }
      mbar_arrive_remote(xfull_peer + bsel * 8);  // release: the stores above are visible first
      // 3. add the peer's partial logits
      if (!wwait(&x_full[bsel], (j >> 1) & 1, true)) { fail(8); ok = false; break; }
      float s[kN];
      const float4* xr = reinterpret_cast<const float4*>(sX + bsel * (C::X_BYTES / 4) + h * kN);
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const float4 x = xr[c ^ hs];
        const int v = (c < 8) ? 0 : 1;
        const int e = (c & 7) * 4;
        s[4 * c + 0] = __uint_as_float(sr[v][e + 0]) + x.x;
        s[4 * c + 1] = __uint_as_float(sr[v][e + 1]) + x.y;
        s[4 * c + 2] = __uint_as_float(sr[v][e + 2]) + x.z;
        s[4 * c + 3] = __uint_as_float(sr[v][e + 3]) + x.w;
      }
      if (j + 2 < nchunks) mbar_arrive_remote(pfree_peer + bsel * 8);
      // 4. mask the empty slots, update the running maximum
      const int st = j % kStages;
      if (!wwait(&kv_full[st], (j / kStages) & 1, false)) { fail(9); ok = false; break; }
      const uint4* meta = reinterpret_cast<const uint4*>(sMeta + st * kN);
      float mc = -INFINITY;
#pragma unroll
      for (int c = 0; c < kN / 16; ++c) {
        const uint4 mv = meta[c];
        const uint32_t words[4] = {mv.x, mv.y, mv.z, mv.w};
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const bool valid = (words[q >> 2] >> ((q & 3) * 8)) & 0xffu;
          float& x = s[c * 16 + q];
          x = valid ? x * p.scale_log2 : -INFINITY;
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
      // 5. probabilities (bf16) into the P buffer; row sum in FP32
      if (j >= 2 && !wwait(&pv_done[bsel], ((j - 2) >> 1) & 1, false)) { fail(10); ok = false; break; }
      float rs = 0.f;
      uint8_t* prow = sP + bsel * C::P_BYTES + h * 128;
      const bool any = m_used != -INFINITY;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
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
        *reinterpret_cast<uint4*>(prow + ((c ^ (h & 7)) << 4)) = pk;
      }
      l = l * alpha + rs;
      // 6. rescale the output accumulator when the maximum moved (warp-wide)
      if (__any_sync(0xffffffffu, rescale)) {
        if (j >= 1 && !wwait(&pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, false)) {
          fail(11); ok = false; break;
        }
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
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[bsel]);
    }
    // 7. output
    if (ok && nchunks > 0 && !wwait(&pv_done[(nchunks - 1) & 1], ((nchunks - 1) >> 1) & 1, false)) {
      fail(12);
      ok = false;
    }
    if (ok && nchunks > 0) {
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const float lse2 = l > 0.f ? m_used + log2f(l) : -INFINITY;
      const bool write_o = h < p.H && (C::SPLIT_V || rank == 0);
      const int vlo = C::v_lo(rank);
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
      if (rank == 0 && h < p.H) {
        if (p.nsplit == 1) {
          if (p.lse != nullptr) p.lse[(size_t)row * p.H + h] = lse2 * 0.6931471805599453f;
        } else {
          p.part_lse[((size_t)row * p.nsplit + split) * p.H + h] = lse2;
        }
      }
    } else if (ok && h < p.H && row_ok) {
      // no selected slots in this split: empty result
      if (p.nsplit > 1 && rank == 0) p.part_lse[((size_t)row * p.nsplit + split) * p.H + h] = -INFINITY;
    }
  }

  tc_fence_before();
  cluster_sync_all();  // the peer may still write into this CTA's shared memory until here
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
  p.q = a.q;
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
  cudaError_t e = cudaFuncSetAttribute(sparse_attn_tc_kernel<DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       Cf::ALLOC);
  if (e != cudaSuccess) return e;
  const long long ctas = 2 * rows * a.nsplit;
  sparse_attn_tc_kernel<DK, DV><<<(unsigned)ctas, kThreads, Cf::ALLOC, c.stream>>>(p);
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
