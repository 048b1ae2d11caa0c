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
// Per CTA:
//   * TMEM: O (128 x 256 FP32) | two 64-column S buffers | the first 256
//     key dims of Q as BF16 pairs (128 columns) = 512 columns.  The other
//     320 dims of Q (80 KB) sit in shared memory, loaded once by TMA.  Q K^T
//     takes its A operand from TMEM for 16 of its 36 K steps;
//   * the rest of shared memory is a ring of four 32-key slots (1152 B per
//     key, 128B-swizzled K-major atoms laid out [atom][slot][row] so that the
//     two slots of a chunk form one 64-row tile).  Each MMA chunk is 64 keys
//     (N = 64): a tcgen05.mma costs the issuing thread about as much for
//     N = 32 as for N = 64, so larger N halves the issue time per key;
//   * six gather warps fill the ring with 16-byte cp.async, three per slot
//     of a chunk (one issuing warp moves only about 18 B/clk);
//   * eight softmax warps, two per TMEM lane quarter: each takes 32 of the
//     chunk's 64 logits, the two exchange their partial row maxima through
//     shared memory, and each writes its BF16 probabilities over part of the
//     chunk's S buffer; O += P V takes P from TMEM and V as the MN-major
//     view of the gathered rows.  With two S/P buffers the softmax of chunk
//     j+1 runs while P V of chunk j executes.
// Online softmax in base 2 with a lazy rescale: the running maximum moves
// only when a chunk exceeds it by more than 8 (so p <= 256), and then the
// TMEM accumulator is rescaled once (each softmax warp its half of the value
// columns), after the previous P V has landed.
//
// Warp roles (480 threads): warp 0 owns TMEM and issues the MMAs (whichever
// is ready: Q K^T of the next chunk or P V of the oldest), warps 1-3 and
// 12-14 gather, warps 4-11 run the softmax (thread = head row) and write the
// output.  Decode splits the selected keys of each query over several CTAs
// and merges the partial results with a combine kernel.  Every barrier that
// receives an asynchronous arrival is waited on before the CTA exits.
#include <cuda_bf16.h>

#include "internal.h"
#include "sm100.cuh"
#include "tma_host.h"

namespace dsa {
namespace {

using namespace sm100;

constexpr int kSlotKeys = 32;   // keys per gather slot
constexpr int kN = 2 * kSlotKeys;  // keys per chunk = N of Q K^T (two adjacent slots)
constexpr int kSBuf = 2;        // S/P buffers in TMEM
// Warps: 0 MMA, 1-3 gather the even slot of every chunk, 4-11 softmax (two
// per TMEM lane quarter: warps 4-7 take keys 0-31 of a chunk, 8-11 keys
// 32-63), 12-14 gather the odd slot.  One issuing warp moves only about
// 18 B/clk of 16-byte cp.async; three per slot let both slots of a chunk land
// in parallel.
constexpr int kMmaWarp = 0, kFirstSoftmaxWarp = 4, kSoftmaxWarps = 8;
constexpr int kGatherPerSlot = 3;
constexpr int kFirstGatherB = kFirstSoftmaxWarp + kSoftmaxWarps;
constexpr int kThreads = 32 * (kFirstGatherB + kGatherPerSlot);
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.f;  // log2 units

// SEPV: values come from their own array (not the first DV columns of the
// key row); each slot then also holds this CTA's value atoms, and the ring
// shrinks to one chunk of two slots to make room.
template <int DK, int DV, bool SEPV = false>
struct Cfg {
  static constexpr int KSTEPS = DK / 16;             // 16-wide MMA K steps over the key dim
  static constexpr int NATOM = (DK + 63) / 64;       // 64-column (128-byte) atoms of a key row
  static constexpr int NHALF = DV >= 128 ? 2 : 1;    // value columns split over CTAs
  static constexpr int DVH = DV / NHALF;
  static constexpr int NVATOM = (DVH + 63) / 64;     // value atoms of this CTA's half
  static constexpr int ATOMS = NATOM + (SEPV ? NVATOM : 0);  // atoms gathered per key
  static constexpr int SLOTS = SEPV ? 2 : 4;         // gather ring slots
  static constexpr int NCH = SLOTS / 2;              // chunks held by the ring
  static constexpr int VATOM0 = SEPV ? NATOM : 0;    // first atom read as V (plus half * NVATOM when !SEPV)
  static constexpr uint32_t OCOL = 0;
  static constexpr uint32_t SCOL = (DVH + 31) / 32 * 32;
  static constexpr uint32_t QCOL = SCOL + kSBuf * kN;
  // leading key dims whose Q lives in TMEM (whole 64-wide atoms, or all of DK)
  static constexpr int QT_FIT = (int)(kTmemCols - QCOL) * 2 / 64 * 64;
  static constexpr int QT_DIMS = DK <= QT_FIT ? DK : QT_FIT;
  static constexpr int QT_STEPS = QT_DIMS / 16;
  static constexpr int QT_BLOCKS = (QT_DIMS + 63) / 64;  // 32-column stores per row
  static constexpr int QS_ATOMS = (DK - QT_DIMS) / 64;   // Q atoms in shared memory
  static constexpr int Q_ATOM = 128 * 128;               // 128 head rows x 128 bytes
  static constexpr int SLOT_ATOM = kSlotKeys * 128;
  static constexpr int ATOM_STRIDE = SLOTS * SLOT_ATOM;
  static constexpr int RING = ATOMS * ATOM_STRIDE;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = OFF_Q + QS_ATOMS * Q_ATOM;
  static constexpr int OFF_MASK = OFF_KV + RING;
  // partial row maxima exchanged by the two softmax warps of a lane quarter,
  // one set per S buffer: [kSBuf][2 sides][128 rows]
  static constexpr int OFF_XM = OFF_MASK + SLOTS * 4;
  static constexpr int OFF_BAR = OFF_XM + kSBuf * 2 * 128 * 4;
  static constexpr int NBARS = 2 + 2 * SLOTS + 3 * kSBuf + 1 + kSBuf * 4 + 4 + SLOTS;
  static constexpr int OFF_MISC = OFF_BAR + NBARS * 8;
  static constexpr int BYTES = OFF_MISC + 16;
  // the dynamic shared memory base is checked for 1024-byte alignment at run
  // time (the swizzled layouts need it), so no slack is allocated
  static constexpr int ALLOC = BYTES;
  static_assert(DK % 64 == 0 || QT_DIMS == DK, "Q split on whole atoms");
  static_assert(QT_DIMS % 16 == 0 && DVH <= 256 && DVH % 16 == 0, "shape");
  static_assert(QCOL + (QT_DIMS / 2 + 31) / 32 * 32 <= kTmemCols, "TMEM layout");
  static_assert(ALLOC <= 232448, "shared memory per CTA");
};

struct AttnParams {
  KvMap map;        // per-sequence lengths, paged or contiguous caches
  const uint16_t* q;
  const uint16_t* kv;
  const uint16_t* v;    // separate values (SEPV kernels only)
  const int32_t* idx;   // null: every row dense
  int dense_rows;       // rows with t < dense_rows take keys 0..pos(t), idx unread
  int kslots;           // slots per row (k; the longest visible run when dense)
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



// PAGED: the caches are page pools (block table lookup per gathered key);
// the contiguous form computes the row directly.
template <int DK, int DV, bool SEPV, bool PAGED>
__global__ void __launch_bounds__(kThreads, 1)
    sparse_attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, AttnParams p) {
  using C = Cfg<DK, DV, SEPV>;
  constexpr int kSlots = C::SLOTS;
  extern __shared__ uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023u) {
    // self-check: the layouts below need a 1024-byte aligned base
    if (threadIdx.x == 0) report_error(p.err, DSA_ERR_DEVICE_BOUNDS, ERR_SITE_ATTN | (0xAu << 8));
    return;
  }
  uint8_t* smem = smem_raw;
  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sKV = smem + C::OFF_KV;
  uint32_t* sMask = reinterpret_cast<uint32_t*>(smem + C::OFF_MASK);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* q_full = bars;                     // Q atoms in shared memory (TMA)
  uint64_t* q_ready = q_full + 1;              // Q rows in TMEM (4 softmax warps)
  uint64_t* kv_full = q_ready + 1;
  uint64_t* kv_empty = kv_full + kSlots;
  uint64_t* s_full = kv_empty + kSlots;
  uint64_t* p_full = s_full + kSBuf;           // [kSBuf] P written (4 softmax warps)
  uint64_t* pv_done = p_full + kSBuf;          // [kSBuf] P V of the buffer complete (MMA commit)
  uint64_t* mma_done = pv_done + kSBuf;
  uint64_t* mx_bar = mma_done + 1;             // [kSBuf][4 quarters] both partial maxima written
  uint64_t* lx_bar = mx_bar + kSBuf * 4;       // [4 quarters] both partial row sums written
  uint64_t* kv_kfree = lx_bar + 4;             // [kSlots] Q K^T of the slot's chunk done (MMA commit)
  float* sXM = reinterpret_cast<float*>(smem + C::OFF_XM);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int half = blockIdx.x % C::NHALF;
  const int rest = blockIdx.x / C::NHALF;
  const int row = rest / p.nsplit;  // b * T + t
  const int split = rest - row * p.nsplit;
  const int b = row / p.T;
  const int t = row - b * p.T;
  const int slot0 = split * p.kc;
  // self-check: a CTA outside the launch's rows does no work
  const bool row_ok = row >= 0 && row < p.rows && split >= 0 && split < p.nsplit && slot0 >= 0;
  const int Lb = row_ok ? p.map.len(b, p.err, ERR_SITE_ATTN) : 0;
  const int pos = Lb - p.T + t;                 // this query's position
  const bool dense = p.idx == nullptr || t < p.dense_rows;
  // dense rows read keys 0..pos in slot order (slot i holds key i)
  const int slot1 = min(dense ? pos + 1 : p.kslots, min(p.kslots, slot0 + p.kc));
  const int nchunks = row_ok && slot1 > slot0 ? (slot1 - slot0 + kN - 1) / kN : 0;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_ready, kSoftmaxWarps);
    for (int i = 0; i < kSlots; ++i) {
      mbar_init(&kv_full[i], 32 * kGatherPerSlot);
      mbar_init(&kv_empty[i], 1);
      mbar_init(&kv_kfree[i], 1);
    }
    for (int i = 0; i < kSBuf; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], kSoftmaxWarps);
      mbar_init(&pv_done[i], 1);
    }
    mbar_init(mma_done, 1);
    for (int i = 0; i < kSBuf * 4 + 4; ++i) mbar_init(&mx_bar[i], 2);
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
  // every lane polls; the warp proceeds only if all lanes saw the phase
  auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
    const bool r = mbar_wait(bar, parity, p.wait_ns, ab);
    return __all_sync(0xffffffffu, r);
  };

  if (warp != kMmaWarp && (warp < kFirstSoftmaxWarp || warp >= kFirstGatherB)) {
    // ------------------------------------------------------------ gather
    // slot half h of every chunk; warp g of the half copies atoms g, g+3, g+6
    const int h = warp < kFirstSoftmaxWarp ? 0 : 1;
    const int g = h == 0 ? warp - 1 : warp - kFirstGatherB;
    bool q_issued = false;
    if (h == 0 && g == 0 && lane == 0 && nchunks > 0 && C::QS_ATOMS > 0) {
      prefetch_tmap(&tm_q);
      mbar_arrive_expect_tx(q_full, C::QS_ATOMS * C::Q_ATOM);
      for (int a = 0; a < C::QS_ATOMS; ++a)
        tma_load_2d(sQ + a * C::Q_ATOM, &tm_q, q_full, C::QT_DIMS + a * 64, row * p.H);
      q_issued = true;
    }
    const int c16 = lane & 7, rg = lane >> 3;  // 16-byte column chunk, row group
    const int32_t* irow = dense ? nullptr : p.idx + (size_t)row * p.k;
    // in the paged form, the cache row of the sequence's key 0 (every
    // sequence has at least T keys), which empty slots copy (pool row 0 if
    // that page is unmapped); a contiguous cache copies row b * S
    long long row0 = PAGED && nchunks > 0 ? p.map.row<true>(b, 0) : 0;
    if (row0 < 0) row0 = 0;
    // indices of this half of chunk j, loaded one chunk ahead
    int ivn[kSlotKeys / 4];
    auto load_idx = [&](int j) {
#pragma unroll
      for (int m = 0; m < kSlotKeys / 4; ++m) {
        const int slot = slot0 + j * kN + h * kSlotKeys + rg + 4 * m;
        ivn[m] = (j < nchunks && slot < slot1) ? (dense ? slot : irow[slot]) : -1;
      }
    };
    load_idx(0);
    // The atoms of a key row that this CTA's P V reads (its value half, or
    // the separate value atoms) are refilled once P V of the slot's last
    // chunk is done; the others as soon as its Q K^T is, so most of the next
    // gather overlaps the softmax and P V before it.
    const int vlo = half * C::DVH / 64, vhi = ((half + 1) * C::DVH - 1) / 64;
    auto reads_v = [&](int a) { return !SEPV && a >= vlo && a <= vhi; };
    for (int j = 0; j < nchunks; ++j) {
      const int st = 2 * (j % C::NCH) + h;     // ring slot of this half of chunk j
      int iv[kSlotKeys / 4];
#pragma unroll
      for (int m = 0; m < kSlotKeys / 4; ++m) iv[m] = ivn[m];
      if (j >= C::NCH && !wwait(&kv_kfree[st], (uint32_t)((j / C::NCH) - 1) & 1)) { fail(1); break; }
      uint8_t* slotp = sKV + st * C::SLOT_ATOM;
      size_t crows[kSlotKeys / 4];
      uint32_t mask = 0;
#pragma unroll
      for (int m = 0; m < kSlotKeys / 4; ++m) {
        const int r = rg + 4 * m;
        int v = iv[m];
        if (v >= Lb) {
          if (c16 == 0) report_error(p.err, DSA_ERR_DEVICE_BOUNDS, ERR_SITE_ATTN);
          v = -1;
        }
        // cache row of key v: a page lookup in the paged form (an unmapped
        // page is reported and the slot emptied); the contiguous form keeps
        // the row arithmetic out of this loop
        long long cr = 0;
        if constexpr (PAGED) {
          cr = v >= 0 ? p.map.row<true>(b, v) : -1;
          if (v >= 0 && cr < 0) {
            if (c16 == 0) report_error(p.err, DSA_ERR_DEVICE_BOUNDS, ERR_SITE_ATTN | (1u << 8));
            v = -1;
          }
        }
        const bool valid = v >= 0;
        // lanes 0, 8, 16, 24 hold rows 4m .. 4m+3
        const uint32_t bal = __ballot_sync(0xffffffffu, valid);
        mask |= ((bal & 1u) | ((bal >> 7) & 2u) | ((bal >> 14) & 4u) | ((bal >> 21) & 8u)) << (4 * m);
        // an empty or invalid slot copies the sequence's first key row (a
        // finite row of the caller's cache), which then meets probability 0
        // in P V
        const size_t crow = PAGED ? (size_t)(valid ? cr : row0) : (size_t)b * p.S + (valid ? v : 0);
        crows[m] = crow;
        // phase 1: key atoms that P V does not read
        const uint16_t* src = p.kv + crow * DK;
#pragma unroll
        for (int a0 = 0; a0 < C::NATOM; a0 += kGatherPerSlot) {
          const int a = a0 + g;
          if (a < C::NATOM && a * 128 + c16 * 16 < DK * 2 && !reads_v(a))
            cp_async16(slotp + a * C::ATOM_STRIDE + r * 128 + ((c16 ^ (r & 7)) << 4), src + a * 64 + c16 * 8);
        }
      }
      // phase 2: the atoms P V reads, once P V of the slot's last chunk is done
      if (j >= C::NCH && !wwait(&kv_empty[st], (uint32_t)((j / C::NCH) - 1) & 1)) { fail(1); break; }
#pragma unroll
      for (int m = 0; m < kSlotKeys / 4; ++m) {
        const int r = rg + 4 * m;
        const size_t crow = crows[m];
        if constexpr (!SEPV) {
          const uint16_t* src = p.kv + crow * DK;
#pragma unroll
          for (int a0 = 0; a0 < C::NATOM; a0 += kGatherPerSlot) {
            const int a = a0 + g;
            if (a < C::NATOM && a * 128 + c16 * 16 < DK * 2 && reads_v(a))
              cp_async16(slotp + a * C::ATOM_STRIDE + r * 128 + ((c16 ^ (r & 7)) << 4), src + a * 64 + c16 * 8);
          }
        } else {
          // this CTA's value columns [half * DVH, (half + 1) * DVH) of the
          // value row, in atoms NATOM, NATOM + 1, ...
          const uint16_t* vsrc = p.v + crow * DV + half * C::DVH;
#pragma unroll
          for (int va0 = 0; va0 < C::NVATOM; va0 += kGatherPerSlot) {
            const int va = va0 + g;
            if (va < C::NVATOM && va * 64 + c16 * 8 < C::DVH)
              cp_async16(slotp + (C::NATOM + va) * C::ATOM_STRIDE + r * 128 + ((c16 ^ (r & 7)) << 4),
                         vsrc + va * 64 + c16 * 8);
          }
        }
      }
      if (g == 0 && lane == 0) sMask[st] = mask;
      cp_async_commit();
      load_idx(j + 1);
      cp_async_wait<0>();
      fence_proxy_async_smem();
      mbar_arrive(&kv_full[st]);
    }
    cp_async_wait<0>();
    // drain: the Q load must have landed before this CTA's memory is reused
    if (q_issued) mbar_wait(q_full, 0, p.wait_ns, no_abort);
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issue
    // chunk j uses S buffer j % 2 and ring slots 2 (j % NCH), 2 (j % NCH) + 1
    if (lane == 0) {
      constexpr uint32_t idesc_qk = make_idesc(kFmtBF16, kFmtBF16, 0, 0, 128, kN);
      constexpr uint32_t idesc_pv = make_idesc(kFmtBF16, kFmtBF16, 0, 1, 128, C::DVH);
      // descriptors are built once; a step only adds its byte offset >> 4 to
      // the start-address field (no carry: shared addresses are < 256 KB)
      const uint64_t kdesc0 = make_sdesc(smem_u32(sKV), 16, 1024, kSwizzle128);
      const uint64_t qdesc0 = make_sdesc(smem_u32(sQ), 16, 1024, kSwizzle128);
      const uint64_t vdesc0 = make_sdesc(
          smem_u32(sKV) + (uint32_t)(SEPV ? C::VATOM0 : half * C::DVH / 64) * C::ATOM_STRIDE, C::ATOM_STRIDE, 1024,
          kSwizzle128);
      bool ok = nchunks == 0 || ((C::QS_ATOMS == 0 || mbar_wait(q_full, 0, p.wait_ns, ab)) &&
                                 mbar_wait(q_ready, 0, p.wait_ns, ab));
      if (!ok) fail(3);
      // Issue whichever MMA is ready: Q K^T of chunk qk once its rows have
      // landed and P V of chunk qk - kSBuf has freed its S buffer; P V of
      // chunk pv once its probabilities are written.
      int qk = 0, pv = 0;
      // P V of chunk pv: 4 K steps of 16 keys, A = P (TMEM), B = V (MN-major);
      // its commits free the chunk's S buffer and both ring slots
      auto issue_pv = [&]() {
        tc_fence_after();
        const int s0 = (2 * pv) % kSlots, sb = pv % kSBuf;
        const uint64_t vst = vdesc0 + (uint64_t)((s0 * C::SLOT_ATOM) >> 4);
        if (!SEPV) {
#pragma unroll
          for (int ks = 0; ks < kN / 16; ++ks) {
            const uint64_t vdesc = vst + (uint64_t)((ks * 16 * 128) >> 4);
            mma_bf16_ts(tmem + C::OCOL, tmem + C::SCOL + sb * kN + ks * 8, vdesc, idesc_pv,
                        (pv > 0 || ks > 0) ? 1u : 0u);
          }
        } else {
          // values in their own atoms: one N = 64 MMA per 64-column atom
          constexpr uint32_t idesc_pv64 = make_idesc(kFmtBF16, kFmtBF16, 0, 1, 128, 64);
#pragma unroll
          for (int nb = 0; nb < C::NVATOM; ++nb)
#pragma unroll
            for (int ks = 0; ks < kN / 16; ++ks) {
              const uint64_t vdesc = vst + (uint64_t)((nb * C::ATOM_STRIDE + ks * 16 * 128) >> 4);
              mma_bf16_ts(tmem + C::OCOL + nb * 64, tmem + C::SCOL + sb * kN + ks * 8, vdesc, idesc_pv64,
                          (pv > 0 || ks > 0) ? 1u : 0u);
            }
        }
        mma_commit(&pv_done[sb]);
        mma_commit(&kv_empty[s0]);
        mma_commit(&kv_empty[s0 + 1]);
        ++pv;
      };
      uint64_t t_idle = 0;
      uint32_t spins = 0;
      while (ok && pv < nchunks) {
        bool progressed = false;
        if (qk < nchunks && qk < pv + kSBuf) {
          const int s0 = (2 * qk) % kSlots, sb = qk % kSBuf;
          const uint32_t par = (uint32_t)((2 * qk) / kSlots) & 1;
          if (mbar_test_wait(&kv_full[s0], par) && mbar_test_wait(&kv_full[s0 + 1], par) &&
              (qk < kSBuf || mbar_test_wait(&pv_done[sb], ((qk / kSBuf) - 1) & 1))) {
            fence_proxy_async_smem();
            tc_fence_after();
            const uint64_t kst = kdesc0 + (uint64_t)((s0 * C::SLOT_ATOM) >> 4);
            const uint32_t dS = tmem + C::SCOL + sb * kN;
#pragma unroll
            for (int ks = 0; ks < C::KSTEPS; ++ks) {
              const int d = ks * 16;
              const uint64_t bdesc = kst + (uint64_t)(((d / 64) * C::ATOM_STRIDE + (d % 64) * 2) >> 4);
              if (ks < C::QT_STEPS) {
                mma_bf16_ts(dS, tmem + C::QCOL + ks * 8, bdesc, idesc_qk, ks > 0 ? 1u : 0u);
              } else {
                const int dq = d - C::QT_DIMS;
                const uint64_t adesc = qdesc0 + (uint64_t)(((dq / 64) * C::Q_ATOM + (dq % 64) * 2) >> 4);
                mma_bf16(dS, adesc, bdesc, idesc_qk, ks > 0 ? 1u : 0u);
              }
            }
            mma_commit(&s_full[sb]);
            // the slots' atoms that P V does not read may be refilled now
            mma_commit(&kv_kfree[s0]);
            mma_commit(&kv_kfree[s0 + 1]);
            ++qk;
            progressed = true;
          }
        }
        if (pv < qk && mbar_test_wait(&p_full[pv % kSBuf], (pv / kSBuf) & 1)) {
          issue_pv();
          progressed = true;
        }
        if (progressed) {
          spins = 0;
          continue;
        }
        // nothing ready: doze briefly on the event most likely next, with
        // bounded idle time, and abort when another role failed
        if (pv < qk)
          mbar_try_wait_hint(&p_full[pv % kSBuf], (pv / kSBuf) & 1, 200);
        else
          mbar_try_wait_hint(&kv_full[(2 * qk) % kSlots], (uint32_t)((2 * qk) / kSlots) & 1, 200);
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
      // drain: the last arrivals of each commit barrier are not always waited
      // by their consumers; make sure they have landed before the CTA exits
      for (int c = max(0, 2 * pv - kSlots); c < 2 * pv; ++c)
        mbar_wait(&kv_empty[c % kSlots], (c / kSlots) & 1, p.wait_ns, no_abort);
      for (int c = max(0, 2 * qk - kSlots); c < 2 * qk; ++c)
        mbar_wait(&kv_kfree[c % kSlots], (c / kSlots) & 1, p.wait_ns, no_abort);
      for (int i = max(0, pv - kSBuf); i < pv; ++i)
        mbar_wait(&pv_done[i % kSBuf], (i / kSBuf) & 1, p.wait_ns, no_abort);
      for (int i = max(0, qk - kSBuf); i < qk; ++i)
        mbar_wait(&s_full[i % kSBuf], (i / kSBuf) & 1, p.wait_ns, no_abort);
    }
  } else {
    // ------------------------------------------------------------ softmax + output
    // two warps per TMEM lane quarter: side 0 takes keys 0-31 of every chunk
    // and value columns 0-127 of this CTA's half, side 1 keys 32-63 and value
    // columns 128-255; both derive the same running maximum from the
    // exchanged partial maxima
    const int side = (warp - kFirstSoftmaxWarp) >> 2;
    const int quarter = warp & 3;
    const int h = quarter * 32 + lane;              // head row == TMEM lane
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
    const bool head_ok = row_ok && h < p.H;
    constexpr int OHALF = C::DVH / 2;               // output columns per side
    // Q dims [0, QT_DIMS) of row h into TMEM as BF16 pairs (zeros past H);
    // side s writes the 64-dim blocks s, s + 2, ...
    {
      const uint16_t* qrow = p.q + ((size_t)(head_ok ? row : 0) * p.H + (head_ok ? h : 0)) * DK;
      for (int qb = side; qb < C::QT_BLOCKS; qb += 2) {
        uint32_t v[32];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int col = qb * 64 + i * 8;
          uint4 x = make_uint4(0u, 0u, 0u, 0u);
          if (head_ok && col < C::QT_DIMS) x = *reinterpret_cast<const uint4*>(qrow + col);
          v[4 * i] = x.x;
          v[4 * i + 1] = x.y;
          v[4 * i + 2] = x.z;
          v[4 * i + 3] = x.w;
        }
        tmem_st32(tmem + lane_addr + C::QCOL + qb * 32, v);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(q_ready);
    }
    const float sc = p.scale_log2;
    float m_used = -INFINITY, l = 0.f;              // l: this side's share of the row sum
    bool ok = true;
    for (int j = 0; j < nchunks && ok; ++j) {
      const int sb = j % kSBuf, s0 = (2 * j) % kSlots;
      const uint32_t kpar = (uint32_t)((2 * j) / kSlots) & 1;
      // 1. this side's 32 logits and valid keys
      if (!wwait(&s_full[sb], (j / kSBuf) & 1)) { fail(6); ok = false; break; }
      if (!wwait(&kv_full[s0 + side], kpar)) { fail(7); ok = false; break; }
      const uint32_t mask = sMask[s0 + side];
      tc_fence_after();
      const uint32_t saddr = tmem + lane_addr + C::SCOL + sb * kN;
      uint32_t sr[32];
      tmem_ld32(saddr + side * 32, sr);
      tmem_wait_ld_dep(sr);
      float pm = -INFINITY;
      if (mask == 0xffffffffu) {
#pragma unroll
        for (int q = 0; q < 32; ++q) pm = fmaxf(pm, __uint_as_float(sr[q]));
      } else {
#pragma unroll
        for (int q = 0; q < 32; ++q)
          if ((mask >> q) & 1u) pm = fmaxf(pm, __uint_as_float(sr[q]));
      }
      // 2. exchange the partial maxima with the other side of this quarter
      float* xm = sXM + sb * 256;
      xm[side * 128 + h] = pm;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&mx_bar[sb * 4 + quarter]);
      if (!wwait(&mx_bar[sb * 4 + quarter], (j / kSBuf) & 1)) { fail(10); ok = false; break; }
      tc_fence_after();  // the other side's logits are read before P overwrites them
      const float mraw = fmaxf(pm, xm[(side ^ 1) * 128 + h]);
      const float mc = mraw * sc;
      float alpha = 1.f;
      bool rescale = false;
      if (m_used == -INFINITY) {
        m_used = mc;
      } else if (mc > m_used + kRescaleThreshold) {
        alpha = exp2f(m_used - mc);
        m_used = mc;
        rescale = true;
      }
      // 3. rescale this side's output columns when the maximum moved, once
      //    the previous P V has landed
      if (__any_sync(0xffffffffu, rescale)) {
        if (j >= 1 && !wwait(&pv_done[(j - 1) % kSBuf], ((j - 1) / kSBuf) & 1)) { fail(8); ok = false; break; }
        tc_fence_after();
        for (int c = 0; c < OHALF / 32; ++c) {
          uint32_t o[32];
          const uint32_t oaddr = tmem + lane_addr + C::OCOL + side * OHALF + c * 32;
          tmem_ld32(oaddr, o);
          tmem_wait_ld_dep(o);
#pragma unroll
          for (int q = 0; q < 32; ++q) o[q] = __float_as_uint(__uint_as_float(o[q]) * alpha);
          tmem_st32(oaddr, o);
        }
        tmem_wait_st();
      }
      // 4. probabilities of this side's keys as BF16 pairs over P columns
      //    [16 side, 16 side + 16) of the S buffer (side 0's logits there
      //    were read before its maximum was published)
      float rs = 0.f;
      uint32_t pk[16];
      if (m_used == -INFINITY) {
#pragma unroll
        for (int q = 0; q < 16; ++q) pk[q] = 0u;
      } else {
        const float neg_m = -m_used;
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          float e0 = ex2_approx(fmaf(__uint_as_float(sr[2 * q]), sc, neg_m));
          float e1 = ex2_approx(fmaf(__uint_as_float(sr[2 * q + 1]), sc, neg_m));
          if (mask != 0xffffffffu) {
            if (!((mask >> (2 * q)) & 1u)) e0 = 0.f;
            if (!((mask >> (2 * q + 1)) & 1u)) e1 = 0.f;
          }
          rs += e0 + e1;
          pk[q] = pack_bf16x2(e0, e1);
        }
      }
      tmem_st16(saddr + side * 16, pk);
      tmem_wait_st();
      l = l * alpha + rs;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[sb]);
    }
    // 5. output: combine the two partial row sums, then each side writes its
    //    value columns
    if (ok && nchunks > 0) {
      float* xl = sXM + (nchunks % kSBuf) * 256;    // buffer of chunk nchunks - 2, no longer read
      xl[side * 128 + h] = l;
      __syncwarp();
      if (lane == 0) mbar_arrive(&lx_bar[quarter]);
      if (!wwait(&lx_bar[quarter], 0)) {
        fail(11);
        ok = false;
      } else {
        l += xl[(side ^ 1) * 128 + h];
      }
    }
    if (ok && nchunks > 0 && !wwait(&pv_done[(nchunks - 1) % kSBuf], ((nchunks - 1) / kSBuf) & 1)) {
      fail(9);
      ok = false;
    }
    if (ok && nchunks > 0) {
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const float lse2 = l > 0.f ? m_used + log2f(l) : -INFINITY;
      const int vlo = half * C::DVH + side * OHALF;
      for (int c = 0; c < OHALF / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_addr + C::OCOL + side * OHALF + c * 32, o);
        tmem_wait_ld_dep(o);
        if (!head_ok) continue;
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
      if (half == 0 && side == 0 && head_ok) {
        if (p.nsplit == 1) {
          if (p.lse != nullptr) p.lse[(size_t)row * p.H + h] = lse2 * 0.6931471805599453f;
        } else {
          p.part_lse[((size_t)row * p.nsplit + split) * p.H + h] = lse2;
        }
      }
    } else if (ok && head_ok && half == 0 && side == 0) {
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

template <int DK, int DV, bool SEPV, bool PAGED>
cudaError_t launch_tc(const LaunchCtx& c, const AttnArgs& a) {
  using Cf = Cfg<DK, DV, SEPV>;
  AttnParams p = {};
  p.map = a.map;
  p.q = a.q;
  p.kv = a.kv;
  p.v = a.v;
  p.idx = a.idx;
  p.dense_rows = a.dense_rows;
  p.kslots = a.idx != nullptr ? a.k : a.S;
  p.out = a.out;
  p.lse = a.lse;
  p.T = a.T;
  p.S = a.S;
  p.H = a.H;
  p.k = a.k;
  p.rows = a.B * a.T;
  p.nsplit = a.nsplit;
  p.kc = ((p.kslots + a.nsplit - 1) / a.nsplit + kN - 1) / kN * kN;
  p.scale_log2 = a.tau * 1.4426950408889634f;
  p.wait_ns = c.wait_ns;
  p.err = c.err;
  const long long rows = (long long)a.B * a.T;
  p.part_o = a.part;
  p.part_lse = a.part ? a.part + (size_t)rows * a.nsplit * a.H * DV : nullptr;
  // Q as a [rows * H, DK] BF16 matrix read in 128-row x 64-column boxes
  // (only the atoms kept in shared memory are loaded this way)
  CUtensorMap tm_q;
  if (!make_tmap_2d(&tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.q, (uint64_t)rows * a.H, DK, (uint64_t)DK * 2, 128,
                    64, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(sparse_attn_tc_kernel<DK, DV, SEPV, PAGED>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, Cf::ALLOC);
  if (e != cudaSuccess) return e;
  const long long ctas = rows * a.nsplit * Cf::NHALF;
  sparse_attn_tc_kernel<DK, DV, SEPV, PAGED><<<(unsigned)ctas, kThreads, Cf::ALLOC, c.stream>>>(tm_q, p);
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

int attn_choose_nsplit(int rows, int H, int d_v, int k, int num_sms) {
  (void)H;
  // one wave: rows x CTAs per query (value halves) x splits <= SM count
  // (one CTA per SM), at least one split, at most one chunk per split
  const int per_row = rows * (d_v >= 128 ? 2 : 1);
  const int chunks = (k + kN - 1) / kN;
  int target = per_row > 0 ? num_sms / per_row : 1;
  if (target < 1) target = 1;
  if (target > chunks) target = chunks;
  const int kc = ((k + target - 1) / target + kN - 1) / kN * kN;
  return (k + kc - 1) / kc;
}

cudaError_t launch_sparse_attn(const LaunchCtx& c, const AttnArgs& a) {
  if ((long long)a.B * a.T <= 0) return cudaSuccess;
  if (a.nsplit > 1 && a.part == nullptr) return cudaErrorInvalidValue;
  const bool sepv = a.v != nullptr, paged = a.map.page_size != 0;
  if (a.d_k == 576 && a.d_v == 512) {
    if (paged) return sepv ? launch_tc<576, 512, true, true>(c, a) : launch_tc<576, 512, false, true>(c, a);
    return sepv ? launch_tc<576, 512, true, false>(c, a) : launch_tc<576, 512, false, false>(c, a);
  }
  if (a.d_k == 80 && a.d_v == 64) {
    if (paged) return sepv ? launch_tc<80, 64, true, true>(c, a) : launch_tc<80, 64, false, true>(c, a);
    return sepv ? launch_tc<80, 64, true, false>(c, a) : launch_tc<80, 64, false, false>(c, a);
  }
  return cudaErrorInvalidValue;
}

}  // namespace dsa
