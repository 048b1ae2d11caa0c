// Step B: per-query top-k over the visible part of a score row.
//
// Keep the min(k, n) best of the n = pos(t) + 1 visible scores, ties to the
// lower index (ouchyi thread, "Nasil calisiyor" paragraph: only the top-k
// key/value entries are kept, 2,048 per query; tenelement.pl, section
// "Architektura ...", "Selekcja top-k" bullet).  The selection stays on the
// device and reads the row straight from the score tile (sider.ai blog,
// "Uyarilar": candidate selection must not bounce between CPU and GPU and
// must be cache-aware).
//
// Keys: scores mapped to order-preserving 32-bit unsigned keys (-0.0 folded
// onto +0.0).  One block of 1024 threads per row first tries a single pass:
// a radix select over a strided sample of the row gives a lower bound on the
// k-th key, one pass collects every key at or above it into shared memory,
// and step 3 below selects among them.  When the bound admits fewer than k
// keys or more than shared memory holds, the two-pass method runs:
//   1. one pass over the row builds a 2048-bin histogram of the top 11 key
//      bits; a block scan finds the bin B holding the k-th largest key;
//   2. a second pass (the row is now in L2) writes every key above bin B to
//      the output and copies the keys of bin B, with their indices, into
//      shared memory;
//   3. radix select over those candidates (11-bit digits) finds the exact
//      k-th key `thr`; one block scan places the candidates above it, and of
//      the candidates equal to it the lowest indices are kept (a second radix
//      select on the bitwise complement of the index picks them when they do
//      not all fit).
// If bin B holds more candidates than shared memory takes, steps 2-3 run as
// radix passes over the row itself and a final pass in index order.
// Decode rows (few, long) are split over several blocks for steps 1-2: each
// block of a row writes the histogram of its segment into the caller's
// workspace, then each block sums the row's segment histograms, finds bin B
// and, over its own segment, writes the keys above B to the output and
// appends bin B's keys to a per-row candidate list in the workspace (a block
// scan of the per-thread counts, then one global atomic per list and block);
// the row's last block to finish runs step 3 on that list.
#include <type_traits>

#include "internal.h"
#include "sm100.cuh"

namespace dsa {
namespace {

using sm100::pdl_launch_dependents;
using sm100::pdl_wait;

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kBins = 2048;           // top 11 bits
constexpr int kBinShift = 21;
constexpr int kCap = 8192;            // candidates held in shared memory
constexpr int kSegBlocks = 16;        // blocks per row in the split (decode) path
// Split-path workspace per row, in 32-bit words: histogram | counters (keys
// written, candidates) | candidate keys | candidate indices.
constexpr int kWsHist = 0;                     // kSegBlocks segment histograms of kBins words
constexpr int kWsCtr = kSegBlocks * kBins;     // written, candidates, segments done, (spare)
constexpr int kWsKeys = kWsCtr + 4;
constexpr int kWsIdx = kWsKeys + kCap;
constexpr int kWsRowWords = kWsIdx + kCap;

// Block-wide inclusive scan of one value per thread; returns the inclusive
// prefix and writes the block total to *total.
__device__ __forceinline__ unsigned int block_scan(unsigned int v, unsigned int* warp_tot, unsigned int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  if (warp == 0) {
    unsigned int w = warp_tot[lane];
    unsigned int s = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    warp_tot[lane] = s - w;  // exclusive prefix of the warps
    if (lane == 31) *total = s;
  }
  __syncthreads();
  const unsigned int r = x + warp_tot[warp];
  __syncthreads();
  return r;
}

// Find the bin holding the rank-th largest key (rank >= 1) among bins
// counted in hist[0..nb) (nb a power of two up to kBins; larger bin = larger
// keys).
// Returns the bin in *bin and the count of keys in higher bins in *above.
__device__ void find_bin(const unsigned int* hist, int nb, unsigned int rank, unsigned int* warp_tot,
                         unsigned int* s_bin, unsigned int* s_above, unsigned int* s_total) {
  const int per = nb / kThreads > 0 ? nb / kThreads : 1;  // 2 for kBins, 1 for 256
  unsigned int local = 0;
  unsigned int c[2] = {0u, 0u};
  const int t = threadIdx.x;
  // thread t owns bins nb-1-per*t ... (descending)
  if (t * per < nb) {
    for (int i = 0; i < per; ++i) {
      c[i] = hist[nb - 1 - (per * t + i)];
      local += c[i];
    }
  }
  const unsigned int incl = block_scan(local, warp_tot, s_total);
  const unsigned int excl = incl - local;
  if (t * per < nb && excl < rank && incl >= rank) {
    unsigned int run = excl;
    for (int i = 0; i < per; ++i) {
      if (run + c[i] >= rank) {
        *s_bin = (unsigned int)(nb - 1 - (per * t + i));
        *s_above = run;
        break;
      }
      run += c[i];
    }
  }
  __syncthreads();
}

// Radix select over `count` keys delivered by key_of(i) that all share the bits
// in `mask` with `prefix`: finds the rank-th largest key (rank >= 1), refining
// 11 bits at a time (the kBins histogram) from bit `hi` down to bit 0.
// Returns the key; *krem gets how many keys equal to it belong to the top
// `rank`.
template <class KeyOf>
__device__ unsigned int radix_select(KeyOf key_of, int count, unsigned int prefix, unsigned int mask, int hi,
                                     unsigned int rank, unsigned int* hist, unsigned int* warp_tot,
                                     unsigned int* s_bin, unsigned int* s_above, unsigned int* s_total,
                                     unsigned int* krem_out) {
  constexpr int kDigit = 11;                  // kBins = 2^11
  unsigned int krem = rank;
  while (hi > 0) {
    const int bits = hi >= kDigit ? kDigit : hi;
    const int shift = hi - bits;
    const unsigned int dmask = (1u << bits) - 1u;
    const int nb = 1 << bits;
    for (int x = threadIdx.x; x < nb; x += kThreads) hist[x] = 0u;
    __syncthreads();
    for (int i = threadIdx.x; i < count; i += kThreads) {
      const unsigned int key = key_of(i);
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & dmask], 1u);
    }
    __syncthreads();
    find_bin(hist, nb, krem, warp_tot, s_bin, s_above, s_total);
    prefix |= *s_bin << shift;
    mask |= dmask << shift;
    krem -= *s_above;
    hi = shift;
    __syncthreads();
  }
  *krem_out = krem;
  return prefix;
}

struct Smem {
  unsigned int hist[kBins];
  unsigned int ck[kCap];  // candidate keys
  int ci[kCap];           // candidate indices
  int eqi[kCap];          // indices of the candidates equal to the k-th key
  unsigned int warp_tot[kWarps];
  unsigned int bin, above, total, krem2;
  int cnt, ncand, eq_base;
  int warp_eq[kWarps];
};

// Steps 2-3 on a row whose threshold bin B (and the count above it) is known.
// keys_in_bin: number of keys in bin B over the whole row.
// Self-check on every output slot: a position outside [0, k) is recorded as
// DSA_ERR_DEVICE_BOUNDS (detail names the write site) and skipped.
__device__ __forceinline__ void put(int32_t* out, int k, int pos, int value, DevErr* err, unsigned site) {
  if (pos >= 0 && pos < k) {
    out[pos] = value;
  } else {
    report_error(err, DSA_ERR_DEVICE_BOUNDS, ERR_SITE_TOPK | (site << 8));
  }
}

// Exact selection among nc candidate keys held in shared memory (sm.ck,
// sm.ci), all sharing the bits `mask` with `prefix` (bits below `hi` free):
// emit the `need` largest, ties to the lower index, after the sm.cnt slots
// already written.
__device__ void select_candidates(int nc, unsigned int prefix, unsigned int mask, int hi, unsigned int need, int k,
                                  int32_t* out, Smem& sm, DevErr* err) {
  const int tid = threadIdx.x;
  const unsigned int* ck = sm.ck;
  unsigned int krem;
  const unsigned int thr = radix_select([ck](int i) { return ck[i]; }, nc, prefix, mask, hi, need, sm.hist,
                                        sm.warp_tot, &sm.bin, &sm.above, &sm.total, &krem);
  // One block scan of (above thr, equal to thr) counts places every output:
  // the keys above thr first, then, when all of them fit, the equal ones.
  // Both counts fit 16 bits (at most kCap candidates).
  const unsigned int base = (unsigned int)sm.cnt;
  unsigned int gt = 0, eq = 0;
  for (int i = tid; i < nc; i += kThreads) {
    const unsigned int key = sm.ck[i];
    gt += key > thr ? 1u : 0u;
    eq += key == thr ? 1u : 0u;
  }
  const unsigned int packed = gt | (eq << 16);
  const unsigned int excl = block_scan(packed, sm.warp_tot, &sm.total) - packed;
  const unsigned int G = sm.total & 0xFFFFu, E = sm.total >> 16;
  const bool all_eq = E == krem;
  unsigned int pg = base + (excl & 0xFFFFu), pe = base + G + (excl >> 16);
  for (int i = tid; i < nc; i += kThreads) {
    const unsigned int key = sm.ck[i];
    if (key > thr) put(out, k, (int)pg++, sm.ci[i], err, 2);
    else if (all_eq && key == thr) put(out, k, (int)pe++, sm.ci[i], err, 3);
  }
  if (all_eq) return;
  // more equal keys than slots: keep the lowest indices.  Gather the equal
  // candidates' indices and select on ~index (lower index = larger key).
  if (tid == 0) {
    sm.cnt = (int)(base + G);
    sm.eq_base = 0;
  }
  __syncthreads();
  for (int i = tid; i < nc; i += kThreads)
    if (sm.ck[i] == thr) {
      const int p = atomicAdd(&sm.eq_base, 1);
      if (p < kCap) sm.eqi[p] = sm.ci[i];
    }
  __syncthreads();
  const int ne = min(sm.eq_base, kCap);
  const int* ci = sm.eqi;
  unsigned int krem2;
  const unsigned int ithr = radix_select([ci](int i) { return ~(unsigned int)ci[i]; }, ne, 0u, 0u, 32, krem, sm.hist,
                                         sm.warp_tot, &sm.bin, &sm.above, &sm.total, &krem2);
  for (int i = tid; i < ne; i += kThreads)
    if (~(unsigned int)sm.eqi[i] >= ithr) put(out, k, atomicAdd(&sm.cnt, 1), sm.eqi[i], err, 4);
}

__device__ void select_from_bin(const float* row, int n, int k, int32_t* out, unsigned int B, unsigned int above,
                                unsigned int keys_in_bin, Smem& sm, DevErr* err) {
  const int tid = threadIdx.x;
  if (B >= (unsigned)kBins || above >= (unsigned)k) {  // threshold bin must exist
    if (tid == 0) report_error(err, DSA_ERR_DEVICE_BOUNDS, ERR_SITE_TOPK | (9u << 8));
    return;
  }
  const unsigned int need = (unsigned int)k - above;  // keys to take from bin B (>= 1)
  if (tid == 0) {
    sm.cnt = 0;
    sm.ncand = 0;
  }
  __syncthreads();
  const bool fits = keys_in_bin <= (unsigned int)kCap;
  // pass 2: keys above bin B go straight out; bin B keys become candidates
  auto visit = [&](float f, int x) {
    const unsigned int key = order_key(f);
    const unsigned int bin = key >> kBinShift;
    if (bin > B) {
      put(out, k, atomicAdd(&sm.cnt, 1), x, err, 1);
    } else if (bin == B && fits) {
      const int p = atomicAdd(&sm.ncand, 1);
      if (p < kCap) {
        sm.ck[p] = key;
        sm.ci[p] = x;
      } else {
        report_error(err, DSA_ERR_DEVICE_BOUNDS, ERR_SITE_TOPK | (7u << 8));
      }
    }
  };
  {
    // 16-byte loads over the aligned body (rows start 16-byte aligned), two
    // in flight per thread; scalar tail
    const int n4 = n / 4;
    const float4* r4 = reinterpret_cast<const float4*>(row);
    int x = tid;
    for (; x + kThreads < n4; x += 2 * kThreads) {
      float4 v[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) v[u] = r4[x + u * kThreads];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int e = 4 * (x + u * kThreads);
        visit(v[u].x, e);
        visit(v[u].y, e + 1);
        visit(v[u].z, e + 2);
        visit(v[u].w, e + 3);
      }
    }
    for (; x < n4; x += kThreads) {
      const float4 v = r4[x];
      visit(v.x, 4 * x);
      visit(v.y, 4 * x + 1);
      visit(v.z, 4 * x + 2);
      visit(v.w, 4 * x + 3);
    }
    for (int e = 4 * n4 + tid; e < n; e += kThreads) visit(row[e], e);
  }
  __syncthreads();
  unsigned int thr, krem;
  if (fits) {
    select_candidates(min(sm.ncand, kCap), B << kBinShift, 0xFFFFFFFFu << kBinShift, kBinShift, need, k, out, sm, err);
    return;
  }
  // bin B too large for shared memory: radix passes over the row itself
  thr = radix_select([row](int i) { return order_key(row[i]); }, n, B << kBinShift, 0xFFFFFFFFu << kBinShift,
                     kBinShift, need, sm.hist, sm.warp_tot, &sm.bin, &sm.above, &sm.total, &krem);
  // keys in bin B above thr, then the krem lowest-indexed keys equal to thr
  if (tid == 0) sm.eq_base = 0;
  __syncthreads();
  const int lane = tid & 31, warp = tid >> 5;
  for (int base = 0; base < n; base += kThreads) {
    const int x = base + tid;
    const bool valid = x < n;
    const unsigned int key = valid ? order_key(row[x]) : 0u;
    if (valid && (key >> kBinShift) == B && key > thr) put(out, k, atomicAdd(&sm.cnt, 1), x, err, 5);
    const bool eq = valid && key == thr;
    const unsigned int bal = __ballot_sync(0xffffffffu, eq);
    if (lane == 0) sm.warp_eq[warp] = __popc(bal);
    __syncthreads();
    int before = sm.eq_base;
    for (int w = 0; w < warp; ++w) before += sm.warp_eq[w];
    before += __popc(bal & ((1u << lane) - 1u));
    if (eq && before < (int)krem) put(out, k, atomicAdd(&sm.cnt, 1), x, err, 6);
    __syncthreads();
    if (tid == 0) {
      int tot = 0;
      for (int w = 0; w < kWarps; ++w) tot += sm.warp_eq[w];
      sm.eq_base += tot;
    }
    __syncthreads();
  }
}

// Row r of the launch: sequence b, query t, n = pos(t) + 1 visible keys.
__device__ __forceinline__ void row_setup(const TopkArgs& a, int r, DevErr* err, int* b, int* t, int* n,
                                          const float** row, int32_t** out) {
  *b = r / a.q_count;
  const int i = r - *b * a.q_count;
  *t = a.q_begin + i;
  *n = a.kv.len(*b, err, ERR_SITE_TOPK) - a.T + *t + 1;
  *row = a.scores + (size_t)r * a.ld;
  *out = a.idx + ((size_t)*b * a.T + *t) * a.k;
}

__device__ void histogram_pass(const float* row, int lo, int hi, unsigned int* hist) {
  // vectorised over the 16-byte aligned middle of [lo, hi)
  const int a0 = (lo + 3) & ~3, a1 = hi & ~3;
  if (a0 >= a1) {
    for (int x = lo + (int)threadIdx.x; x < hi; x += kThreads) atomicAdd(&hist[order_key(row[x]) >> kBinShift], 1u);
    return;
  }
  for (int x = lo + (int)threadIdx.x; x < a0; x += kThreads) atomicAdd(&hist[order_key(row[x]) >> kBinShift], 1u);
  const float4* r4 = reinterpret_cast<const float4*>(row + a0);
  const int n4 = (a1 - a0) / 4;
  int x = threadIdx.x;
  // four independent 16-byte loads in flight per thread
  for (; x + 3 * kThreads < n4; x += 4 * kThreads) {
    float4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = r4[x + u * kThreads];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      atomicAdd(&hist[order_key(v[u].x) >> kBinShift], 1u);
      atomicAdd(&hist[order_key(v[u].y) >> kBinShift], 1u);
      atomicAdd(&hist[order_key(v[u].z) >> kBinShift], 1u);
      atomicAdd(&hist[order_key(v[u].w) >> kBinShift], 1u);
    }
  }
  for (; x < n4; x += kThreads) {
    const float4 v = r4[x];
    atomicAdd(&hist[order_key(v.x) >> kBinShift], 1u);
    atomicAdd(&hist[order_key(v.y) >> kBinShift], 1u);
    atomicAdd(&hist[order_key(v.z) >> kBinShift], 1u);
    atomicAdd(&hist[order_key(v.w) >> kBinShift], 1u);
  }
  for (int x = a1 + (int)threadIdx.x; x < hi; x += kThreads) atomicAdd(&hist[order_key(row[x]) >> kBinShift], 1u);
}

// One pass over the row when a lower bound on the k-th key is known: every
// key at or above `lo` becomes a candidate.  Rows of at most kCap keys take
// all keys; longer rows estimate the bound from a sample of at most
// kSampleBlocks groups of four adjacent keys, one out of every 64 x step keys:
// the bound has about 1.5 k / (16 step) + 16 sampled keys above it, so about
// 1.5 k + 256 step keys of the row are expected above it (3.3 k at 32K keys,
// 4.1 k at 128K; k is short of it with negligible probability).  Returns false
// (nothing written) when the candidates are fewer than k or do not fit in
// shared memory; the caller then runs the two-pass histogram path.
constexpr int kSampleBlocks = 512;
__device__ bool single_pass(const float* row, int n, int k, int32_t* out, Smem& sm, DevErr* err) {
  const int tid = threadIdx.x;
  const float4* r4 = reinterpret_cast<const float4*>(row);
  // The collection pass reads the row in rounds of 2 x kThreads 16-byte
  // loads; thread 0 keeps an L2 bulk prefetch kPfAhead rounds ahead of them,
  // starting before the sample, so that the row streams from HBM while the
  // block has only two loads per thread of its own in flight.
  constexpr int kRound4 = 2 * kThreads;
  constexpr int kPfAhead = 2;
  const int n4 = n / 4;
  auto prefetch_round = [&](int j) {
    const int a = j * kRound4;
    if (a < n4) sm100::prefetch_l2_bulk(r4 + a, (uint32_t)(min(n4 - a, kRound4) * 16));
  };
  if (tid == 0 && n > kCap)
    for (int j = 0; j < kPfAhead; ++j) prefetch_round(j);
  unsigned int lo = 0u;
  if (n > kCap) {
    const int nblk = n / 64;                         // 64-key blocks (>= 128 here)
    const int step = (nblk + kSampleBlocks - 1) / kSampleBlocks;
    const int ns = nblk / step;                      // sampled blocks, <= kSampleBlocks
    const int m = 4 * ns;
    const int rs = min(m, (3 * k) / (2 * 16 * step) + 16);
    for (int i = tid; i < ns; i += kThreads) {
      const float4 v = r4[(size_t)i * step * 16];
      sm.ck[4 * i] = order_key(v.x);
      sm.ck[4 * i + 1] = order_key(v.y);
      sm.ck[4 * i + 2] = order_key(v.z);
      sm.ck[4 * i + 3] = order_key(v.w);
    }
    __syncthreads();
    // The bound only has to lie at or below the rs-th sampled key: two 11-bit
    // digits of the keys' top 22 bits fix it to within 2^10 units of the
    // order key, which adds a negligible number of candidates.
    const unsigned int* ck = sm.ck;
    unsigned int krem;
    lo = radix_select([ck](int i) { return ck[i] >> 10; }, m, 0u, 0u, 22, (unsigned int)rs, sm.hist, sm.warp_tot,
                      &sm.bin, &sm.above, &sm.total, &krem)
         << 10;
  }
  if (tid == 0) {
    sm.cnt = 0;
    sm.ncand = 0;
  }
  __syncthreads();
  // Candidate test order_key(f) >= lo.  Above the key of +0.0 (a positive
  // bound, the usual case) it is a signed compare of the raw bits with
  // lo & 0x7FFFFFFF, one instruction per key: negative floats, -0.0 and
  // negative NaNs fail it and positive NaNs pass it, as with the keys.  The
  // key itself is formed only for the candidates.
  auto collect = [&](auto raw_tag) {
    constexpr bool kRaw = decltype(raw_tag)::value;
    const int rlo = (int)(lo & 0x7FFFFFFFu);
    auto visit = [&](float f, int x) {
      const bool hit = kRaw ? __float_as_int(f) >= rlo : order_key(f) >= lo;
      if (hit) {
        const int p = atomicAdd(&sm.ncand, 1);
        if (p < kCap) {
          sm.ck[p] = order_key(f);
          sm.ci[p] = x;
        }
      }
    };
    int x = tid;
    for (; x + kThreads < n4; x += 2 * kThreads) {
      if (tid == 0) prefetch_round(x / kRound4 + kPfAhead);
      float4 v[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) v[u] = r4[x + u * kThreads];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int e = 4 * (x + u * kThreads);
        visit(v[u].x, e);
        visit(v[u].y, e + 1);
        visit(v[u].z, e + 2);
        visit(v[u].w, e + 3);
      }
    }
    for (; x < n4; x += kThreads) {
      const float4 v = r4[x];
      visit(v.x, 4 * x);
      visit(v.y, 4 * x + 1);
      visit(v.z, 4 * x + 2);
      visit(v.w, 4 * x + 3);
    }
    for (int e = 4 * n4 + tid; e < n; e += kThreads) visit(row[e], e);
  };
  if (lo > 0x80000000u)
    collect(std::true_type{});
  else
    collect(std::false_type{});
  __syncthreads();
  const int nc = sm.ncand;
  if (nc < k || nc > kCap) return false;
  select_candidates(nc, 0u, 0u, 32, (unsigned int)k, k, out, sm, err);
  return true;
}

// The whole selection of one row held in memory (n > k visible scores).
__device__ void select_row(const float* row, int n, int k, int32_t* out, Smem& sm, DevErr* err) {
  if (single_pass(row, n, k, out, sm, err)) return;
  // two passes: histogram of the top 11 bits, then the threshold bin
  __syncthreads();
  for (int x = threadIdx.x; x < kBins; x += kThreads) sm.hist[x] = 0u;
  if (threadIdx.x == 0) sm.bin = 0xFFFFFFFFu;
  __syncthreads();
  histogram_pass(row, 0, n, sm.hist);
  __syncthreads();
  find_bin(sm.hist, kBins, (unsigned int)k, sm.warp_tot, &sm.bin, &sm.above, &sm.total);
  const unsigned int B = sm.bin, above = sm.above;
  const unsigned int inbin = B < (unsigned)kBins ? sm.hist[B] : 0u;
  __syncthreads();
  select_from_bin(row, n, k, out, B, above, inbin, sm, err);
}

// One block per row.
__global__ void __launch_bounds__(kThreads, 2) topk_row_kernel(TopkArgs a, DevErr* err) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw);
  int b, t, n;
  const float* row;
  int32_t* out;
  row_setup(a, blockIdx.x, err, &b, &t, &n, &row, &out);
  const int k = a.k;
  if (n <= k) {
    for (int x = threadIdx.x; x < k; x += kThreads) out[x] = x < n ? x : -1;
    return;
  }
  select_row(row, n, k, out, sm, err);
}

// ---------------------------------------------------------------- selection without a score tile
// The indexer first scores a strided sample of the keys (column j = key
// j * kstride) into a small tile; per row, the rank-rs sample score is a
// threshold at or above which about `target` keys of the whole row are
// expected.  The indexer then scores every key and appends the (order key,
// index) pairs at or above the row's threshold to the row's candidate list
// (at most cap slots), and one block per row selects among them exactly:
// every key at or above the threshold is a candidate, so with at least k
// candidates and no overflow the row's top k are among them.  Rows whose
// candidates fall short or overflow are listed for repair: the indexer scores
// just those rows into a small tile and select_row finishes them.

// Threshold per row, its candidate count and overflow flag cleared, its
// repair slot unset (block 0 also clears the repair count).
__global__ void __launch_bounds__(kThreads, 2)
    topk_threshold_kernel(TopkArgs a, const float* sample, long long ld_s, int kstride, int target, int cap,
                          unsigned int* thr, unsigned int* cnt, int* row_slot, int* row_fail, unsigned int* nfail,
                          unsigned int* wl_cnt, int nwl, DevErr* err) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw);
  const int r = blockIdx.x;
  int b, t, n;
  const float* row;
  int32_t* out;
  row_setup(a, r, err, &b, &t, &n, &row, &out);
  if (threadIdx.x == 0) {
    cnt[r] = 0u;
    row_slot[r] = -1;
    row_fail[r] = 0;
    if (r == 0) *nfail = 0u;
  }
  // warp lists the indexer's grid may leave unwritten read as empty
  if (r == 0)
    for (int i = threadIdx.x; i < nwl; i += kThreads) wl_cnt[i] = 0u;
  if (n <= cap) {  // the candidate list holds every visible key
    if (threadIdx.x == 0) thr[r] = 0u;
    return;
  }
  const int ns = (n - 1) / kstride + 1;          // visible sample keys
  long long rs = ((long long)target * ns + n - 1) / n;
  if (rs < 1) rs = 1;
  if (rs > ns) rs = ns;
  const float* srow = sample + (size_t)r * ld_s;
  unsigned int krem, key;
  if (ns <= kCap) {
    for (int i = threadIdx.x; i < ns; i += kThreads) sm.ck[i] = order_key(srow[i]);
    __syncthreads();
    const unsigned int* ck = sm.ck;
    key = radix_select([ck](int i) { return ck[i]; }, ns, 0u, 0u, 32, (unsigned int)rs, sm.hist, sm.warp_tot,
                       &sm.bin, &sm.above, &sm.total, &krem);
  } else {
    key = radix_select([srow](int i) { return order_key(srow[i]); }, ns, 0u, 0u, 32, (unsigned int)rs, sm.hist,
                       sm.warp_tot, &sm.bin, &sm.above, &sm.total, &krem);
  }
  if (threadIdx.x == 0) thr[r] = key;
}

// Exact selection among a row's candidates; a row that cannot be finished
// from them is listed for repair (and gets the best selection its candidates
// allow in the meantime).
__global__ void __launch_bounds__(kThreads, 2)
    topk_cand_select_kernel(TopkArgs a, const unsigned int* cand_key, const int32_t* cand_idx,
                            const unsigned int* cnt, int cap, const int* row_fail, int* row_slot, int* fail_rows,
                            unsigned int* nfail, int max_fail, DevErr* err) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw);
  const int r = blockIdx.x;
  int b, t, n;
  const float* row;
  int32_t* out;
  row_setup(a, r, err, &b, &t, &n, &row, &out);
  const int k = a.k;
  if (n <= k) {
    for (int x = threadIdx.x; x < k; x += kThreads) out[x] = x < n ? x : -1;
    return;
  }
  const unsigned int c = cnt[r];
  const bool complete =
      c >= (unsigned int)k && c <= (unsigned int)cap && c <= (unsigned int)kCap && row_fail[r] == 0;
  const int nc = (int)min(c, (unsigned int)min(cap, kCap));
  for (int i = threadIdx.x; i < nc; i += kThreads) {
    sm.ck[i] = cand_key[(size_t)r * cap + i];
    sm.ci[i] = cand_idx[(size_t)r * cap + i];
  }
  if (threadIdx.x == 0) sm.cnt = 0;
  __syncthreads();
  const int keep = min(nc, k);
  if (keep > 0) select_candidates(nc, 0u, 0u, 32, (unsigned int)keep, k, out, sm, err);
  __syncthreads();
  for (int x = keep + threadIdx.x; x < k; x += kThreads) out[x] = -1;
  if (!complete && threadIdx.x == 0) {
    const unsigned int slot = atomicAdd(nfail, 1u);
    if (slot < (unsigned int)max_fail) {
      fail_rows[slot] = r;
      row_slot[r] = (int)slot;
    } else {
      report_error(err, DSA_ERR_DEVICE_BOUNDS, ERR_SITE_TOPK | (0x40u << 8));
    }
  }
}

// The epilogue warps' candidate lists into per-row lists: one block per
// warp list.  The indexer appends 32 consecutive keys of one query at a time,
// so neighbouring entries mostly share a row: the lanes of a warp holding the
// same row reserve their slots with one returning atomic (the lowest such
// lane adds the group's size), latency hidden by the many blocks in flight.
__global__ void __launch_bounds__(256)
    topk_scatter_kernel(const int32_t* wl_row, const int32_t* wl_idx, const unsigned int* wl_key,
                        const unsigned int* wl_cnt, long long wl_cap, unsigned int* cnt, unsigned int* cand_key,
                        int32_t* cand_idx, int cap) {
  const long long base = (long long)blockIdx.x * wl_cap;
  const long long n = min((long long)wl_cnt[blockIdx.x], wl_cap);
  const int lane = threadIdx.x & 31;
  // every thread runs the same number of rounds (whole warps take part in
  // the match); lanes past the end hold row -1 and take no slot
  for (long long i0 = 0; i0 < n; i0 += 256) {
    const long long i = i0 + threadIdx.x;
    const bool valid = i < n;
    const int r = valid ? wl_row[base + i] : -1;
    const unsigned int same = __match_any_sync(0xffffffffu, r);
    const int leader = __ffs(same) - 1;
    unsigned int first = 0u;
    if (valid && lane == leader) first = atomicAdd(&cnt[r], (unsigned int)__popc(same));
    first = __shfl_sync(0xffffffffu, first, leader);
    if (valid) {
      const unsigned int pos = first + (unsigned int)__popc(same & ((1u << lane) - 1u));
      if (pos < (unsigned int)cap) {
        cand_key[(size_t)r * cap + pos] = wl_key[base + i];
        cand_idx[(size_t)r * cap + pos] = wl_idx[base + i];
      }
    }
  }
}

// Repair: rows listed by topk_cand_select_kernel, scored in full into
// tile[slot] by the indexer, selected as topk_row_kernel would.
__global__ void __launch_bounds__(kThreads, 2)
    topk_repair_kernel(TopkArgs a, const float* tile, long long ld, const int* fail_rows, const unsigned int* nfail,
                       int max_fail, DevErr* err) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw);
  const int slot = blockIdx.x;
  if ((unsigned int)slot >= min(*nfail, (unsigned int)max_fail)) return;
  const int r = fail_rows[slot];
  int b, t, n;
  const float* row;
  int32_t* out;
  row_setup(a, r, err, &b, &t, &n, &row, &out);
  if (n <= a.k) return;  // never listed
  select_row(tile + (size_t)slot * ld, n, a.k, out, sm, err);
}

// ---------------------------------------------------------------- split path
// The allocation-free form (dsa_topk_static): a histogram array of kBins
// words per row, cleared by topk_zero_kernel; topk_seg_hist_kernel adds each
// segment's histogram, topk_seg_select_kernel (one block per row) finds the
// bin and runs steps 2-3.

__global__ void __launch_bounds__(kThreads, 1) topk_seg_hist_kernel(TopkArgs a, unsigned int* ghist, int hstride, DevErr* err) {
  __shared__ unsigned int hist[kBins];
  pdl_launch_dependents();
  pdl_wait();
  const int r = blockIdx.x / kSegBlocks, seg = blockIdx.x - r * kSegBlocks;
  int b, t, n;
  const float* row;
  int32_t* out;
  row_setup(a, r, err, &b, &t, &n, &row, &out);
  if (n <= a.k) return;
  for (int x = threadIdx.x; x < kBins; x += kThreads) hist[x] = 0u;
  __syncthreads();
  const int per = ((n + kSegBlocks - 1) / kSegBlocks + 3) & ~3;
  const int lo = seg * per, hi = min(n, lo + per);
  if (lo < hi) histogram_pass(row, lo, hi, hist);
  __syncthreads();
  unsigned int* gh = ghist + (size_t)r * hstride;
  for (int x = threadIdx.x; x < kBins; x += kThreads)
    if (hist[x]) atomicAdd(&gh[x], hist[x]);
}

// Split path (few long rows, as in decode), two launches:
//  1. topk_seg_hist2_kernel: each of kSegBlocks blocks of a row writes the
//     histogram of its segment into the row's slot for it (plain stores, so
//     nothing needs clearing first); segment 0 also clears the row's counters;
//  2. topk_seg_collect_final_kernel: every block sums the row's segment
//     histograms, finds the threshold bin B, writes its segment's keys above
//     B and appends bin B's keys to the row's candidates; the last block of
//     the row to finish (an atomic count, no waiting) then selects the rest
//     from the candidates.

__global__ void __launch_bounds__(kThreads, 1) topk_seg_hist2_kernel(TopkArgs a, unsigned int* ws, DevErr* err) {
  __shared__ unsigned int hist[kBins];
  pdl_launch_dependents();
  pdl_wait();
  const int r = blockIdx.x / kSegBlocks, seg = blockIdx.x - r * kSegBlocks;
  int b, t, n;
  const float* row;
  int32_t* out;
  row_setup(a, r, err, &b, &t, &n, &row, &out);
  if (n <= a.k) return;
  for (int x = threadIdx.x; x < kBins; x += kThreads) hist[x] = 0u;
  __syncthreads();
  const int per = ((n + kSegBlocks - 1) / kSegBlocks + 3) & ~3;
  const int lo = seg * per, hi = min(n, lo + per);
  if (lo < hi) histogram_pass(row, lo, hi, hist);
  __syncthreads();
  unsigned int* w = ws + (size_t)r * kWsRowWords;
  for (int x = threadIdx.x; x < kBins; x += kThreads) w[kWsHist + seg * kBins + x] = hist[x];
  if (seg == 0 && threadIdx.x < 4) w[kWsCtr + threadIdx.x] = 0u;
}

__global__ void __launch_bounds__(kThreads, 1) topk_seg_collect_final_kernel(TopkArgs a, unsigned int* ws,
                                                                            DevErr* err) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw);
  // the decode attention may start its prologue now
  pdl_launch_dependents();
  pdl_wait();
  unsigned int* hist = sm.hist;
  unsigned int* warp_tot = sm.warp_tot;
  const int r = blockIdx.x / kSegBlocks, seg = blockIdx.x - r * kSegBlocks;
  int b, t, n;
  const float* row;
  int32_t* out;
  row_setup(a, r, err, &b, &t, &n, &row, &out);
  const int k = a.k;
  if (n <= k) {
    if (seg == 0)
      for (int x = threadIdx.x; x < k; x += kThreads) out[x] = x < n ? x : -1;
    return;
  }
  unsigned int* w = ws + (size_t)r * kWsRowWords;
  // the row's histogram: the sum of its segments' (all loads in flight)
  for (int x = threadIdx.x; x < kBins; x += kThreads) {
    unsigned int v[kSegBlocks];
#pragma unroll
    for (int sg = 0; sg < kSegBlocks; ++sg) v[sg] = w[kWsHist + sg * kBins + x];
    unsigned int sum = 0u;
#pragma unroll
    for (int sg = 0; sg < kSegBlocks; ++sg) sum += v[sg];
    hist[x] = sum;
  }
  if (threadIdx.x == 0) sm.bin = 0xFFFFFFFFu;
  __syncthreads();
  find_bin(hist, kBins, (unsigned int)k, warp_tot, &sm.bin, &sm.above, &sm.total);
  const unsigned int B = sm.bin, above = sm.above;
  unsigned int* cnt = w + kWsCtr;
  unsigned int* ncand = w + kWsCtr + 1;
  unsigned int* ck = w + kWsKeys;
  int* ci = reinterpret_cast<int*>(w + kWsIdx);
  const int per = ((n + kSegBlocks - 1) / kSegBlocks + 3) & ~3;
  const int lo = seg * per, hi = min(n, lo + per);
  __shared__ unsigned int s_base_out, s_base_cand, s_last;
  if (B < (unsigned)kBins && lo < hi) {
    // Rounds of eight keys per thread (two 16-byte loads), the same number for
    // every thread: each round counts its hits per thread, one block scan gives
    // every thread its offsets, and one global atomic per list reserves the
    // block's range.
    const float4* r4 = reinterpret_cast<const float4*>(row);
    const int n4lo = lo / 4, n4hi = hi / 4;  // lo is a multiple of 4
    const int tail = hi - 4 * n4hi;          // fewer than 4 keys after the last 16-byte load
    const int rounds = (n4hi - n4lo + 2 * kThreads - 1) / (2 * kThreads) + (tail > 0 ? 1 : 0);
    for (int rd = 0; rd < rounds; ++rd) {
      float f[8];
      int x[8];
      bool ok[8];
      const int base = n4lo + rd * 2 * kThreads;
      if (base < n4hi) {
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int i4 = base + u * kThreads + (int)threadIdx.x;
          const bool v = i4 < n4hi;
          const float4 q = v ? r4[i4] : make_float4(0.f, 0.f, 0.f, 0.f);
          f[4 * u] = q.x; f[4 * u + 1] = q.y; f[4 * u + 2] = q.z; f[4 * u + 3] = q.w;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            x[4 * u + e] = 4 * i4 + e;
            ok[4 * u + e] = v;
          }
        }
      } else {  // the last round takes the tail keys, one per thread
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          ok[e] = e == 0 && (int)threadIdx.x < tail;
          x[e] = 4 * n4hi + (int)threadIdx.x;
          f[e] = ok[e] ? row[x[e]] : 0.f;
        }
      }
      unsigned int up = 0, cb = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const unsigned int bin = order_key(f[e]) >> kBinShift;
        up += (ok[e] && bin > B) ? 1u : 0u;
        cb += (ok[e] && bin == B) ? 1u : 0u;
      }
      // both counts fit 16 bits: at most 8 per thread and 8192 per block
      const unsigned int packed = up | (cb << 16);
      const unsigned int incl = block_scan(packed, warp_tot, &sm.total);
      const unsigned int excl = incl - packed;
      if (threadIdx.x == 0) {
        const unsigned int tot = sm.total;
        s_base_out = (tot & 0xFFFFu) ? atomicAdd(cnt, tot & 0xFFFFu) : 0u;
        s_base_cand = (tot >> 16) ? atomicAdd(ncand, tot >> 16) : 0u;
      }
      __syncthreads();
      unsigned int po = s_base_out + (excl & 0xFFFFu), pc = s_base_cand + (excl >> 16);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const unsigned int key = order_key(f[e]);
        const unsigned int bin = key >> kBinShift;
        if (ok[e] && bin > B) put(out, k, (int)po++, x[e], err, 10);
        if (ok[e] && bin == B) {
          if (pc < (unsigned)kCap) {
            ck[pc] = key;
            ci[pc] = x[e];
          }
          ++pc;
        }
      }
      __syncthreads();  // s_base_* are rewritten by the next round
    }
  }
  // the last block of the row to get here finishes the row
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = atomicAdd(&w[kWsCtr + 2], 1u) == (unsigned int)(kSegBlocks - 1) ? 1u : 0u;
  __syncthreads();
  if (s_last == 0u) return;
  __threadfence();
  const unsigned int inbin = B < (unsigned)kBins ? hist[B] : 0u;
  const unsigned int written = atomicAdd(cnt, 0u), nc = atomicAdd(ncand, 0u);
  __syncthreads();
  if (B >= (unsigned)kBins || written != above || nc != inbin || nc > (unsigned)kCap) {
    // (the first two cannot happen with a consistent histogram; the passes
    // over the row rewrite every slot from the start)
    select_from_bin(row, n, k, out, B, above, inbin, sm, err);
    return;
  }
  for (int i = threadIdx.x; i < (int)nc; i += kThreads) {
    sm.ck[i] = ck[i];
    sm.ci[i] = ci[i];
  }
  if (threadIdx.x == 0) sm.cnt = (int)above;
  __syncthreads();
  select_candidates((int)nc, B << kBinShift, 0xFFFFFFFFu << kBinShift, kBinShift, (unsigned int)k - above, k, out,
                    sm, err);
}

__global__ void __launch_bounds__(kThreads, 2) topk_seg_select_kernel(TopkArgs a, unsigned int* ghist, DevErr* err) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw);
  int b, t, n;
  const float* row;
  int32_t* out;
  row_setup(a, blockIdx.x, err, &b, &t, &n, &row, &out);
  const int k = a.k;
  if (n <= k) {
    for (int x = threadIdx.x; x < k; x += kThreads) out[x] = x < n ? x : -1;
    return;
  }
  unsigned int* gh = ghist + (size_t)blockIdx.x * kBins;
  for (int x = threadIdx.x; x < kBins; x += kThreads) sm.hist[x] = gh[x];
  if (threadIdx.x == 0) sm.bin = 0xFFFFFFFFu;
  __syncthreads();
  find_bin(sm.hist, kBins, (unsigned int)k, sm.warp_tot, &sm.bin, &sm.above, &sm.total);
  const unsigned int B = sm.bin, above = sm.above;
  const unsigned int inbin = B < (unsigned)kBins ? sm.hist[B] : 0u;
  __syncthreads();
  select_from_bin(row, n, k, out, B, above, inbin, sm, err);
}

// Merge of candidate lists (key-split rows): row r's candidates are
// nparts lists of k (score, global index) pairs, index -1 = empty.  Keeps the
// k best by (score descending, index ascending) -- the top-k of the whole row
// when each list is the top-k of a disjoint key range -- as global indices,
// and, with idx_local set, the same selection as indices local to the key
// range [local_begin, local_begin + local_count) (-1 outside it).
__global__ void __launch_bounds__(kThreads, 1)
    topk_merge_kernel(const float* cand_scores, const int32_t* cand_idx, int rows, int nparts, int k, int32_t* idx,
                      int local_begin, int local_count, int32_t* idx_local, DevErr* err) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw);
  const int r = blockIdx.x;
  int32_t* out = idx + (size_t)r * k;
  if (threadIdx.x == 0) {
    sm.ncand = 0;
    sm.cnt = 0;
  }
  __syncthreads();
  for (int x = threadIdx.x; x < nparts * k; x += kThreads) {
    const int part = x / k, j = x - part * k;
    const size_t o = ((size_t)part * rows + r) * k + j;
    const int gi = cand_idx[o];
    if (gi >= 0) {
      const int q = atomicAdd(&sm.ncand, 1);
      if (q < kCap) {
        sm.ck[q] = order_key(cand_scores[o]);
        sm.ci[q] = gi;
      }
    }
  }
  __syncthreads();
  const int nc = min(sm.ncand, kCap);
  const int keep = min(nc, k);
  if (keep > 0) select_candidates(nc, 0u, 0u, 32, (unsigned int)keep, k, out, sm, err);
  __syncthreads();
  for (int x = keep + threadIdx.x; x < k; x += kThreads) out[x] = -1;
  if (idx_local != nullptr) {
    __syncthreads();
    for (int x = threadIdx.x; x < k; x += kThreads) {
      const int g = out[x];
      idx_local[(size_t)r * k + x] = (g >= local_begin && g - local_begin < local_count) ? g - local_begin : -1;
    }
  }
}

// Rows that see at most k keys keep all of them: idx = 0..n-1, then -1.
// No score is read.
__global__ void topk_fill_kernel(TopkArgs a, DevErr* err) {
  int b, t, n;
  const float* row;
  int32_t* out;
  row_setup(a, blockIdx.x, err, &b, &t, &n, &row, &out);
  for (int x = threadIdx.x; x < a.k; x += blockDim.x) out[x] = x < n ? x : -1;
}

// Zero the first `words` words of each of `rows` rows of `stride` words.
// Launched as a programmatic dependent of the indexer, it clears the
// histograms while the scores are still being written, then waits for the
// indexer so that its own completion implies the scores' (the histogram
// kernel after it waits for this grid only).
__global__ void topk_zero_kernel(unsigned int* p, int rows, int stride, int words) {
  pdl_launch_dependents();
  const size_t n = (size_t)rows * words;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
    p[(i / words) * stride + i % words] = 0u;
  pdl_wait();
}

}  // namespace

size_t topk_workspace_bytes(int rows) { return (size_t)rows * kWsRowWords * sizeof(unsigned int); }

bool topk_uses_workspace(int rows, int S, int num_sms) { return rows * 2 < num_sms && S >= 16 * kThreads; }

cudaError_t launch_topk(const LaunchCtx& c, const TopkArgs& a, void* ws, size_t ws_bytes) {
  const int rows = a.B * a.q_count;
  if (rows <= 0) return cudaSuccess;
  const size_t smem = sizeof(Smem);
  cudaError_t e;
  if ((long long)a.S - a.T + a.q_begin + a.q_count <= a.k) {
    // every row sees at most k keys whatever its sequence's length
    topk_fill_kernel<<<rows, 256, 0, c.stream>>>(a, c.err);
    note_launches(1);
    return cudaGetLastError();
  }
  // few long rows: split the histogram pass over several blocks per row
  const bool split =
      ws != nullptr && ws_bytes >= topk_workspace_bytes(rows) && topk_uses_workspace(rows, a.S, c.num_sms);
  if (!split) {
    e = cudaFuncSetAttribute(topk_row_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    topk_row_kernel<<<rows, kThreads, smem, c.stream>>>(a, c.err);
    note_launches(1);
    return cudaGetLastError();
  }
  // two launches, each a programmatic dependent of the one before (the
  // first of the indexer's): each starts while its predecessor drains
  unsigned int* w = static_cast<unsigned int*>(ws);
  e = cudaFuncSetAttribute(topk_seg_collect_final_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  if ((e = launch_pdl(topk_seg_hist2_kernel, dim3(rows * kSegBlocks), dim3(kThreads), 0, c.stream, a, w, c.err)) !=
      cudaSuccess)
    return e;
  if ((e = launch_pdl(topk_seg_collect_final_kernel, dim3(rows * kSegBlocks), dim3(kThreads), smem, c.stream, a, w,
                      c.err)) != cudaSuccess)
    return e;
  note_launches(2);
  return cudaGetLastError();
}

}  // namespace dsa

namespace dsa {

cudaError_t launch_topk_merge(const LaunchCtx& c, const float* cand_scores, const int32_t* cand_idx, int rows,
                              int nparts, int k, int32_t* idx, int local_begin, int local_count,
                              int32_t* idx_local) {
  if (rows <= 0) return cudaSuccess;
  if ((long long)nparts * k > kCap) return cudaErrorInvalidValue;
  const size_t smem = sizeof(Smem);
  cudaError_t e = cudaFuncSetAttribute(topk_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  topk_merge_kernel<<<rows, kThreads, smem, c.stream>>>(cand_scores, cand_idx, rows, nparts, k, idx, local_begin,
                                                        local_count, idx_local, c.err);
  note_launches(1);
  return cudaGetLastError();
}

int topk_merge_max_candidates() { return kCap; }

int topk_cand_cap() { return kCap; }

cudaError_t launch_topk_threshold(const LaunchCtx& c, const TopkArgs& a, const float* sample, long long ld_s,
                                  int kstride, int target, int cap, unsigned int* thr, unsigned int* cnt, int* row_slot,
                                  int* row_fail, unsigned int* nfail, unsigned int* wl_cnt, int nwl) {
  const int rows = a.B * a.q_count;
  if (rows <= 0) return cudaSuccess;
  const size_t smem = sizeof(Smem);
  cudaError_t e = cudaFuncSetAttribute(topk_threshold_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  topk_threshold_kernel<<<rows, kThreads, smem, c.stream>>>(a, sample, ld_s, kstride, target, cap, thr, cnt, row_slot,
                                                            row_fail, nfail, wl_cnt, nwl, c.err);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_topk_scatter(const LaunchCtx& c, const int32_t* wl_row, const int32_t* wl_idx,
                                const unsigned int* wl_key, const unsigned int* wl_cnt, long long wl_cap, int nwarps,
                                unsigned int* cnt, unsigned int* cand_key, int32_t* cand_idx, int cap) {
  if (nwarps <= 0) return cudaSuccess;
  topk_scatter_kernel<<<nwarps, 256, 0, c.stream>>>(wl_row, wl_idx, wl_key, wl_cnt, wl_cap, cnt, cand_key, cand_idx,
                                                    cap);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_topk_cand_select(const LaunchCtx& c, const TopkArgs& a, const unsigned int* cand_key,
                                    const int32_t* cand_idx, const unsigned int* cnt, int cap, const int* row_fail,
                                    int* row_slot, int* fail_rows, unsigned int* nfail, int max_fail) {
  const int rows = a.B * a.q_count;
  if (rows <= 0) return cudaSuccess;
  const size_t smem = sizeof(Smem);
  cudaError_t e = cudaFuncSetAttribute(topk_cand_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  topk_cand_select_kernel<<<rows, kThreads, smem, c.stream>>>(a, cand_key, cand_idx, cnt, cap, row_fail, row_slot,
                                                              fail_rows, nfail, max_fail, c.err);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_topk_repair(const LaunchCtx& c, const TopkArgs& a, const float* tile, long long ld,
                               const int* fail_rows, const unsigned int* nfail, int max_fail) {
  const size_t smem = sizeof(Smem);
  cudaError_t e = cudaFuncSetAttribute(topk_repair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  topk_repair_kernel<<<max_fail, kThreads, smem, c.stream>>>(a, tile, ld, fail_rows, nfail, max_fail, c.err);
  note_launches(1);
  return cudaGetLastError();
}

// Split path with a caller-provided histogram array (B * q_count * 2048
// words): zero it, histogram each row over several blocks, select per row.
cudaError_t launch_topk_split_into(const LaunchCtx& c, const TopkArgs& a, unsigned int* hist) {
  const int rows = a.B * a.q_count;
  if (rows <= 0) return cudaSuccess;
  topk_zero_kernel<<<64, 256, 0, c.stream>>>(hist, rows, kBins, kBins);
  topk_seg_hist_kernel<<<rows * kSegBlocks, kThreads, 0, c.stream>>>(a, hist, kBins, c.err);
  const size_t smem = sizeof(Smem);
  cudaError_t e = cudaFuncSetAttribute(topk_seg_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  topk_seg_select_kernel<<<rows, kThreads, smem, c.stream>>>(a, hist, c.err);
  note_launches(3);
  return cudaGetLastError();
}

}  // namespace dsa
