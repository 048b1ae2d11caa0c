// Host side of libdsa.so: argument checks, workspace layout, launch order.
// The arithmetic of every step lives in the kernel files; this file only
// validates, carves the caller's workspace and enqueues launches.
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "internal.h"

namespace dsa {

__device__ DevErr g_dsa_err;

static std::atomic<unsigned long long> g_launches{0};
void note_launches(int n) { g_launches.fetch_add((unsigned long long)n, std::memory_order_relaxed); }

namespace {

constexpr int kMaxDevices = 64;
constexpr long long kDefaultWaitNs = 2000000000LL;  // 2 s per bounded wait
long long g_wait_ns = kDefaultWaitNs;

struct DeviceInfo {
  DevErr* err = nullptr;
  int num_sms = 0;
  bool ready = false;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

dsa_status device_info(DeviceInfo* out, int* dev_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DSA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_dsa_err) != cudaSuccess) return DSA_ERR_CUDA;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return DSA_ERR_CUDA;
    d.err = static_cast<DevErr*>(p);
    d.num_sms = sms;
    d.ready = true;
  }
  *out = d;
  *dev_out = dev;
  return DSA_OK;
}

dsa_status make_ctx(void* stream, LaunchCtx* c) {
  DeviceInfo d;
  int dev = 0;
  dsa_status st = device_info(&d, &dev);
  if (st != DSA_OK) return st;
  c->stream = static_cast<cudaStream_t>(stream);
  c->err = d.err;
  c->wait_ns = g_wait_ns;
  c->num_sms = d.num_sms;
  c->device = dev;
  return DSA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool is_pow2_in(int v, int lo, int hi) { return v >= lo && v <= hi && (v & (v - 1)) == 0; }

// Basic validity of the shape (sizes positive, ranges supported).
dsa_status check_shape(const dsa_shape* s) {
  if (s == nullptr) return DSA_ERR_INVALID_ARG;
  if (s->B <= 0 || s->T <= 0 || s->S <= 0 || s->k <= 0 || s->H <= 0 || s->H_I <= 0 || s->D_I <= 0 ||
      s->d_k <= 0 || s->d_v <= 0)
    return DSA_ERR_INVALID_ARG;
  if (s->T > s->S) return DSA_ERR_INVALID_ARG;
  if (s->mode != DSA_PREFILL && s->mode != DSA_DECODE) return DSA_ERR_INVALID_ARG;
  if (s->D_I != 32 && s->D_I != 64 && s->D_I != 128) return DSA_ERR_UNSUPPORTED;
  if (!is_pow2_in(s->H_I, 4, 64)) return DSA_ERR_UNSUPPORTED;
  if (!((s->d_k == 576 && s->d_v == 512) || (s->d_k == 80 && s->d_v == 64))) return DSA_ERR_UNSUPPORTED;
  if (s->H > 128 || s->H % 8 != 0) return DSA_ERR_UNSUPPORTED;
  if (s->k > 2048) return DSA_ERR_UNSUPPORTED;
  if ((long long)s->S >= (1LL << 31) / 8) return DSA_ERR_UNSUPPORTED;
  if (s->page_size < 0) return DSA_ERR_INVALID_ARG;
  if (s->page_size > 0) {
    if (s->page_size % 16 != 0) return DSA_ERR_UNSUPPORTED;
    if (s->block_table == nullptr || s->num_pages <= 0 ||
        (long long)s->pages_per_seq * s->page_size < (long long)s->S)
      return DSA_ERR_INVALID_ARG;
    if ((long long)s->num_pages * s->page_size >= (1LL << 31) / 8) return DSA_ERR_UNSUPPORTED;
  }
  return DSA_OK;
}

// Where each sequence's keys are (lengths, paged or contiguous caches).
KvMap kv_map(const dsa_shape* s) {
  KvMap m;
  m.seqlens = s->seqlens;
  m.block_table = s->page_size > 0 ? s->block_table : nullptr;
  m.S = s->S;
  m.T = s->T;
  m.page_size = s->page_size > 0 ? s->page_size : 0;
  m.pages_per_seq = s->page_size > 0 ? s->pages_per_seq : 0;
  m.num_pages = s->page_size > 0 ? s->num_pages : 0;
  return m;
}

// Query rows t < dense_rows see at most k keys for every length up to S
// (pos(t) + 1 <= S - T + t + 1 <= k): their selection is all visible keys.
int dense_rows_of(const dsa_shape* s) {
  const long long d = (long long)s->k - ((long long)s->S - s->T);
  return d <= 0 ? 0 : (d >= s->T ? s->T : (int)d);
}

int q_block_of(const dsa_shape* s) {
  int qb = s->q_block > 0 ? s->q_block : 4096;
  return qb < s->T ? qb : s->T;
}

int64_t scores_ld(const dsa_shape* s) { return (int64_t)round_up((size_t)s->S, 64); }

float tau_of(const dsa_shape* s) {
  return s->softmax_scale > 0.f ? s->softmax_scale : 1.0f / sqrtf((float)s->d_k);
}

// Selection without a score tile: prefill over long contexts with a
// contiguous key cache (the sample reads every kSampleStride-th cache row).
constexpr int kSampleStride = 32;
constexpr int kRepairRows = 64;   // rows of one block that can fall back to a materialised score row
constexpr int kTargetNum = 3, kTargetDen = 2;   // about 1.5 k candidates expected per row
constexpr int kRowCap = 6144;     // candidates a row's list holds (<= the top-k's shared capacity)
constexpr int kWarpSlack = 2;     // warp lists hold twice the expected candidates

// The fused selection applies: prefill over a contiguous cache long enough
// for the key sample to leave few candidates per row.
bool fused_select_ok(const dsa_shape* s) {
  return s->mode == DSA_PREFILL && s->page_size == 0 && s->S % kSampleStride == 0 &&
         s->S >= 4 * topk_cand_cap();
}

// Workspace layout (each region 256-byte aligned):
//   [score tile, or the fused selection's regions][attention split partials]
//   [top-k histograms]
// The fused selection's regions, for R = B * q_rows rows: the key-sample
// tile [R, ld_s] FP32; thresholds, candidate counts, repair slots and
// overflow flags [R]; the indexer warps' candidate lists (row, index, key)
// [nwl, wl_cap] and their counts [nwl]; the per-row candidate keys and
// indices [R, cap]; the repair list and its count; the repair tile
// [kRepairRows, ld] FP32.
struct WsLayout {
  bool fused;
  size_t sample_off, thr_off, cnt_off, slot_off, rfail_off, wrow_off, widx_off, wkey_off, wcnt_off, ckey_off,
      cidx_off, fail_off, nfail_off, repair_off;
  int64_t ld_s;
  int cap, nwl;
  long long wl_cap;
  size_t scores_off, scores_bytes;
  size_t part_off, part_bytes;
  size_t topk_off, topk_bytes;
  size_t total;
  int nsplit, nsplit_dense;
  int q_rows;
};

// fused: the fused selection's regions in place of the score tile (only
// where fused_select_ok holds)
WsLayout ws_layout(const dsa_shape* s, int num_sms, bool fused) {
  WsLayout L;
  L.q_rows = s->mode == DSA_DECODE ? s->T : q_block_of(s);
  L.scores_off = 0;
  L.fused = fused && fused_select_ok(s);
  L.cap = kRowCap < topk_cand_cap() ? kRowCap : topk_cand_cap();
  L.ld_s = (int64_t)round_up((size_t)(s->S / kSampleStride), 64);
  if (L.fused) {
    const size_t R = (size_t)s->B * L.q_rows;
    // one list per indexer epilogue warp (a persistent grid of at most one
    // CTA per SM), together kWarpSlack times the expected candidates
    L.nwl = num_sms * indexer_epilogue_warps(s->H_I);
    const long long expect = (long long)R * s->k * kTargetNum / kTargetDen;
    L.wl_cap = (expect * kWarpSlack + L.nwl - 1) / L.nwl;
    const size_t W = (size_t)L.nwl * L.wl_cap;
    size_t o = 0;
    L.sample_off = o; o += round_up(R * L.ld_s * sizeof(float), 256);
    L.thr_off = o; o += round_up(R * 4, 256);
    L.cnt_off = o; o += round_up(R * 4, 256);
    L.slot_off = o; o += round_up(R * 4, 256);
    L.rfail_off = o; o += round_up(R * 4, 256);
    L.wrow_off = o; o += round_up(W * 4, 256);
    L.widx_off = o; o += round_up(W * 4, 256);
    L.wkey_off = o; o += round_up(W * 4, 256);
    L.wcnt_off = o; o += round_up((size_t)L.nwl * 4, 256);
    L.ckey_off = o; o += round_up(R * L.cap * 4, 256);
    L.cidx_off = o; o += round_up(R * L.cap * 4, 256);
    L.fail_off = o; o += round_up(kRepairRows * 4, 256);
    L.nfail_off = o; o += 256;
    L.repair_off = o; o += round_up((size_t)kRepairRows * scores_ld(s) * sizeof(float), 256);
    L.scores_bytes = o;
  } else {
    L.scores_bytes = round_up((size_t)s->B * L.q_rows * scores_ld(s) * sizeof(float), 256);
  }
  L.nsplit = s->mode == DSA_DECODE ? attn_choose_nsplit(s->B * s->T, s->H, s->d_v, s->k, num_sms) : 1;
  // dense attention (dsa_dense_attn) splits a decode row's S keys instead
  L.nsplit_dense = s->mode == DSA_DECODE ? attn_choose_nsplit(s->B * s->T, s->H, s->d_v, s->S, num_sms) : 1;
  L.part_off = L.scores_off + L.scores_bytes;
  size_t pb = attn_partial_floats(s->B * s->T, s->H, s->d_v, L.nsplit) * sizeof(float);
  const size_t pb_dense = attn_partial_floats(s->B * s->T, s->H, s->d_v, L.nsplit_dense) * sizeof(float);
  // the decode kernel's FP16 partials (MLA rows with the selection)
  const size_t pb_dec = s->mode == DSA_DECODE && s->d_k == 576 && s->d_v == 512
                            ? attn_decode_partial_bytes(s->B * s->T, s->H, attn_decode_nsplit(s->k))
                            : 0;
  if (pb_dense > pb) pb = pb_dense;
  if (pb_dec > pb) pb = pb_dec;
  L.part_bytes = round_up(pb, 256);
  L.topk_off = L.part_off + L.part_bytes;
  const int topk_rows = s->B * L.q_rows;
  L.topk_bytes = topk_uses_workspace(topk_rows, s->S, num_sms) ? round_up(topk_workspace_bytes(topk_rows), 256) : 0;
  L.total = L.topk_off + L.topk_bytes;
  return L;
}

// The layout a call given ws_bytes of workspace takes: the score tile when
// it fits, else the fused selection's regions when they fit, else the score
// tile's (which the caller then reports as too small).
WsLayout ws_choose(const dsa_shape* s, int num_sms, size_t ws_bytes) {
  WsLayout L = ws_layout(s, num_sms, false);
  if (ws_bytes >= L.total || !fused_select_ok(s)) return L;
  WsLayout F = ws_layout(s, num_sms, true);
  return ws_bytes >= F.total ? F : L;
}

dsa_status from_cuda(cudaError_t e) { return e == cudaSuccess ? DSA_OK : DSA_ERR_CUDA; }

dsa_status run_indexer(const LaunchCtx& c, const dsa_shape* s, const uint8_t* q_I, const float* q_scale,
                       const float* w, const uint8_t* k_I, const float* k_scale, int q_begin, int q_count,
                       float* scores, int64_t ld) {
  IndexerArgs a = {};
  a.kv = kv_map(s);
  a.kstride = 1;
  a.q_I = q_I; a.q_scale = q_scale; a.w = w; a.k_I = k_I; a.k_scale = k_scale;
  a.scores = scores; a.ld = ld;
  a.B = s->B; a.T = s->T; a.S = s->S; a.H_I = s->H_I; a.D_I = s->D_I;
  a.q_begin = q_begin; a.q_count = q_count;
  return from_cuda(launch_indexer(c, a));
}

dsa_status run_topk(const LaunchCtx& c, const dsa_shape* s, const float* scores, int64_t ld, int q_begin,
                    int q_count, int32_t* idx, void* ws, size_t ws_bytes) {
  TopkArgs a = {};
  a.kv = kv_map(s);
  a.scores = scores; a.ld = ld; a.idx = idx;
  a.B = s->B; a.T = s->T; a.S = s->S; a.k = s->k;
  a.q_begin = q_begin; a.q_count = q_count;
  return from_cuda(launch_topk(c, a, ws, ws_bytes));
}

// Steps A and B for query rows [q0, q0 + cnt) (cnt <= q_rows) without the
// score tile: key sample -> thresholds -> candidates -> exact selection ->
// repair of the rows that fell short or overflowed.
dsa_status run_select_fused(const LaunchCtx& c, const dsa_shape* s, const WsLayout& L, char* ws, const uint8_t* q_I,
                            const float* q_scale, const float* w, const uint8_t* k_I, const float* k_scale, int q0,
                            int cnt, int32_t* idx) {
  float* sample = reinterpret_cast<float*>(ws + L.sample_off);
  unsigned int* thr = reinterpret_cast<unsigned int*>(ws + L.thr_off);
  unsigned int* ccnt = reinterpret_cast<unsigned int*>(ws + L.cnt_off);
  int* slot = reinterpret_cast<int*>(ws + L.slot_off);
  int* rfail = reinterpret_cast<int*>(ws + L.rfail_off);
  int32_t* wrow = reinterpret_cast<int32_t*>(ws + L.wrow_off);
  int32_t* widx = reinterpret_cast<int32_t*>(ws + L.widx_off);
  unsigned int* wkey = reinterpret_cast<unsigned int*>(ws + L.wkey_off);
  unsigned int* wcnt = reinterpret_cast<unsigned int*>(ws + L.wcnt_off);
  unsigned int* ckey = reinterpret_cast<unsigned int*>(ws + L.ckey_off);
  int32_t* cidx = reinterpret_cast<int32_t*>(ws + L.cidx_off);
  int* fail = reinterpret_cast<int*>(ws + L.fail_off);
  unsigned int* nfail = reinterpret_cast<unsigned int*>(ws + L.nfail_off);
  float* repair = reinterpret_cast<float*>(ws + L.repair_off);
  IndexerArgs ia = {};
  ia.kv = kv_map(s);
  ia.kstride = 1;
  ia.q_I = q_I; ia.q_scale = q_scale; ia.w = w; ia.k_I = k_I; ia.k_scale = k_scale;
  ia.B = s->B; ia.T = s->T; ia.S = s->S; ia.H_I = s->H_I; ia.D_I = s->D_I;
  ia.q_begin = q0; ia.q_count = cnt;
  TopkArgs ta = {};
  ta.kv = kv_map(s);
  ta.scores = nullptr; ta.ld = 0; ta.idx = idx;
  ta.B = s->B; ta.T = s->T; ta.S = s->S; ta.k = s->k;
  ta.q_begin = q0; ta.q_count = cnt;
  cudaError_t e;
  // 1. scores of every kSampleStride-th key, when some row sees more keys
  //    than its candidate list holds
  const bool long_rows = (long long)s->S - s->T + q0 + cnt > L.cap;
  if (long_rows) {
    IndexerArgs sa = ia;
    sa.kstride = kSampleStride;
    sa.scores = sample;
    sa.ld = L.ld_s;
    if ((e = launch_indexer(c, sa)) != cudaSuccess) return DSA_ERR_CUDA;
  }
  // 2. per-row thresholds (about 1.5 k expected candidates); counts,
  //    flags and the warp lists' lengths cleared
  if ((e = launch_topk_threshold(c, ta, sample, L.ld_s, kSampleStride, s->k * kTargetNum / kTargetDen, L.cap, thr, ccnt,
                                 slot, rfail, nfail, wcnt, L.nwl)) != cudaSuccess)
    return DSA_ERR_CUDA;
  // 3. every key scored; each epilogue warp appends its candidates to its own list
  IndexerArgs ca = ia;
  ca.thr = thr;
  ca.wl_row = wrow;
  ca.wl_idx = widx;
  ca.wl_key = wkey;
  ca.wl_cnt = wcnt;
  ca.wl_cap = L.wl_cap;
  ca.row_fail = rfail;
  if ((e = launch_indexer(c, ca)) != cudaSuccess) return DSA_ERR_CUDA;
  // 4. the warp lists into per-row lists
  if ((e = launch_topk_scatter(c, wrow, widx, wkey, wcnt, L.wl_cap, L.nwl, ccnt, ckey, cidx, L.cap)) != cudaSuccess)
    return DSA_ERR_CUDA;
  // 5. exact selection among each row's candidates
  if ((e = launch_topk_cand_select(c, ta, ckey, cidx, ccnt, L.cap, rfail, slot, fail, nfail, kRepairRows)) !=
      cudaSuccess)
    return DSA_ERR_CUDA;
  // 6. repair (both launches return at once when no row was listed)
  IndexerArgs ra = ia;
  ra.row_slot = slot;
  ra.scores = repair;
  ra.ld = scores_ld(s);
  if ((e = launch_indexer(c, ra)) != cudaSuccess) return DSA_ERR_CUDA;
  TopkArgs rt = ta;
  if ((e = launch_topk_repair(c, rt, repair, scores_ld(s), fail, nfail, kRepairRows)) != cudaSuccess)
    return DSA_ERR_CUDA;
  return DSA_OK;
}

// Steps A and B for rows [q0, q0 + cnt) through the workspace: fused when it
// applies, else the score tile and dsa_topk's selection.
dsa_status run_select(const LaunchCtx& c, const dsa_shape* s, const WsLayout& L, void* ws, const uint8_t* q_I,
                      const float* q_scale, const float* w, const uint8_t* k_I, const float* k_scale, int q0, int cnt,
                      int32_t* idx) {
  if (L.fused) return run_select_fused(c, s, L, static_cast<char*>(ws), q_I, q_scale, w, k_I, k_scale, q0, cnt, idx);
  float* scores = reinterpret_cast<float*>(static_cast<char*>(ws) + L.scores_off);
  const int64_t ld = scores_ld(s);
  dsa_status st = run_indexer(c, s, q_I, q_scale, w, k_I, k_scale, q0, cnt, scores, ld);
  if (st != DSA_OK) return st;
  return run_topk(c, s, scores, ld, q0, cnt, idx, L.topk_bytes ? static_cast<char*>(ws) + L.topk_off : nullptr,
                  L.topk_bytes);
}

// idx null: dense causal attention of every row; otherwise rows t <
// dense_rows read keys 0..pos(t) and the rest read idx.
dsa_status run_attn(const LaunchCtx& c, const dsa_shape* s, const uint16_t* q, const uint16_t* kv,
                    const uint16_t* v, const int32_t* idx, int dense_rows, uint16_t* out, float* lse, float* part,
                    int nsplit) {
  AttnArgs a = {};
  a.map = kv_map(s);
  a.q = q; a.kv = kv; a.v = v; a.idx = idx; a.dense_rows = dense_rows;
  a.out = out; a.lse = lse; a.part = part;
  a.B = s->B; a.T = s->T; a.S = s->S; a.H = s->H; a.d_k = s->d_k; a.d_v = s->d_v; a.k = s->k;
  a.nsplit = nsplit;
  a.tau = tau_of(s);
  a.decode = s->mode == DSA_DECODE;
  if (a.decode && attn_decode_supported(a)) return from_cuda(launch_sparse_attn_decode(c, a, part));
  return from_cuda(launch_sparse_attn(c, a));
}

bool indexer_ptrs_ok(const uint8_t* q_I, const float* q_scale, const float* w, const uint8_t* k_I,
                     const float* k_scale) {
  return q_I && q_scale && w && k_I && k_scale && aligned16(q_I) && aligned16(k_I);
}

}  // namespace

dsa_status api_check_shape(const dsa_shape* s) { return check_shape(s); }
KvMap api_kv_map(const dsa_shape* s) { return kv_map(s); }
dsa_status api_make_ctx(void* stream, LaunchCtx* c) { return make_ctx(stream, c); }

}  // namespace dsa

using namespace dsa;

extern "C" {

int dsa_version(void) { return 200; }

const char* dsa_status_string(dsa_status st) {
  switch (st) {
    case DSA_OK: return "ok";
    case DSA_ERR_INVALID_ARG: return "invalid argument";
    case DSA_ERR_UNSUPPORTED: return "unsupported shape";
    case DSA_ERR_WORKSPACE: return "workspace missing or too small";
    case DSA_ERR_CUDA: return "CUDA error";
    case DSA_ERR_TIMEOUT: return "device wait timed out";
    case DSA_ERR_DEVICE_BOUNDS: return "device index out of bounds";
  }
  return "unknown status";
}

unsigned long long dsa_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

void dsa_set_wait_timeout_us(long long microseconds) {
  g_wait_ns = microseconds > 0 ? microseconds * 1000LL : kDefaultWaitNs;
}

size_t dsa_workspace_size(const dsa_shape* s) {
  if (check_shape(s) != DSA_OK) return 0;
  DeviceInfo d;
  int dev = 0;
  int sms = 148;
  if (device_info(&d, &dev) == DSA_OK) sms = d.num_sms;
  return ws_layout(s, sms, false).total;
}

size_t dsa_select_workspace_size(const dsa_shape* s) {
  if (check_shape(s) != DSA_OK) return 0;
  DeviceInfo d;
  int dev = 0;
  int sms = 148;
  if (device_info(&d, &dev) == DSA_OK) sms = d.num_sms;
  return ws_layout(s, sms, true).total;
}

dsa_status dsa_indexer_scores(const dsa_shape* s, const uint8_t* q_I, const float* q_scale, const float* w,
                              const uint8_t* k_I, const float* k_scale, int q_begin, int q_count,
                              float* scores, int64_t ld_scores, void* stream) {
  dsa_status st = check_shape(s);
  if (st != DSA_OK) return st;
  if (!indexer_ptrs_ok(q_I, q_scale, w, k_I, k_scale) || scores == nullptr || !aligned16(scores))
    return DSA_ERR_INVALID_ARG;
  if (q_begin < 0 || q_count < 0 || q_begin + q_count > s->T) return DSA_ERR_INVALID_ARG;
  if (ld_scores < s->S || ld_scores % 4 != 0) return DSA_ERR_INVALID_ARG;
  LaunchCtx c;
  if ((st = make_ctx(stream, &c)) != DSA_OK) return st;
  return run_indexer(c, s, q_I, q_scale, w, k_I, k_scale, q_begin, q_count, scores, ld_scores);
}

dsa_status dsa_topk(const dsa_shape* s, const float* scores, int64_t ld_scores, int q_begin, int q_count,
                    int32_t* idx, void* ws, size_t ws_bytes, void* stream) {
  dsa_status st = check_shape(s);
  if (st != DSA_OK) return st;
  if (scores == nullptr || idx == nullptr || !aligned16(scores)) return DSA_ERR_INVALID_ARG;
  if (q_begin < 0 || q_count < 0 || q_begin + q_count > s->T) return DSA_ERR_INVALID_ARG;
  if (ld_scores < s->S || ld_scores % 4 != 0) return DSA_ERR_INVALID_ARG;
  LaunchCtx c;
  if ((st = make_ctx(stream, &c)) != DSA_OK) return st;
  return run_topk(c, s, scores, ld_scores, q_begin, q_count, idx, ws, ws_bytes);
}

dsa_status dsa_select(const dsa_shape* s, const uint8_t* q_I, const float* q_scale, const float* w,
                      const uint8_t* k_I, const float* k_scale, int q_begin, int q_count, int32_t* idx, void* ws,
                      size_t ws_bytes, void* stream) {
  dsa_status st = check_shape(s);
  if (st != DSA_OK) return st;
  if (!indexer_ptrs_ok(q_I, q_scale, w, k_I, k_scale) || idx == nullptr) return DSA_ERR_INVALID_ARG;
  if (q_begin < 0 || q_count < 0 || q_begin + q_count > s->T) return DSA_ERR_INVALID_ARG;
  LaunchCtx c;
  if ((st = make_ctx(stream, &c)) != DSA_OK) return st;
  WsLayout L = ws_layout(s, c.num_sms, true);
  if (ws == nullptr || ws_bytes < L.total) return DSA_ERR_WORKSPACE;
  for (int q0 = q_begin; q0 < q_begin + q_count; q0 += L.q_rows) {
    const int cnt = (q_begin + q_count - q0) < L.q_rows ? (q_begin + q_count - q0) : L.q_rows;
    if ((st = run_select(c, s, L, ws, q_I, q_scale, w, k_I, k_scale, q0, cnt, idx)) != DSA_OK) return st;
  }
  return DSA_OK;
}

dsa_status dsa_sparse_attn(const dsa_shape* s, const uint16_t* q, const uint16_t* kv, const uint16_t* v,
                           const int32_t* idx, uint16_t* out, float* lse, void* ws, size_t ws_bytes, void* stream) {
  dsa_status st = check_shape(s);
  if (st != DSA_OK) return st;
  if (!q || !kv || !idx || !out || !aligned16(q) || !aligned16(kv) || !aligned16(out) || (v && !aligned16(v)))
    return DSA_ERR_INVALID_ARG;
  LaunchCtx c;
  if ((st = make_ctx(stream, &c)) != DSA_OK) return st;
  WsLayout L = ws_layout(s, c.num_sms, false);
  float* part = nullptr;
  if (L.nsplit > 1 || (s->mode == DSA_DECODE && attn_decode_nsplit(s->k) > 1)) {
    if (ws == nullptr || ws_bytes < L.total) return DSA_ERR_WORKSPACE;
    part = reinterpret_cast<float*>(static_cast<char*>(ws) + L.part_off);
  }
  return run_attn(c, s, q, kv, v, idx, 0, out, lse, part, L.nsplit);
}

dsa_status dsa_dense_attn(const dsa_shape* s, const uint16_t* q, const uint16_t* kv, const uint16_t* v,
                          uint16_t* out, float* lse, void* ws, size_t ws_bytes, void* stream) {
  dsa_status st = check_shape(s);
  if (st != DSA_OK) return st;
  if (!q || !kv || !out || !aligned16(q) || !aligned16(kv) || !aligned16(out) || (v && !aligned16(v)))
    return DSA_ERR_INVALID_ARG;
  LaunchCtx c;
  if ((st = make_ctx(stream, &c)) != DSA_OK) return st;
  WsLayout L = ws_layout(s, c.num_sms, false);
  float* part = nullptr;
  if (L.nsplit_dense > 1) {
    if (ws == nullptr || ws_bytes < L.total) return DSA_ERR_WORKSPACE;
    part = reinterpret_cast<float*>(static_cast<char*>(ws) + L.part_off);
  }
  return run_attn(c, s, q, kv, v, nullptr, 0, out, lse, part, L.nsplit_dense);
}

dsa_status dsa_forward(const dsa_shape* s, const dsa_inputs* in, uint16_t* out, float* lse, int32_t* idx_out,
                       void* ws, size_t ws_bytes, void* stream) {
  dsa_status st = check_shape(s);
  if (st != DSA_OK) return st;
  if (in == nullptr || out == nullptr || idx_out == nullptr) return DSA_ERR_INVALID_ARG;
  if (!indexer_ptrs_ok(in->q_I, in->q_scale, in->w, in->k_I, in->k_scale)) return DSA_ERR_INVALID_ARG;
  if (!in->q || !in->kv || !aligned16(in->q) || !aligned16(in->kv) || !aligned16(out) || (in->v && !aligned16(in->v)))
    return DSA_ERR_INVALID_ARG;
  LaunchCtx c;
  if ((st = make_ctx(stream, &c)) != DSA_OK) return st;
  WsLayout L = ws_choose(s, c.num_sms, ws == nullptr ? 0 : ws_bytes);
  if (ws == nullptr || ws_bytes < L.total) return DSA_ERR_WORKSPACE;
  float* scores = reinterpret_cast<float*>(static_cast<char*>(ws) + L.scores_off);
  float* part = L.part_bytes ? reinterpret_cast<float*>(static_cast<char*>(ws) + L.part_off) : nullptr;
  const int64_t ld = scores_ld(s);
  // rows whose visible keys all fit in k: no scores, the selection is 0..pos
  const int d_rows = dense_rows_of(s);
  if (d_rows > 0 &&
      (st = run_topk(c, s, scores, ld, 0, d_rows, idx_out, nullptr, 0)) != DSA_OK)
    return st;
  for (int q0 = d_rows; q0 < s->T; q0 += L.q_rows) {
    const int cnt = (s->T - q0) < L.q_rows ? (s->T - q0) : L.q_rows;
    if ((st = run_select(c, s, L, ws, in->q_I, in->q_scale, in->w, in->k_I, in->k_scale, q0, cnt, idx_out)) !=
        DSA_OK)
      return st;
  }
  return run_attn(c, s, in->q, in->kv, in->v, idx_out, d_rows, out, lse, part, L.nsplit);
}

dsa_status dsa_prefill(const dsa_shape* s, const dsa_inputs* in, uint16_t* out, float* lse, int32_t* idx_out,
                       void* ws, size_t ws_bytes, void* stream) {
  if (s == nullptr) return DSA_ERR_INVALID_ARG;
  dsa_shape m = *s;
  m.mode = DSA_PREFILL;
  return dsa_forward(&m, in, out, lse, idx_out, ws, ws_bytes, stream);
}

dsa_status dsa_decode(const dsa_shape* s, const dsa_inputs* in, uint16_t* out, float* lse, int32_t* idx_out,
                      void* ws, size_t ws_bytes, void* stream) {
  if (s == nullptr) return DSA_ERR_INVALID_ARG;
  if (s->T != 1) return DSA_ERR_INVALID_ARG;
  dsa_shape m = *s;
  m.mode = DSA_DECODE;
  return dsa_forward(&m, in, out, lse, idx_out, ws, ws_bytes, stream);
}

dsa_status dsa_selftest_wait_timeout(void* stream) {
  LaunchCtx c;
  dsa_status st = make_ctx(stream, &c);
  if (st != DSA_OK) return st;
  return from_cuda(launch_wait_timeout_probe(c));
}

dsa_status dsa_get_device_error(void* stream, int* detail) {
  if (detail) *detail = 0;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return DSA_ERR_CUDA;
  DeviceInfo d;
  int dev = 0;
  dsa_status st = device_info(&d, &dev);
  if (st != DSA_OK) return st;
  DevErr host = {0u, 0u};
  if (cudaMemcpy(&host, d.err, sizeof(DevErr), cudaMemcpyDeviceToHost) != cudaSuccess) return DSA_ERR_CUDA;
  DevErr zero = {0u, 0u};
  if (cudaMemcpy(d.err, &zero, sizeof(DevErr), cudaMemcpyHostToDevice) != cudaSuccess) return DSA_ERR_CUDA;
  if (detail) *detail = (int)host.detail;
  return static_cast<dsa_status>(host.code);
}

}  // extern "C"
