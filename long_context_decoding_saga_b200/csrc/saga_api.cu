// saga_api.cu - host side of libsaga: argument validation, workspace layout,
// TMA descriptors, launch sizing and the extern "C" entry points of saga.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <mutex>

#include "saga.h"
#include "saga_internal.h"

namespace saga {
cudaError_t launch_split(int D, int NP, int mode, const CUtensorMap& tf, const CUtensorMap& tp, const SplitParams& p,
                         dim3 grid, cudaStream_t st, int* occupancy_out);
cudaError_t launch_from_scores(int D, int NP, const SplitParams& p, dim3 grid, cudaStream_t st, int* occ = nullptr);
cudaError_t launch_dense(int D, int NP, const CUtensorMap& kf, const CUtensorMap& kp, const CUtensorMap& vf,
                         const CUtensorMap& vp, const SplitParams& p, dim3 grid, cudaStream_t st, int* occ);
cudaError_t launch_combine(int D, const CombineParams& p, cudaStream_t st);
cudaError_t launch_select(const SelectParams& p, int rows, cudaStream_t st);
cudaError_t launch_select_cluster(const SelectParams& p, int rows, cudaStream_t st);
cudaError_t launch_append(const AppendParams& p, cudaStream_t st);
cudaError_t launch_qkv(const QkvParams& p, const CUtensorMap& tw, cudaStream_t st);
cudaError_t launch_fill(float* dst, float v, int n, cudaStream_t st);
}  // namespace saga

using namespace saga;

namespace {

thread_local char g_err[512] = "";
thread_local cudaEvent_t g_trace_start = nullptr, g_trace_end = nullptr;
thread_local unsigned g_test_wait_ns = 0;  // saga_test_expire_next_wait

cudaError_t trace_record(cudaEvent_t ev, cudaStream_t st) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cudaError_t e = cudaStreamIsCapturing(st, &cs);
  if (e != cudaSuccess) return e;
  return cudaEventRecordWithFlags(ev, st, cs == cudaStreamCaptureStatusActive ? cudaEventRecordExternal : cudaEventRecordDefault);
}

int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

int ok() {
  g_err[0] = '\0';
  return SAGA_OK;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(SAGA_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

struct DevInfo {
  int sms = 0;
  bool init = false;
};
DevInfo g_dev[128];
std::mutex g_dev_mu;

int device_sms(int* sms) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 128) return fail(SAGA_ERR_CUDA, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (!g_dev[dev].init) {
    int v = 0;
    e = cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    g_dev[dev].sms = v;
    g_dev[dev].init = true;
  }
  *sms = g_dev[dev].sms;
  return SAGA_OK;
}

// Sub-groups per key head: at d = 64 a group of 16 or more query heads runs
// as CTAs of 8 heads each (the 8-head kernel keeps two CTAs per SM and a
// light epilogue; the sub-groups' repeated key tiles come from L2), when the
// sub-groups split along value-head boundaries.
// Query heads per CTA.  At d = 64 a group of many query heads runs as
// sub-group CTAs that share each key tile through L2: 16 heads a CTA on
// reuse steps, 8 on the refresh path (score dump and compare/gather from the
// scores).  Measured per step against 8 everywhere: reuse steps of the
// 32-head groups 578 vs 725 us (batch 16) and 329 vs 418 us (batch 4);
// refresh steps 2786 vs 2551 us with 16.
int head_split(const saga_shape* s, bool refresh_path) {
  const int G = s->h_q / s->h_k, hpv = s->h_q / s->h_v;
  const int sub = refresh_path ? 8 : 16;
  if (s->d == 64 && G >= 2 * sub && G % sub == 0 && (sub % hpv == 0 || hpv % sub == 0)) return G / sub;
  return 1;
}

int np_for_group(int G) { return G <= 4 ? 4 : G <= 8 ? 8 : G <= 16 ? 16 : G <= 32 ? 32 : 64; }

int validate_shape(const saga_shape* s) {
  if (s == nullptr) return fail(SAGA_ERR_ARG, "shape is NULL");
  if (s->batch < 1 || s->h_q < 1 || s->h_k < 1 || s->h_v < 1 || s->l_cap < 1)
    return fail(SAGA_ERR_ARG, "shape fields must be >= 1 (batch=%d h_q=%d h_k=%d h_v=%d l_cap=%d)", s->batch, s->h_q,
                s->h_k, s->h_v, s->l_cap);
  if (s->d != 64 && s->d != 128) return fail(SAGA_ERR_UNSUPPORTED, "head dim d=%d not supported (64 or 128)", s->d);
  if (s->h_q % s->h_k != 0 || s->h_q % s->h_v != 0)
    return fail(SAGA_ERR_ARG, "h_q=%d must be a multiple of h_k=%d and h_v=%d", s->h_q, s->h_k, s->h_v);
  if (s->h_v % s->h_k != 0 && s->h_k % s->h_v != 0)
    return fail(SAGA_ERR_UNSUPPORTED, "one of h_k=%d, h_v=%d must divide the other", s->h_k, s->h_v);
  const int G = s->h_q / s->h_k;
  if (G > kMaxG) return fail(SAGA_ERR_UNSUPPORTED, "h_q/h_k=%d exceeds %d", G, kMaxG);
  if (s->d == 128 && G > 32) return fail(SAGA_ERR_UNSUPPORTED, "d=128 supports h_q/h_k <= 32 (got %d)", G);
  const int nvh = s->h_v >= s->h_k ? s->h_v / s->h_k : 1;
  if (nvh > kMaxNvh) return fail(SAGA_ERR_UNSUPPORTED, "h_v/h_k=%d exceeds %d", nvh, kMaxNvh);
  if ((long long)s->batch * s->h_k * s->l_cap >= (1ll << 31) ||
      (long long)s->batch * s->h_v * s->l_cap >= (1ll << 31) || (long long)s->batch * s->h_q >= (1 << 24))
    return fail(SAGA_ERR_UNSUPPORTED, "cache too large for 32-bit row coordinates");
  return SAGA_OK;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

WsLayout ws_layout(const saga_shape* s, int sms) {
  WsLayout w{};
  const int groups = s->batch * s->h_k;
  const long long rows = (long long)s->batch * s->h_q;
  const int tiles_cap = (s->l_cap + kTile - 1) / kTile;
  const long long by_sm = (32ll * kMaxCtasPerSm * sms + groups - 1) / groups;
  w.s_cap = (int)std::max(1ll, std::min((long long)tiles_cap, by_sm));
  w.ld_scores = ((long long)s->l_cap + 3) & ~3ll;
  size_t off = 0;
  w.status = off;
  off = align256(off + 16);
  w.part_o = off;
  off = align256(off + (size_t)rows * w.s_cap * s->d * 4);
  w.part_m = off;
  off = align256(off + (size_t)rows * w.s_cap * 4);
  w.part_l = off;
  off = align256(off + (size_t)rows * w.s_cap * 4);
  w.part_cnt = off;
  off = align256(off + (size_t)rows * w.s_cap * 4);
  w.scores = off;
  off = align256(off + (size_t)rows * w.ld_scores * 4);
  w.hist = off;
  off = align256(off + (size_t)rows * 256 * 4);
  w.idx = off;
  off = align256(off + (size_t)rows * s->l_cap * 4);
  w.total = off;
  return w;
}

// Split count per (batch, key head): minimise waves / splits over the
// resident-CTA slots of the device, at most one split per 128-token tile.
int choose_splits(int groups, int L_est, int slots, int s_cap) {
  const int tiles = std::max(1, (L_est + kTile - 1) / kTile);
  const int smax = std::max(1, std::min(s_cap, tiles));
  int best = 1;
  double best_cost = 1e30;
  for (int S = 1; S <= smax; ++S) {
    const long long ctas = (long long)groups * S;
    const long long waves = (ctas + slots - 1) / slots;
    const double cost = (double)waves / S * (1.0 + 1e-3 * S);
    if (cost < best_cost - 1e-12) {
      best_cost = cost;
      best = S;
    }
  }
  return best;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D view of the key cache: rows = B*h_k*l_cap tokens, d bf16 columns;
// boxes of 64 columns (one 128-byte swizzle atom) by `box_rows` rows.
// 2-D view of the value cache: rows = B*h_v*l_cap tokens, d bf16 columns;
// boxes of 64 columns by `box_rows` rows, stored row-major (no swizzle).
int make_value_map(CUtensorMap* m, const void* v_cache, const saga_shape* s, int box_rows) {
  EncodeTiledFn enc = get_encode();
  if (enc == nullptr) return fail(SAGA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable from the driver");
  cuuint64_t dims[2] = {(cuuint64_t)s->d, (cuuint64_t)s->batch * s->h_v * s->l_cap};
  cuuint64_t strides[1] = {(cuuint64_t)s->d * 2};
  cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(v_cache), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(SAGA_ERR_CUDA, "cuTensorMapEncodeTiled (values) failed (%d)", (int)r);
  return SAGA_OK;
}

int make_key_map(CUtensorMap* m, const void* k_cache, const saga_shape* s, int box_rows) {
  EncodeTiledFn enc = get_encode();
  if (enc == nullptr) return fail(SAGA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable from the driver");
  cuuint64_t dims[2] = {(cuuint64_t)s->d, (cuuint64_t)s->batch * s->h_k * s->l_cap};
  cuuint64_t strides[1] = {(cuuint64_t)s->d * 2};
  cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(k_cache), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(SAGA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return SAGA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Prepared {
  WsLayout ws;
  int sms;
  char* base;
};

int prepare_ws(const saga_shape* s, void* workspace, size_t ws_bytes, Prepared* out) {
  int rc = device_sms(&out->sms);
  if (rc) return rc;
  out->ws = ws_layout(s, out->sms);
  if (workspace == nullptr) return fail(SAGA_ERR_WORKSPACE, "workspace is NULL");
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return fail(SAGA_ERR_WORKSPACE, "workspace not 256-byte aligned");
  if (ws_bytes < out->ws.total)
    return fail(SAGA_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, out->ws.total);
  out->base = static_cast<char*>(workspace);
  return SAGA_OK;
}

// New token's rows for the fused append (all null: no append).
struct NewRows {
  uint16_t* k_cache = nullptr;
  uint16_t* v_cache = nullptr;
  const uint16_t* k_new = nullptr;
  const uint16_t* v_new = nullptr;
};

void fill_split_common(SplitParams& p, const saga_shape* s, const Prepared& pr, const void* q, const void* k_cache,
                       int seq_len, const int* seq_len_dev, bool refresh_path) {
  memset(&p, 0, sizeof(p));
  p.q = static_cast<const uint16_t*>(q);
  p.k_cache = static_cast<const uint16_t*>(k_cache);
  p.status = reinterpret_cast<unsigned*>(pr.base + pr.ws.status);
  p.seq_len_dev = seq_len_dev;
  p.seq_len = seq_len;
  p.batch = s->batch;
  p.h_q = s->h_q;
  p.h_k = s->h_k;
  p.h_v = s->h_v;
  p.l_cap = s->l_cap;
  p.s_cap = pr.ws.s_cap;
  p.ld_scores = pr.ws.ld_scores;
  p.hsplit = head_split(s, refresh_path);
  p.G = s->h_q / s->h_k / p.hsplit;
  const int hpv = s->h_q / s->h_v;  // query heads per value head
  p.nvh = p.G >= hpv ? p.G / hpv : 1;
  p.hpv = p.G / p.nvh;
  p.scale = (float)(1.0 / sqrt((double)s->d));
  p.part_o = reinterpret_cast<float*>(pr.base + pr.ws.part_o);
  p.part_m = reinterpret_cast<float*>(pr.base + pr.ws.part_m);
  p.part_l = reinterpret_cast<float*>(pr.base + pr.ws.part_l);
  p.part_cnt = reinterpret_cast<int*>(pr.base + pr.ws.part_cnt);
}

int splits_for(const saga_shape* s, const Prepared& pr, int seq_len, int NP, int hsplit, int mode,
               const CUtensorMap& tf, const CUtensorMap& tp, int* S, bool dense = false) {
  int occ = 0;
  SplitParams dummy{};
  cudaError_t e = dense ? launch_dense(s->d, NP, tf, tp, tf, tp, dummy, dim3(1), nullptr, &occ)
                        : launch_split(s->d, NP, mode, tf, tp, dummy, dim3(1), nullptr, &occ);
  if (e != cudaSuccess) return cuda_fail(e, "occupancy query");
  if (occ < 1) return fail(SAGA_ERR_UNSUPPORTED, "split kernel does not fit on an SM");
  // A small step (at most 16 key tiles per SM) is latency-bound: one split
  // per SM, which leaves a second CTA slot to the next call's kernel (it
  // starts its setup and L2 prefetch early).  Larger steps fill every slot.
  const int groups = s->batch * s->h_k * hsplit;
  const long long tiles = (long long)groups * ((seq_len + kTile - 1) / kTile);
  int slots = (occ > 1 && tiles <= 16ll * pr.sms) ? pr.sms : occ * pr.sms;
  // With one split CTA per SM, the combine CTAs of the previous call (up to
  // four share an SM once its split CTA has left) would hold back as many
  // split CTAs of this call until the combine ends: a small step leaves
  // them their SMs.
  const int combine_ctas = s->batch * s->h_q * (s->d / 32);
  const int reserve = (combine_ctas + 3) / 4;
  if (occ == 1 && tiles <= 16ll * pr.sms && reserve <= pr.sms / 8) slots = pr.sms - reserve;
  *S = choose_splits(groups, seq_len, slots, pr.ws.s_cap);
  return SAGA_OK;
}

int clear_status_word(const Prepared& pr, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(pr.base + pr.ws.status, 0, 16, st);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(status)");
  return SAGA_OK;
}

// Scores of every cached token and the exact
// threshold (refresh).  clear_status zeroes the status word first.
int run_refresh(const saga_shape* s, const Prepared& pr, const void* q, const void* k_cache, int seq_len,
                const int* seq_len_dev, int n_top, float* tau, cudaStream_t st, cudaEvent_t ev_start = nullptr,
                const NewRows& nr = NewRows(), bool clear_status = false) {
  const int hsplit = head_split(s, true);
  const int G = s->h_q / s->h_k / hsplit, NP = np_for_group(G);
  CUtensorMap tf, tp;
  int rc = make_key_map(&tf, k_cache, s, kTile);
  if (rc) return rc;
  rc = make_key_map(&tp, k_cache, s, kUnit);
  if (rc) return rc;
  int S = 1;
  rc = splits_for(s, pr, seq_len, NP, hsplit, kSplitDump, tf, tp, &S);
  if (rc) return rc;
  const size_t rows = (size_t)s->batch * s->h_q;
  if (clear_status) {
    rc = clear_status_word(pr, st);
    if (rc) return rc;
  }
  if (ev_start != nullptr) {
    cudaError_t et = trace_record(ev_start, st);
    if (et != cudaSuccess) return cuda_fail(et, "trace event record");
  }
  SplitParams p;
  fill_split_common(p, s, pr, q, k_cache, seq_len, seq_len_dev, true);
  p.k_cache_w = nr.k_cache;
  p.v_cache_w = nr.v_cache;
  p.k_new = nr.k_new;
  p.v_new = nr.v_new;
  p.scores_out = reinterpret_cast<float*>(pr.base + pr.ws.scores);
  // The select: one CTA per row scanning the whole row when the rows fill the
  // GPU or are short; else one thread-block cluster of CTAs per row, each CTA
  // a chunk.  Measured on refresh steps: rows of 32K scores (32 rows) 688 vs
  // 746 us and 512 rows of 128K 10.95 vs 11.94 ms per step with one CTA per
  // row than with rows in chunks over three kernels; for 12 and 32 rows of
  // 128K the cluster kernel against those three kernels: 1546 vs 1730 us and
  // 1048 vs 1158 us.  For groups of at most kDumpHistMaxNp heads the dump
  // also counts the top byte of the scores from two bins below the stale
  // threshold's up, and the select skips its first pass when those bins hold
  // N scores (else it counts the row itself, so any tau is exact).  With 12
  // heads per CTA that counting had cost the dump two thirds of its time (485
  // vs 175 us for 28 layers in one call), more than the pass it saves (148 vs
  // 55 us); with 4 heads the refresh steps are 11-16 % faster with it.
  uint32_t* hist = nullptr;
  if (NP <= kDumpHistMaxNp) {
    hist = reinterpret_cast<uint32_t*>(pr.base + pr.ws.hist);
    cudaError_t em = cudaMemsetAsync(hist, 0, rows * 256 * 4, st);
    if (em != cudaSuccess) return cuda_fail(em, "cudaMemsetAsync(hist)");
    p.hist_out = hist;
    p.hist_floor = 1;
    p.tau = tau;  // the stale threshold, read by the dump before the select overwrites it
  }
  const bool one_cta_per_row = rows >= (size_t)pr.sms || seq_len <= 32768;
  p.nsplit = S;
  cudaError_t e = launch_split(s->d, NP, kSplitDump, tf, tp, p, dim3(S * hsplit, s->h_k, s->batch), st, nullptr);
  if (e != cudaSuccess) return cuda_fail(e, "score dump launch");
  SelectParams sp{};
  sp.scores = p.scores_out;
  sp.ld = pr.ws.ld_scores;
  sp.hist = hist;
  sp.tau = tau;
  sp.spec = 1;  // tau holds the stale thresholds until the select writes the new ones
  sp.status = p.status;
  sp.seq_len_dev = seq_len_dev;
  sp.row_len = seq_len;
  sp.l_cap = s->l_cap;
  sp.n_top = n_top;
  e = one_cta_per_row ? launch_select(sp, (int)rows, st) : launch_select_cluster(sp, (int)rows, st);
  if (e != cudaSuccess) return cuda_fail(e, "radix select launch");
  return SAGA_OK;
}

}  // namespace

extern "C" {

int saga_abi_version(void) { return 102; }

const char* saga_last_error(void) { return g_err; }

size_t saga_workspace_bytes(const saga_shape* s) {
  if (validate_shape(s)) return 0;
  int sms = 0;
  if (device_sms(&sms)) return 0;
  return ws_layout(s, sms).total;
}

size_t atopn_select_workspace_bytes(int rows) {
  if (rows < 1) return 0;
  return 256;
}

int saga_kv_append(const saga_shape* s, void* k_cache, void* v_cache, const void* k_new, const void* v_new, int pos,
                   const int* seq_len_dev, void* stream) {
  int rc = validate_shape(s);
  if (rc) return rc;
  if (!k_cache || !v_cache || !k_new || !v_new) return fail(SAGA_ERR_ARG, "NULL tensor pointer");
  if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(k_new) || !aligned16(v_new))
    return fail(SAGA_ERR_ARG, "tensor pointers must be 16-byte aligned");
  if (pos < 0 || pos >= s->l_cap) return fail(SAGA_ERR_ARG, "pos=%d outside [0, l_cap=%d)", pos, s->l_cap);
  AppendParams p{};
  p.k_cache = static_cast<uint16_t*>(k_cache);
  p.v_cache = static_cast<uint16_t*>(v_cache);
  p.k_new = static_cast<const uint16_t*>(k_new);
  p.v_new = static_cast<const uint16_t*>(v_new);
  p.seq_len_dev = seq_len_dev;
  p.status = nullptr;
  p.pos = pos;
  p.batch = s->batch;
  p.h_k = s->h_k;
  p.h_v = s->h_v;
  p.d = s->d;
  p.l_cap = s->l_cap;
  cudaError_t e = launch_append(p, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "append launch");
  return ok();
}

static int validate_qkv(const saga_shape* s, int hidden) {
  int rc = validate_shape(s);
  if (rc) return rc;
  if (s->batch > kQkvN) return fail(SAGA_ERR_UNSUPPORTED, "saga_qkv_project supports batch <= %d (got %d)", kQkvN, s->batch);
  if (hidden < 8 || hidden % 8 != 0) return fail(SAGA_ERR_ARG, "hidden=%d must be a positive multiple of 8", hidden);
  if (hidden > kQkvMaxHidden) return fail(SAGA_ERR_UNSUPPORTED, "hidden=%d exceeds %d", hidden, kQkvMaxHidden);
  const long long n_cols = (long long)(s->h_q + s->h_k + s->h_v) * s->d;
  if (n_cols * hidden >= (1ll << 31)) return fail(SAGA_ERR_UNSUPPORTED, "projection too large for 32-bit indexing");
  return SAGA_OK;
}

constexpr size_t kQkvWorkspaceBytes = 256;  // the status word at offset 0, the rest reserved

size_t saga_qkv_workspace_bytes(const saga_shape* s, int hidden) {
  if (validate_qkv(s, hidden)) return 0;
  return kQkvWorkspaceBytes;
}

int saga_qkv_project(const saga_shape* s, int hidden, const void* x, const void* w_qkv, void* q_out, void* k_cache,
                     void* v_cache, int pos, const int* seq_len_dev, void* workspace, size_t ws_bytes, void* stream) {
  int rc = validate_qkv(s, hidden);
  if (rc) return rc;
  if (!x || !w_qkv || !q_out || !k_cache || !v_cache) return fail(SAGA_ERR_ARG, "NULL tensor pointer");
  if (!aligned16(x) || !aligned16(w_qkv) || !aligned16(q_out) || !aligned16(k_cache) || !aligned16(v_cache))
    return fail(SAGA_ERR_ARG, "tensor pointers must be 16-byte aligned");
  if (pos < 0 || pos >= s->l_cap) return fail(SAGA_ERR_ARG, "pos=%d outside [0, l_cap=%d)", pos, s->l_cap);
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(SAGA_ERR_WORKSPACE, "workspace must be a 256-byte aligned device buffer");
  if (ws_bytes < kQkvWorkspaceBytes)
    return fail(SAGA_ERR_WORKSPACE, "workspace of %zu bytes, %zu needed", ws_bytes, kQkvWorkspaceBytes);
  int sms = 0;
  rc = device_sms(&sms);
  if (rc) return rc;
  QkvParams p{};
  p.x = static_cast<const uint16_t*>(x);
  p.w = static_cast<const uint16_t*>(w_qkv);
  p.q = static_cast<uint16_t*>(q_out);
  p.k_cache = static_cast<uint16_t*>(k_cache);
  p.v_cache = static_cast<uint16_t*>(v_cache);
  p.seq_len_dev = seq_len_dev;
  p.status = static_cast<unsigned*>(workspace);
  p.pos = pos;
  p.batch = s->batch;
  p.hidden = hidden;
  p.n_cols = (s->h_q + s->h_k + s->h_v) * s->d;
  p.h_q = s->h_q;
  p.h_k = s->h_k;
  p.h_v = s->h_v;
  p.d = s->d;
  p.l_cap = s->l_cap;
  int m_tiles = 0;
  qkv_mma_plan(p.n_cols, hidden, sms, &m_tiles, &p.splits, &p.kb_total, &p.stages, &p.kbs_max);
  // w_qkv as rows of `hidden` bf16: boxes of 64 columns (one 128-byte swizzle row) by 128 rows
  CUtensorMap tw;
  EncodeTiledFn enc = get_encode();
  if (enc == nullptr) return fail(SAGA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable from the driver");
  cuuint64_t dims[2] = {(cuuint64_t)hidden, (cuuint64_t)p.n_cols};
  cuuint64_t strides[1] = {(cuuint64_t)hidden * 2};
  cuuint32_t box[2] = {(cuuint32_t)kQkvTileK, (cuuint32_t)kQkvTileM};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = enc(&tw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(w_qkv), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(SAGA_ERR_CUDA, "cuTensorMapEncodeTiled (weights) failed (%d)", (int)r);
  cudaError_t e = launch_qkv(p, tw, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "qkv launch");
  return ok();
}

int atopn_refresh_threshold(const saga_shape* s, const void* q, const void* k_cache, int seq_len,
                            const int* seq_len_dev, int n_top, float* tau, void* workspace, size_t ws_bytes,
                            void* stream) {
  int rc = validate_shape(s);
  if (rc) return rc;
  if (!q || !k_cache || !tau) return fail(SAGA_ERR_ARG, "NULL tensor pointer");
  if (!aligned16(q) || !aligned16(k_cache)) return fail(SAGA_ERR_ARG, "q and k_cache must be 16-byte aligned");
  if (seq_len < 1 || seq_len > s->l_cap) return fail(SAGA_ERR_ARG, "seq_len=%d outside [1, l_cap=%d]", seq_len, s->l_cap);
  if (n_top < 1) return fail(SAGA_ERR_ARG, "n_top=%d must be >= 1", n_top);
  Prepared pr;
  rc = prepare_ws(s, workspace, ws_bytes, &pr);
  if (rc) return rc;
  rc = run_refresh(s, pr, q, k_cache, seq_len, seq_len_dev, n_top, tau, static_cast<cudaStream_t>(stream));
  if (rc) return rc;
  return ok();
}

int atopn_select_threshold(const float* scores, int rows, int row_len, long long row_stride, int n_top, float* tau,
                           void* workspace, size_t ws_bytes, void* stream) {
  if (!scores || !tau) return fail(SAGA_ERR_ARG, "NULL pointer");
  if (rows < 1 || row_len < 1 || row_stride < row_len || (row_stride & 3) != 0)
    return fail(SAGA_ERR_ARG, "bad rows=%d row_len=%d row_stride=%lld", rows, row_len, row_stride);
  if (!aligned16(scores)) return fail(SAGA_ERR_ARG, "scores must be 16-byte aligned");
  if (n_top < 1) return fail(SAGA_ERR_ARG, "n_top=%d must be >= 1", n_top);
  if (workspace == nullptr || ws_bytes < atopn_select_workspace_bytes(rows))
    return fail(SAGA_ERR_WORKSPACE, "workspace too small");
  SelectParams sp{};
  sp.scores = scores;
  sp.ld = row_stride;
  sp.tau = tau;
  sp.status = static_cast<unsigned*>(workspace);
  sp.seq_len_dev = nullptr;
  sp.row_len = row_len;
  sp.l_cap = row_len;
  sp.n_top = n_top;
  cudaError_t e = launch_select(sp, rows, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "radix select launch");
  return ok();
}

}  // extern "C"

namespace {

// One attention step; with nr set, the new token's rows are appended at
// seq_len - 1 by the attention kernels themselves.  clear_status zeroes the
// workspace status word once every argument has been checked, just before
// the first enqueue.
int decode_impl(const saga_shape* s, const void* q, const void* k_cache, const void* v_cache, int seq_len,
                const int* seq_len_dev, int n_top, int refresh_interval, long long step, float* tau, void* out,
                int out_dtype, int* sel_count, int* sel_idx, void* workspace, size_t ws_bytes, void* stream,
                const NewRows& nr, bool clear_status = false) {
  int rc = validate_shape(s);
  if (rc) return rc;
  if (!q || !k_cache || !v_cache || !tau || !out) return fail(SAGA_ERR_ARG, "NULL tensor pointer");
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out))
    return fail(SAGA_ERR_ARG, "tensor pointers must be 16-byte aligned");
  if (seq_len < 1 || seq_len > s->l_cap) return fail(SAGA_ERR_ARG, "seq_len=%d outside [1, l_cap=%d]", seq_len, s->l_cap);
  if (n_top < 1) return fail(SAGA_ERR_ARG, "n_top=%d must be >= 1", n_top);
  if (refresh_interval < 1) return fail(SAGA_ERR_ARG, "refresh_interval=%d must be >= 1", refresh_interval);
  if (step < 0) return fail(SAGA_ERR_ARG, "step=%lld must be >= 0", step);
  if (out_dtype != SAGA_OUT_F32 && out_dtype != SAGA_OUT_BF16) return fail(SAGA_ERR_ARG, "bad out_dtype %d", out_dtype);
  if (sel_idx != nullptr && sel_count == nullptr) return fail(SAGA_ERR_ARG, "sel_idx requires sel_count");
  Prepared pr;
  rc = prepare_ws(s, workspace, ws_bytes, &pr);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool refresh = (step % refresh_interval) == 0;
  const bool no_threshold = n_top >= s->l_cap;  // every possible length is covered by N
  const bool refresh_path = refresh && !no_threshold;
  const int hsplit = head_split(s, refresh_path);
  const int G = s->h_q / s->h_k / hsplit, NP = np_for_group(G);
  const int rows = s->batch * s->h_q;

  CUtensorMap tf, tp;
  rc = make_key_map(&tf, k_cache, s, kTile);
  if (rc) return rc;
  rc = make_key_map(&tp, k_cache, s, kUnit);
  if (rc) return rc;

  cudaEvent_t ev0 = g_trace_start, ev1 = g_trace_end;
  g_trace_start = g_trace_end = nullptr;
  const unsigned test_wait_ns = g_test_wait_ns;
  g_test_wait_ns = 0;

  SplitParams p;
  fill_split_common(p, s, pr, q, k_cache, seq_len, seq_len_dev, refresh_path);
  p.v_cache = static_cast<const uint16_t*>(v_cache);
  p.tau = tau;
  p.want_counts = sel_count != nullptr;
  p.idxbuf = sel_idx != nullptr ? reinterpret_cast<int*>(pr.base + pr.ws.idx) : nullptr;
  cudaError_t e;
  int S = 1;
  if (refresh_path) {
    rc = run_refresh(s, pr, q, k_cache, seq_len, seq_len_dev, n_top, tau, st, ev0, nr, clear_status);
    if (rc) return rc;
    // the compare/gather pass reads scores, not keys: it runs with every
    // CTA slot filled (it is latency-bound on its score loads per tile)
    {
      int occ = 0;
      SplitParams dummy{};
      e = launch_from_scores(s->d, NP, dummy, dim3(1), nullptr, &occ);
      if (e != cudaSuccess) return cuda_fail(e, "occupancy query");
      if (occ < 1) return fail(SAGA_ERR_UNSUPPORTED, "from-scores kernel does not fit on an SM");
      S = choose_splits(s->batch * s->h_k * hsplit, seq_len, occ * pr.sms, pr.ws.s_cap);
    }
    p.scores_in = reinterpret_cast<const float*>(pr.base + pr.ws.scores);
    p.nsplit = S;
    e = launch_from_scores(s->d, NP, p, dim3(S * hsplit, s->h_k, s->batch), st);
    if (e != cudaSuccess) return cuda_fail(e, "from-scores launch");
  } else {
    const int mode = no_threshold ? kSplitDense : kSplitSparse;
    // every token kept and one value head per group: the dense kernel (value
    // tiles by TMA, no lists)
    const bool dense = no_threshold && p.nvh == 1 && s->h_v <= s->h_k && NP <= 16;
    CUtensorMap vf, vp;
    if (dense) {
      rc = make_value_map(&vf, v_cache, s, kTile);
      if (rc) return rc;
      rc = make_value_map(&vp, v_cache, s, kUnit);
      if (rc) return rc;
    }
    rc = splits_for(s, pr, seq_len, NP, hsplit, mode, tf, tp, &S, dense);
    if (rc) return rc;
    p.nsplit = S;
    if (!dense) p.test_wait_ns = test_wait_ns;
    if (clear_status) {
      rc = clear_status_word(pr, st);
      if (rc) return rc;
    }
    if (ev0 != nullptr) {
      e = trace_record(ev0, st);
      if (e != cudaSuccess) return cuda_fail(e, "trace event record");
    }
    if (refresh) {
      e = launch_fill(tau, -INFINITY, rows, st);
      if (e != cudaSuccess) return cuda_fail(e, "threshold fill launch");
    }
    if (no_threshold) p.tau = nullptr;  // every token kept; the threshold is not read
    p.k_cache_w = nr.k_cache;
    p.v_cache_w = nr.v_cache;
    p.k_new = nr.k_new;
    p.v_new = nr.v_new;
    e = dense ? launch_dense(s->d, NP, tf, tp, vf, vp, p, dim3(S * hsplit, s->h_k, s->batch), st, nullptr)
              : launch_split(s->d, NP, mode, tf, tp, p, dim3(S * hsplit, s->h_k, s->batch), st, nullptr);
    if (e != cudaSuccess) return cuda_fail(e, dense ? "dense launch" : "split launch");
  }
  if (ev1 != nullptr) {
    e = trace_record(ev1, st);
    if (e != cudaSuccess) return cuda_fail(e, "trace event record");
  }
  CombineParams c{};
  c.part_o = p.part_o;
  c.part_m = p.part_m;
  c.part_l = p.part_l;
  c.part_cnt = p.part_cnt;
  c.idxbuf = p.idxbuf;
  c.out = out;
  c.sel_count = sel_count;
  c.sel_idx = sel_idx;
  c.status = p.status;
  c.seq_len_dev = seq_len_dev;
  c.seq_len = seq_len;
  c.rows = rows;
  c.nsplit = S;
  c.s_cap = pr.ws.s_cap;
  c.l_cap = s->l_cap;
  c.out_bf16 = out_dtype == SAGA_OUT_BF16;
  e = launch_combine(s->d, c, st);
  if (e != cudaSuccess) return cuda_fail(e, "combine launch");
  return ok();
}

}  // namespace

extern "C" {

int saga_decode_attn(const saga_shape* s, const void* q, const void* k_cache, const void* v_cache, int seq_len,
                     const int* seq_len_dev, int n_top, int refresh_interval, long long step, float* tau, void* out,
                     int out_dtype, int* sel_count, int* sel_idx, void* workspace, size_t ws_bytes, void* stream) {
  return decode_impl(s, q, k_cache, v_cache, seq_len, seq_len_dev, n_top, refresh_interval, step, tau, out, out_dtype,
                     sel_count, sel_idx, workspace, ws_bytes, stream, NewRows());
}

int saga_decode_step(const saga_shape* s, const void* q, const void* k_new, const void* v_new, void* k_cache,
                     void* v_cache, int seq_len, const int* seq_len_dev, int n_top, int refresh_interval,
                     long long step, float* tau, void* out, int out_dtype, int* sel_count, int* sel_idx,
                     void* workspace, size_t ws_bytes, void* stream) {
  if (k_new == nullptr || v_new == nullptr) return fail(SAGA_ERR_ARG, "NULL k_new / v_new");
  if (!aligned16(k_new) || !aligned16(v_new)) return fail(SAGA_ERR_ARG, "k_new and v_new must be 16-byte aligned");
  NewRows nr;
  nr.k_cache = static_cast<uint16_t*>(k_cache);
  nr.v_cache = static_cast<uint16_t*>(v_cache);
  nr.k_new = static_cast<const uint16_t*>(k_new);
  nr.v_new = static_cast<const uint16_t*>(v_new);
  return decode_impl(s, q, k_cache, v_cache, seq_len, seq_len_dev, n_top, refresh_interval, step, tau, out, out_dtype,
                     sel_count, sel_idx, workspace, ws_bytes, stream, nr);
}

int saga_test_expire_next_wait(unsigned limit_ns) {
  g_test_wait_ns = limit_ns;
  return ok();
}

int saga_trace_next_attention(void* ev_start, void* ev_end) {
  if ((ev_start == nullptr) != (ev_end == nullptr)) return fail(SAGA_ERR_ARG, "pass both events or neither");
  g_trace_start = static_cast<cudaEvent_t>(ev_start);
  g_trace_end = static_cast<cudaEvent_t>(ev_end);
  return ok();
}

int saga_get_status(const void* workspace, void* stream, unsigned* status) {
  if (workspace == nullptr || status == nullptr) return fail(SAGA_ERR_ARG, "NULL pointer");
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  e = cudaMemcpy(status, workspace, sizeof(unsigned), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy(status)");
  return ok();
}

}  // extern "C"

namespace saga {
// saga_decode_attn that zeroes the workspace status word once the arguments
// have been checked (used by the allocation-free entry point).
int decode_attn_clearing_status(const saga_shape* s, const void* q, const void* k_cache, const void* v_cache,
                                int seq_len, const int* seq_len_dev, int n_top, int refresh_interval, long long step,
                                float* tau, void* out, int out_dtype, int* sel_count, int* sel_idx, void* workspace,
                                size_t ws_bytes, void* stream) {
  return decode_impl(s, q, k_cache, v_cache, seq_len, seq_len_dev, n_top, refresh_interval, step, tau, out, out_dtype,
                     sel_count, sel_idx, workspace, ws_bytes, stream, NewRows(), true);
}
}  // namespace saga

