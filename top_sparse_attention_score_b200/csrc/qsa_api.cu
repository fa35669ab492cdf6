// qsa_api.cu -- the C ABI declared in include/qsa.h: argument checks, workspace
// planning and kernel launches.  Every step of the computation runs in the
// kernels of the qsa_*.cuh files; nothing here touches the data.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <string>

#include "qsa.h"
#include "qsa_attn.cuh"
#include "qsa_cache_write.cuh"
#include "qsa_common.cuh"
#include "qsa_index_score.cuh"
#include "qsa_merge.cuh"
#include "qsa_topk.cuh"

namespace {

thread_local std::string g_error;
std::atomic<uint64_t> g_launches{0};

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_error = buf;
  return code;
}

int ok() {
  g_error.clear();
  return QSA_OK;
}

// Count a launch and turn a launch error into QSA_ERR_CUDA.
int launched(const char* what) {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(QSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return QSA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int check_cache(const qsa_cache* c) {
  if (!c) return fail(QSA_ERR_ARG, "cache is NULL");
  if (!c->k || !c->v || !c->ks || !c->vs || !c->idx_key)
    return fail(QSA_ERR_ARG, "cache has a NULL array");
  if (c->max_cells < 1 || c->max_cells > QSA_MAX_CELLS)
    return fail(QSA_ERR_ARG, "cache max_cells %d out of [1, %d]", c->max_cells, QSA_MAX_CELLS);
  if (!aligned16(c->k) || !aligned16(c->v) || !aligned16(c->ks) || !aligned16(c->vs) ||
      !aligned16(c->idx_key))
    return fail(QSA_ERR_ARG, "cache arrays must be 16-byte aligned");
  return QSA_OK;
}

// Opt the kernels that need it into large dynamic shared memory, once per device.
int prepare_device() {
  static std::atomic<uint64_t> done_mask{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return fail(QSA_ERR_CUDA, "cudaGetDevice failed");
  const uint64_t bit = 1ull << (dev & 63);
  if (done_mask.load() & bit) return QSA_OK;
  cudaError_t e = cudaFuncSetAttribute(qsa::topk_final_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       2 * (qsa::kMaxWindowBits / 32) * 4);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(qsa::attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(sizeof(qsa::AttnSmem)));
  if (e != cudaSuccess) return fail(QSA_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
  done_mask.fetch_or(bit);
  return QSA_OK;
}

// ---- workspace plan -------------------------------------------------------

struct TopkPlan {
  size_t hist, ctr, sure, cand, end;
  int cand_cap;
};

TopkPlan plan_topk(size_t at, int rows, int vmax, int top_k) {
  TopkPlan p;
  p.cand_cap = std::min(vmax, std::max(8 * top_k, 16384));
  p.hist = align_up(at, 256);
  p.ctr = align_up(p.hist + static_cast<size_t>(rows) * qsa::kBins * 4, 256);
  p.sure = align_up(p.ctr + static_cast<size_t>(rows) * 4 * 4, 256);
  p.cand = align_up(p.sure + static_cast<size_t>(rows) * top_k * 4, 256);
  p.end = align_up(p.cand + static_cast<size_t>(rows) * p.cand_cap * 8, 256);
  return p;
}

qsa::TopkWs topk_ws(void* base, const TopkPlan& p) {
  char* b = static_cast<char*>(base);
  qsa::TopkWs w;
  w.hist = reinterpret_cast<uint32_t*>(b + p.hist);
  w.ctr = reinterpret_cast<uint32_t*>(b + p.ctr);
  w.sure = reinterpret_cast<int32_t*>(b + p.sure);
  w.cand = reinterpret_cast<uint2*>(b + p.cand);
  w.cand_cap = p.cand_cap;
  return w;
}

struct StepPlan {
  int64_t ld;        // scores row stride
  size_t scores;     // [rows][ld] fp32
  TopkPlan topk;
  size_t ids;        // [rows][top_k] int32 (used when the caller passes no ids_out)
  size_t part;       // [rows][24][nsplit][258] fp32 (nsplit > 1)
  size_t total;
};

int auto_nsplit(int rows, int top_k) {
  // Enough (row, KV head, split) CTAs to cover the 148 SMs twice, pieces of >= 32 cells.
  const int want = (2 * 148 + 2 * rows - 1) / (2 * rows);
  return std::max(1, std::min({QSA_MAX_SPLITS, std::max(1, top_k / 32), want}));
}

StepPlan plan_step(int rows, int ncells, int vmax, int top_k, int nsplit) {
  StepPlan p;
  p.ld = static_cast<int64_t>(align_up(static_cast<size_t>(ncells), 4));
  p.scores = 0;
  const size_t after_scores = static_cast<size_t>(rows) * p.ld * 4;
  p.topk = plan_topk(after_scores, rows, vmax, top_k);
  p.ids = p.topk.end;
  p.part = align_up(p.ids + static_cast<size_t>(rows) * top_k * 4, 256);
  const size_t part_bytes =
      nsplit > 1 ? static_cast<size_t>(rows) * QSA_HQ * nsplit * QSA_PART_STRIDE * 4 : 0;
  p.total = align_up(p.part + part_bytes, 256);
  return p;
}

// ---- launches -------------------------------------------------------------

int launch_index_score(const qsa_cache* c, int rows, int ncells, const uint16_t* iq,
                       const float* iw, float* scores, int64_t ld, cudaStream_t s) {
  const dim3 grid((ncells + qsa::kScoreCellsPerCta - 1) / qsa::kScoreCellsPerCta,
                  (rows + qsa::kScoreRowsPerCta - 1) / qsa::kScoreRowsPerCta);
  qsa::index_score_kernel<<<grid, 128, 0, s>>>(reinterpret_cast<const __half*>(c->idx_key), ncells,
                                               reinterpret_cast<const __half*>(iq), iw, rows,
                                               scores, ld);
  return launched("index_score_kernel");
}

int launch_topk(const float* scores, int64_t ld, int rows, int vis0, int top_k, void* ws,
                const TopkPlan& p, int32_t* ids, cudaStream_t s) {
  const qsa::TopkWs w = topk_ws(ws, p);
  const int vmax = vis0 + rows - 1;
  // hist and ctr are adjacent up to alignment padding; zero both regions.
  const int64_t nzero = static_cast<int64_t>((p.sure - p.hist) / 4);
  const int zblocks = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(592, (nzero + 255) / 256)));
  qsa::topk_zero_kernel<<<zblocks, 256, 0, s>>>(w.hist, nzero);
  int r = launched("topk_zero_kernel");
  if (r) return r;
  const dim3 grid((vmax + qsa::kTopkChunk - 1) / qsa::kTopkChunk, rows);
  qsa::topk_hist_kernel<<<grid, qsa::kTopkThreads, 0, s>>>(scores, ld, vis0, top_k, w);
  if ((r = launched("topk_hist_kernel"))) return r;
  qsa::topk_filter_kernel<<<grid, qsa::kTopkThreads, 0, s>>>(scores, ld, vis0, top_k, w);
  if ((r = launched("topk_filter_kernel"))) return r;
  const int win = std::min(qsa::kMaxWindowBits, static_cast<int>(align_up(vmax, 32)));
  const size_t smem = 2 * static_cast<size_t>(win / 32) * 4;
  qsa::topk_final_kernel<<<rows, qsa::kFinalThreads, smem, s>>>(scores, ld, vis0, top_k, w, win,
                                                                ids);
  return launched("topk_final_kernel");
}

int launch_attn(const qsa_cache* c, int rows, const float* q, const int32_t* ids, int top_k,
                int nsplit, float scale, float* part, float* out, cudaStream_t s) {
  qsa::AttnArgs a;
  a.k = c->k;
  a.v = c->v;
  a.ks = reinterpret_cast<const __half*>(c->ks);
  a.vs = reinterpret_cast<const __half*>(c->vs);
  a.q = q;
  a.ids = ids;
  a.top_k = top_k;
  a.max_cells = c->max_cells;
  a.nsplit = nsplit;
  a.piece = (top_k + nsplit - 1) / nsplit;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.part = part;
  a.out = out;
  const dim3 grid(nsplit, QSA_HKV, rows);
  qsa::attn_kernel<<<grid, 128, sizeof(qsa::AttnSmem), s>>>(a);
  return launched("attn_kernel");
}

int launch_merge(const float* part, int rows, int nsplit, float* out, cudaStream_t s) {
  qsa::merge_kernel<<<rows * QSA_HQ, 256, 0, s>>>(part, nsplit, out);
  return launched("merge_kernel");
}

// The whole step for `rows` query rows; row r sees vis0 + r cells of ncells.
int run_step(const qsa_cache* c, int rows, int vis0, int ncells, const float* q,
             const uint16_t* iq, const float* iw, int top_k, int nsplit, float scale, void* ws,
             size_t ws_bytes, float* out, int32_t* ids_out, cudaStream_t s) {
  if (!q || !iq || !iw || !out) return fail(QSA_ERR_ARG, "q, iq, iw and out must not be NULL");
  if (!ws) return fail(QSA_ERR_WORKSPACE, "workspace is NULL");
  if (!aligned16(q) || !aligned16(iq) || !aligned16(out) || !aligned16(ws) ||
      (ids_out && !aligned16(ids_out)))
    return fail(QSA_ERR_ARG, "q, iq, out, ids_out and ws must be 16-byte aligned");
  const int vmax = vis0 + rows - 1;
  const StepPlan p = plan_step(rows, ncells, vmax, top_k, nsplit);
  if (ws_bytes < p.total)
    return fail(QSA_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, p.total);
  int r = prepare_device();
  if (r) return r;
  char* base = static_cast<char*>(ws);
  float* scores = reinterpret_cast<float*>(base + p.scores);
  int32_t* ids = ids_out ? ids_out : reinterpret_cast<int32_t*>(base + p.ids);
  float* part = reinterpret_cast<float*>(base + p.part);
  if ((r = launch_index_score(c, rows, ncells, iq, iw, scores, p.ld, s))) return r;
  if ((r = launch_topk(scores, p.ld, rows, vis0, top_k, base, p.topk, ids, s))) return r;
  if ((r = launch_attn(c, rows, q, ids, top_k, nsplit, scale, part, out, s))) return r;
  if (nsplit > 1 && (r = launch_merge(part, rows, nsplit, out, s))) return r;
  return ok();
}

}  // namespace

extern "C" {

size_t qsa_workspace_bytes(int mode, int rows, int L, int top_k, int nsplit) {
  if (rows < 1 || L < rows || top_k < 1 || top_k > QSA_MAX_TOPK || nsplit < 0 ||
      nsplit > QSA_MAX_SPLITS || L > QSA_MAX_CELLS)
    return 0;
  if (mode == QSA_MODE_DECODE) {
    if (rows > QSA_MAX_DECODE) return 0;
    const int ns = nsplit ? nsplit : auto_nsplit(rows, top_k);
    return plan_step(rows, L, L, top_k, ns).total;
  }
  if (mode == QSA_MODE_PREFILL) {
    const int ns = nsplit ? nsplit : auto_nsplit(rows, top_k);
    return plan_step(rows, L, L, top_k, ns).total;
  }
  return 0;
}

int qsa_cache_write(const qsa_cache* cache, int pos0, int n, const float* k, const float* v,
                    const uint16_t* idx_key, void* stream) {
  int r = check_cache(cache);
  if (r) return r;
  if (!k || !v || !idx_key) return fail(QSA_ERR_ARG, "k, v and idx_key must not be NULL");
  if (n < 1 || pos0 < 0 || static_cast<int64_t>(pos0) + n > cache->max_cells)
    return fail(QSA_ERR_ARG, "cells [%d, %d + %d) outside the cache of %d", pos0, pos0, n,
                cache->max_cells);
  const dim3 grid(n, QSA_HKV, 2);
  qsa::cache_write_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      cache->k, cache->v, reinterpret_cast<__half*>(cache->ks), reinterpret_cast<__half*>(cache->vs),
      reinterpret_cast<__half*>(cache->idx_key), pos0, k, v, reinterpret_cast<const __half*>(idx_key));
  if ((r = launched("cache_write_kernel"))) return r;
  return ok();
}

int qsa_decode(const qsa_cache* cache, int L, int n, const float* q, const uint16_t* iq,
               const float* iw, int top_k, int nsplit, float scale, void* ws, size_t ws_bytes,
               float* out, int32_t* ids_out, void* stream) {
  int r = check_cache(cache);
  if (r) return r;
  if (n < 1 || n > QSA_MAX_DECODE) return fail(QSA_ERR_ARG, "n = %d outside [1, 8]", n);
  if (L < n || L > cache->max_cells)
    return fail(QSA_ERR_ARG, "L = %d outside [n, max_cells = %d]", L, cache->max_cells);
  if (top_k < 1 || top_k > QSA_MAX_TOPK) return fail(QSA_ERR_ARG, "top_k = %d out of range", top_k);
  if (nsplit < 0 || nsplit > QSA_MAX_SPLITS) return fail(QSA_ERR_ARG, "nsplit = %d out of range", nsplit);
  const int ns = nsplit ? nsplit : auto_nsplit(n, top_k);
  return run_step(cache, n, L - n + 1, L, q, iq, iw, top_k, ns, scale, ws, ws_bytes, out, ids_out,
                  static_cast<cudaStream_t>(stream));
}

int qsa_prefill_chunk(const qsa_cache* cache, int pos0, int T, const float* q,
                      const uint16_t* iq, const float* iw, int top_k, float scale, void* ws,
                      size_t ws_bytes, float* out, int32_t* ids_out, void* stream) {
  int r = check_cache(cache);
  if (r) return r;
  if (T < 1 || pos0 < 0 || static_cast<int64_t>(pos0) + T > cache->max_cells)
    return fail(QSA_ERR_ARG, "chunk [%d, %d + %d) outside the cache of %d", pos0, pos0, T,
                cache->max_cells);
  if (top_k < 1 || top_k > QSA_MAX_TOPK) return fail(QSA_ERR_ARG, "top_k = %d out of range", top_k);
  const int ns = auto_nsplit(T, top_k);
  return run_step(cache, T, pos0 + 1, pos0 + T, q, iq, iw, top_k, ns, scale, ws, ws_bytes, out,
                  ids_out, static_cast<cudaStream_t>(stream));
}

int qsa_index_score(const qsa_cache* cache, int rows, int ncells, const uint16_t* iq,
                    const float* iw, float* scores, int64_t ld, void* stream) {
  int r = check_cache(cache);
  if (r) return r;
  if (!iq || !iw || !scores) return fail(QSA_ERR_ARG, "iq, iw and scores must not be NULL");
  if (rows < 1 || ncells < 1 || ncells > cache->max_cells)
    return fail(QSA_ERR_ARG, "rows = %d, ncells = %d out of range", rows, ncells);
  if (ld < ncells || ld % 4) return fail(QSA_ERR_ARG, "ld = %lld must be >= ncells and a multiple of 4",
                                         static_cast<long long>(ld));
  if (!aligned16(iq) || !aligned16(scores)) return fail(QSA_ERR_ARG, "iq and scores must be 16-byte aligned");
  if ((r = launch_index_score(cache, rows, ncells, iq, iw, scores, ld,
                              static_cast<cudaStream_t>(stream))))
    return r;
  return ok();
}

size_t qsa_topk_workspace_bytes(int rows, int L, int top_k) {
  if (rows < 1 || L < 1 || top_k < 1 || top_k > QSA_MAX_TOPK || L > QSA_MAX_CELLS) return 0;
  return plan_topk(0, rows, L, top_k).end;
}

int qsa_topk(const float* scores, int64_t ld, int rows, int vis0, int top_k, void* ws,
             size_t ws_bytes, int32_t* ids, void* stream) {
  if (!scores || !ids) return fail(QSA_ERR_ARG, "scores and ids must not be NULL");
  if (rows < 1 || vis0 < 1 || top_k < 1 || top_k > QSA_MAX_TOPK)
    return fail(QSA_ERR_ARG, "rows = %d, vis0 = %d, top_k = %d out of range", rows, vis0, top_k);
  const int64_t vmax = static_cast<int64_t>(vis0) + rows - 1;
  if (vmax > ld || ld % 4 || vmax > QSA_MAX_CELLS)
    return fail(QSA_ERR_ARG, "rows see up to %lld cells but ld = %lld (must be >= and a multiple of 4)",
                static_cast<long long>(vmax), static_cast<long long>(ld));
  if (!aligned16(scores) || !aligned16(ids)) return fail(QSA_ERR_ARG, "scores and ids must be 16-byte aligned");
  if (!ws) return fail(QSA_ERR_WORKSPACE, "workspace is NULL");
  const TopkPlan p = plan_topk(0, rows, static_cast<int>(vmax), top_k);
  if (ws_bytes < p.end) return fail(QSA_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, p.end);
  if (!aligned16(ws)) return fail(QSA_ERR_ARG, "ws must be 16-byte aligned");
  int r = prepare_device();
  if (r) return r;
  if ((r = launch_topk(scores, ld, rows, vis0, top_k, ws, p, ids, static_cast<cudaStream_t>(stream))))
    return r;
  return ok();
}

int qsa_attn(const qsa_cache* cache, int rows, const float* q, const int32_t* ids, int top_k,
             int nsplit, float scale, float* part, float* out, void* stream) {
  int r = check_cache(cache);
  if (r) return r;
  if (!q || !ids) return fail(QSA_ERR_ARG, "q and ids must not be NULL");
  if (rows < 1 || top_k < 1 || top_k > QSA_MAX_TOPK || nsplit < 1 || nsplit > QSA_MAX_SPLITS)
    return fail(QSA_ERR_ARG, "rows = %d, top_k = %d, nsplit = %d out of range", rows, top_k, nsplit);
  if (nsplit == 1 && !out) return fail(QSA_ERR_ARG, "nsplit == 1 needs out");
  if (nsplit > 1 && !part) return fail(QSA_ERR_ARG, "nsplit > 1 needs part");
  if (!aligned16(q) || (out && !aligned16(out)) || (part && !aligned16(part)))
    return fail(QSA_ERR_ARG, "q, part and out must be 16-byte aligned");
  if ((r = prepare_device())) return r;
  if ((r = launch_attn(cache, rows, q, ids, top_k, nsplit, scale, part, out,
                       static_cast<cudaStream_t>(stream))))
    return r;
  return ok();
}

int qsa_merge(const float* part, int rows, int nsplit, float* out, void* stream) {
  if (!part || !out) return fail(QSA_ERR_ARG, "part and out must not be NULL");
  if (rows < 1 || nsplit < 1 || nsplit > QSA_MAX_SPLITS)
    return fail(QSA_ERR_ARG, "rows = %d, nsplit = %d out of range", rows, nsplit);
  int r = launch_merge(part, rows, nsplit, out, static_cast<cudaStream_t>(stream));
  if (r) return r;
  return ok();
}

const char* qsa_last_error(void) { return g_error.c_str(); }

uint64_t qsa_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

}  // extern "C"

// ---- selection without a caller workspace ----------------------------------
//
// A fixed scratch buffer in global memory replaces the workspace for callers
// that cannot allocate (see qsa_topk_static in include/qsa.h).  Host code must
// not pass the symbol itself to a kernel -- on the host it names a stand-in, not
// device memory -- so its device address is looked up once per device.

static __device__ __align__(256) unsigned char g_topk_static_scratch[QSA_STATIC_SCRATCH_BYTES];

namespace {

std::mutex g_static_mu;
void* g_static_addr[64] = {};

// Device address of the scratch buffer on the current device (looked up on first use).
int static_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(QSA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= 64) return fail(QSA_ERR_ARG, "device %d outside the 64 this library tracks", dev);
  std::lock_guard<std::mutex> lock(g_static_mu);
  if (!g_static_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_topk_static_scratch);
    if (e != cudaSuccess || !p)
      return fail(QSA_ERR_CUDA, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
    g_static_addr[dev] = p;
  }
  *out = g_static_addr[dev];
  return QSA_OK;
}

}  // namespace

extern "C" int qsa_topk_static(const float* scores, int64_t ld, int rows, int vis0, int top_k,
                               int32_t* ids, void* stream) {
  if (!scores || !ids) return fail(QSA_ERR_ARG, "scores and ids must not be NULL");
  if (rows < 1 || rows > QSA_STATIC_MAX_ROWS)
    return fail(QSA_ERR_ARG, "rows = %d outside [1, %d] (the fixed scratch holds %d rows)", rows,
                QSA_STATIC_MAX_ROWS, QSA_STATIC_MAX_ROWS);
  if (top_k < 1 || top_k > QSA_STATIC_MAX_TOPK)
    return fail(QSA_ERR_ARG, "top_k = %d outside [1, %d] (the fixed scratch limit)", top_k,
                QSA_STATIC_MAX_TOPK);
  if (vis0 < 1) return fail(QSA_ERR_ARG, "vis0 = %d must be >= 1", vis0);
  const int64_t vmax = static_cast<int64_t>(vis0) + rows - 1;
  if (vmax > ld || ld % 4 || vmax > QSA_MAX_CELLS)
    return fail(QSA_ERR_ARG, "rows see up to %lld cells but ld = %lld (must be >= and a multiple of 4)",
                static_cast<long long>(vmax), static_cast<long long>(ld));
  if (!aligned16(scores) || !aligned16(ids)) return fail(QSA_ERR_ARG, "scores and ids must be 16-byte aligned");
  const TopkPlan p = plan_topk(0, rows, static_cast<int>(vmax), top_k);
  if (p.end > QSA_STATIC_SCRATCH_BYTES)
    return fail(QSA_ERR_ARG, "selection needs %zu bytes of scratch, the fixed buffer has %d", p.end,
                QSA_STATIC_SCRATCH_BYTES);
  void* ws = nullptr;
  int r = static_scratch(&ws);
  if (r) return r;
  if ((r = prepare_device())) return r;
  // launch_topk clears the histogram and counters before every use.
  if ((r = launch_topk(scores, ld, rows, vis0, top_k, ws, p, ids, static_cast<cudaStream_t>(stream))))
    return r;
  return ok();
}
