// qsa_api.cu -- the C ABI declared in include/qsa.h: argument checks, workspace
// planning and kernel launches.  Every step of the computation runs in the
// kernels of the qsa_*.cuh files; nothing here touches the data.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <string>
#include <utility>
#include <vector>

#include "qsa.h"
#include "qsa_attn.cuh"
#include "qsa_cache_write.cuh"
#include "qsa_common.cuh"
#include "qsa_index_score.cuh"
#include "qsa_merge.cuh"
#include "qsa_prefill_select.cuh"
#include "qsa_score_gemm.cuh"
#include "qsa_topk.cuh"
#include "qsa_topk_cluster.cuh"

// One status word per device: a kernel whose bounded wait expires records
// QSA_ERR_TIMEOUT here (read and cleared by qsa_device_status).
static __device__ uint32_t g_device_status;

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

// Per-kernel timing of this thread's calls (qsa_trace_begin / qsa_trace_end): an event
// on the traced stream before the first launch and after every launch.
struct Trace {
  bool on = false;
  cudaStream_t stream = nullptr;
  std::vector<cudaEvent_t> ev;     // ev[0]: the start; ev[i + 1]: after launch i
  std::vector<const char*> names;  // kernel of launch i
  int n = 0;
};
thread_local Trace g_trace;

// Count a launch and turn the error its launch call returned into QSA_ERR_CUDA.
// Only a failed launch clears the runtime's last-error state (which it set): an
// error left there by the caller's own earlier work is neither taken for this
// launch's nor cleared.
int launched(const char* what, cudaError_t e) {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(QSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  }
  if (g_trace.on && g_trace.n + 1 < static_cast<int>(g_trace.ev.size())) {
    g_trace.names[g_trace.n] = what;
    cudaEventRecord(g_trace.ev[++g_trace.n], g_trace.stream);
  }
  return QSA_OK;
}

// Launch with programmatic stream serialisation: the kernel may be scheduled
// while its predecessor on the stream drains; every kernel here waits on
// griddepcontrol.wait before touching memory its predecessors use.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
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

int g_sm_count[64] = {};
uint32_t* g_status_addr[64] = {};
bool g_wide_cluster[64] = {};  // a 16-CTA selection cluster can be scheduled on this device

bool wide_cluster_fits();

// Opt the kernels that need it into large dynamic shared memory and read the
// SM count, once per device.
int prepare_device() {
  static std::atomic<uint64_t> done_mask{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return fail(QSA_ERR_CUDA, "cudaGetDevice failed");
  const uint64_t bit = 1ull << (dev & 63);
  if (done_mask.load() & bit) return QSA_OK;
  cudaError_t e = cudaFuncSetAttribute(qsa::topk_final_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       2 * (qsa::kMaxWindowBits / 32) * 4);
#define QSA_ATTN_SMEM(W, ALL)                                                                   \
  if (e == cudaSuccess)                                                                         \
    e = cudaFuncSetAttribute(qsa::attn_kernel<W, ALL>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                             static_cast<int>(sizeof(qsa::AttnSmem<W>)));
  QSA_ATTN_SMEM(4, false) QSA_ATTN_SMEM(4, true) QSA_ATTN_SMEM(2, false) QSA_ATTN_SMEM(2, true)
#undef QSA_ATTN_SMEM
#define QSA_CLUSTER_SMEM(P, C)                                                                  \
  if (e == cudaSuccess)                                                                         \
    e = cudaFuncSetAttribute(qsa::cluster_select_kernel<P, C>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                             static_cast<int>(qsa::cluster_smem_bytes<P, C>()));
  QSA_CLUSTER_SMEM(1, 8) QSA_CLUSTER_SMEM(2, 8) QSA_CLUSTER_SMEM(4, 8) QSA_CLUSTER_SMEM(8, 8)
  QSA_CLUSTER_SMEM(16, 8) QSA_CLUSTER_SMEM(32, 16)
#undef QSA_CLUSTER_SMEM
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(qsa::cluster_select_kernel<32, qsa::kClusterCtasWide>,
                             cudaFuncAttributeNonPortableClusterSizeAllowed, 1);

  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(qsa::score_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             qsa::kGemmSmemRequest);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(qsa::prefill_threshold_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             qsa::kScoreRowsPerCta * qsa::kBins * 4);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(qsa::score_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             qsa::kSsSmemBytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(qsa::prefill_final_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             qsa::kPfSmemBytes);
  void* status = nullptr;
  if (e == cudaSuccess) e = cudaGetSymbolAddress(&status, g_device_status);
  int sms = 0;
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return fail(QSA_ERR_CUDA, "device set-up: %s", cudaGetErrorString(e));
  g_sm_count[dev & 63] = sms;
  g_wide_cluster[dev & 63] = wide_cluster_fits();
  g_status_addr[dev & 63] = static_cast<uint32_t*>(status);
  done_mask.fetch_or(bit);
  return QSA_OK;
}

uint32_t* device_status() {
  int dev = 0;
  cudaGetDevice(&dev);
  return g_status_addr[dev & 63];
}

int sm_count() {
  int dev = 0;
  cudaGetDevice(&dev);
  return g_sm_count[dev & 63] > 0 ? g_sm_count[dev & 63] : 148;
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
  p.sure = align_up(p.ctr + (static_cast<size_t>(rows) * qsa::kCtrWords + 4) * 4, 256);
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

// Prompt chunks of more than 8 rows select without a score matrix (qsa_prefill_select.cuh):
// per-row thresholds, the GEMM's candidate lists and their counts.  Offsets and sizes are
// planned for the largest grid the launch may use, so they do not depend on the device.
constexpr int kPlanMaxCtas = 296;

struct PrefillPlan {
  int n_tb, n_ct, items, grid_max;
  size_t thr, count, cand, end;
};

// GEMM CTAs for `sms` SMs: at most one per SM (and kPlanMaxCtas), but enough that no CTA
// covers more than one token block's cell tiles.
int prefill_grid(int items, int n_ct, int sms) {
  int grid = std::max(1, std::min({items, sms, kPlanMaxCtas}));
  if ((items + grid - 1) / grid > n_ct) grid = (items + n_ct - 1) / n_ct;
  return grid;
}

PrefillPlan plan_prefill(size_t at, int rows, int ncells) {
  PrefillPlan p;
  p.n_tb = (rows + qsa::kSsTokens - 1) / qsa::kSsTokens;
  p.n_ct = (ncells + qsa::kSsCells - 1) / qsa::kSsCells;
  p.items = p.n_tb * p.n_ct;
  p.grid_max = std::max(std::min(p.items, kPlanMaxCtas), (p.items + p.n_ct - 1) / p.n_ct);
  p.thr = align_up(at, 256);
  p.count = align_up(p.thr + static_cast<size_t>(rows) * 4, 256);
  p.cand = align_up(p.count + static_cast<size_t>(p.grid_max) * 2 * qsa::kSsTokens * 4, 256);
  // grid * per <= items + grid - 1, so every grid up to grid_max fits
  const size_t entries = static_cast<size_t>(qsa::kSsTokens) *
                         (static_cast<size_t>(qsa::kSsCapPerTile) * (p.items + p.grid_max) +
                          2 * static_cast<size_t>(qsa::kSsCapSlack) * p.grid_max);
  p.end = align_up(p.cand + entries * 8, 256);
  return p;
}

bool prefill_select_path(int rows, int vmax, int top_k) {
  return rows > qsa::kScoreRowsPerCta && vmax > top_k;
}

struct StepPlan {
  int64_t ld;        // scores row stride
  size_t scores;     // [rows][ld] fp32 (not used by the prompt selection path)
  TopkPlan topk;
  PrefillPlan pre;   // the prompt selection path
  bool prefill_select;
  size_t ids;        // [rows][top_k] int32 (used when the caller passes no ids_out)
  size_t part;       // [rows][24][nsplit][258] fp32 (nsplit > 1)
  size_t total;
};

int auto_nsplit(int rows, int top_k) {
  // Pieces of at least 32 cells.  Up to 8 rows: 32 pieces.  On a B200 the
  // graph-replayed decode step of 1-8 rows at 64K cells and top_k = 2048 was
  // fastest there or within noise of it for every row count (more pieces
  // shorten the gathers but lengthen the merge).  More rows: about 256 (row,
  // KV head, split) CTAs; large prefill chunks need no splits.
  const int want = rows <= QSA_MAX_DECODE ? 32 : 128 / rows;
  return std::max(1, std::min({QSA_MAX_SPLITS, std::max(1, top_k / 32), want}));
}

StepPlan plan_step(int rows, int ncells, int vmax, int top_k, int nsplit) {
  StepPlan p;
  p.ld = static_cast<int64_t>(align_up(static_cast<size_t>(ncells), 4));
  p.scores = 0;
  p.prefill_select = prefill_select_path(rows, vmax, top_k);
  size_t after;
  if (p.prefill_select) {
    p.pre = plan_prefill(0, rows, ncells);
    after = p.pre.end;
  } else {
    p.topk = plan_topk(static_cast<size_t>(rows) * p.ld * 4, rows, vmax, top_k);
    after = p.topk.end;
  }
  p.ids = after;
  p.part = align_up(p.ids + static_cast<size_t>(rows) * top_k * 4, 256);
  const size_t part_bytes =
      nsplit > 1 ? static_cast<size_t>(rows) * QSA_HQ * nsplit * QSA_PART_STRIDE * 4 : 0;
  p.total = align_up(p.part + part_bytes, 256);
  return p;
}

// ---- launches -------------------------------------------------------------

PFN_cuTensorMapEncodeTiled_v12000 g_encode_tiled = nullptr;
std::mutex g_encode_mu;

int tensor_map_encoder(PFN_cuTensorMapEncodeTiled_v12000* out) {
  std::lock_guard<std::mutex> lock(g_encode_mu);
  if (!g_encode_tiled) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    const cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn)
      return fail(QSA_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
    g_encode_tiled = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  *out = g_encode_tiled;
  return QSA_OK;
}

// Scores of `rows` > 8 rows: the tcgen05 GEMM, keys and queries fed by TMA.
int launch_score_gemm(const qsa_cache* c, int rows, int ncells, const uint16_t* iq, const float* iw,
                      float* scores, int64_t ld, cudaStream_t s) {
  PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  int r = tensor_map_encoder(&encode);
  if (r) return r;
  CUtensorMap tkey, tiq;
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(QSA_DI), static_cast<cuuint64_t>(ncells)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(QSA_DI) * 2};
    const cuuint32_t box[2] = {64u, static_cast<cuuint32_t>(qsa::kGemmCells)};
    const cuuint32_t estr[2] = {1u, 1u};
    const CUresult cr = encode(&tkey, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, c->idx_key, dims, strides, box, estr,
                               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr != CUDA_SUCCESS) return fail(QSA_ERR_CUDA, "tensor map of the keys: error %d", static_cast<int>(cr));
  }
  {
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(QSA_DI), static_cast<cuuint64_t>(QSA_HI),
                                static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(QSA_DI) * 2, static_cast<cuuint64_t>(QSA_HI * QSA_DI) * 2};
    const cuuint32_t box[3] = {64u, 1u, static_cast<cuuint32_t>(qsa::kGemmTokens)};
    const cuuint32_t estr[3] = {1u, 1u, 1u};
    const CUresult cr = encode(&tiq, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<uint16_t*>(iq), dims, strides,
                               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr != CUDA_SUCCESS) return fail(QSA_ERR_CUDA, "tensor map of the queries: error %d", static_cast<int>(cr));
  }
  CUtensorMap tout;
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(ncells), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 4};
    const cuuint32_t box[2] = {32u, static_cast<cuuint32_t>(qsa::kGemmTokens)};
    const cuuint32_t estr[2] = {1u, 1u};
    const CUresult cr = encode(&tout, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, scores, dims, strides, box, estr,
                               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                               CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr != CUDA_SUCCESS) return fail(QSA_ERR_CUDA, "tensor map of the scores: error %d", static_cast<int>(cr));
  }
  qsa::GemmArgs a;
  a.iw = iw;
  a.scores = scores;
  a.ld = ld;
  a.T = rows;
  a.ncells = ncells;
  a.status = device_status();
  const int items = ((rows + qsa::kGemmTokens - 1) / qsa::kGemmTokens) *
                    ((ncells + qsa::kGemmCells - 1) / qsa::kGemmCells);
  const dim3 grid(std::max(1, std::min(items, sm_count())));
  return launched("score_gemm_kernel", launch_pdl(qsa::score_gemm_kernel, grid, dim3(qsa::kGemmThreads),
                                                  qsa::kGemmSmemRequest, s, tkey, tiq, tout, a));
}

// Rows <= 8 only: the scores of the decode GEMV, which also appends the `append`
// cells (at ncells - rows .. ncells - 1) when given.
int launch_index_gemv(const qsa_cache* c, int rows, int ncells, const uint16_t* iq, const float* iw,
                      float* scores, int64_t ld, const qsa_new_cells* append, cudaStream_t s) {
  qsa::ScoreAppend app = {};
  if (append) {
    app.k = append->k;
    app.v = append->v;
    app.key = reinterpret_cast<const __half*>(append->idx_key);
    app.kc = c->k;
    app.vc = c->v;
    app.ks = reinterpret_cast<__half*>(c->ks);
    app.vs = reinterpret_cast<__half*>(c->vs);
    app.idx_key = reinterpret_cast<__half*>(c->idx_key);
    app.from = ncells - rows;
    app.n = rows;
  }
  const int score_ctas = qsa::score_ctas_for(ncells, sm_count());
  const dim3 grid(score_ctas + 4 * app.n, (rows + qsa::kScoreRowsPerCta - 1) / qsa::kScoreRowsPerCta);
  return launched("index_score_kernel",
                  launch_pdl(qsa::index_score_kernel, grid, dim3(128), 0, s,
                             reinterpret_cast<const __half*>(c->idx_key), ncells,
                             reinterpret_cast<const __half*>(iq), iw, rows, scores, ld, app, score_ctas));
}

int launch_index_score(const qsa_cache* c, int rows, int ncells, const uint16_t* iq,
                       const float* iw, float* scores, int64_t ld, cudaStream_t s) {
  if (rows > qsa::kScoreRowsPerCta) return launch_score_gemm(c, rows, ncells, iq, iw, scores, ld, s);
  return launch_index_gemv(c, rows, ncells, iq, iw, scores, ld, nullptr, s);
}

int launch_zero(void* ws, const TopkPlan& p, cudaStream_t s) {
  // hist and ctr are adjacent up to alignment padding; zero both regions.
  const int64_t nzero = static_cast<int64_t>((p.sure - p.hist) / 4);
  const int zblocks = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(592, (nzero + 255) / 256)));
  return launched("topk_zero_kernel",
                  launch_pdl(qsa::topk_zero_kernel, dim3(zblocks), dim3(256), 0, s,
                             reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + p.hist), nzero));
}

int launch_filter_final(const float* scores, int64_t ld, int rows, int vis0, int top_k,
                        const qsa::TopkWs& w, int32_t* ids, cudaStream_t s) {
  const int vmax = vis0 + rows - 1;
  const dim3 grid((vmax + qsa::kTopkChunk - 1) / qsa::kTopkChunk, rows);
  int r = launched("topk_filter_kernel", launch_pdl(qsa::topk_filter_kernel, grid, dim3(qsa::kTopkThreads), 0,
                                                    s, scores, ld, vis0, top_k, w));
  if (r) return r;
  const int win = std::min(qsa::kMaxWindowBits, static_cast<int>(align_up(vmax, 32)));
  const size_t smem = 2 * static_cast<size_t>(win / 32) * 4;
  return launched("topk_final_kernel", launch_pdl(qsa::topk_final_kernel, dim3(rows), dim3(qsa::kFinalThreads),
                                                  smem, s, scores, ld, vis0, top_k, w, win, ids));
}

// Selection over given scores: zero, histogram (+ thresholds), filter, final.
int launch_topk(const float* scores, int64_t ld, int rows, int vis0, int top_k, void* ws,
                const TopkPlan& p, int32_t* ids, cudaStream_t s) {
  const qsa::TopkWs w = topk_ws(ws, p);
  const int vmax = vis0 + rows - 1;
  int r = launch_zero(ws, p, s);
  if (r) return r;
  const dim3 grid((vmax + qsa::kTopkChunk - 1) / qsa::kTopkChunk, rows);
  if ((r = launched("topk_hist_kernel", launch_pdl(qsa::topk_hist_kernel, grid, dim3(qsa::kTopkThreads), 0, s,
                                                   scores, ld, vis0, top_k, w))))
    return r;
  return launch_filter_final(scores, ld, rows, vis0, top_k, w, ids, s);
}

// Selection by one C-CTA cluster per row (rows of at most C x 512 x PER cells).
template <int PER, int C>
int launch_cluster_select_per(const float* scores, int64_t ld, int rows, int vis0, int top_k,
                              int32_t* ids, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(C, rows);
  cfg.blockDim = dim3(qsa::kClusterThreads);
  cfg.dynamicSmemBytes = qsa::cluster_smem_bytes<PER, C>();
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return launched("cluster_select_kernel",
                  cudaLaunchKernelEx(&cfg, qsa::cluster_select_kernel<PER, C>, scores, ld, vis0, top_k, ids));
}

// Whether one 16-CTA cluster of the wide selection fits on the current device.
bool wide_cluster_fits() {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(qsa::kClusterCtasWide, 1);
  cfg.blockDim = dim3(qsa::kClusterThreads);
  cfg.dynamicSmemBytes = qsa::cluster_smem_bytes<32, qsa::kClusterCtasWide>();
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = qsa::kClusterCtasWide;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  const cudaError_t e =
      cudaOccupancyMaxActiveClusters(&n, qsa::cluster_select_kernel<32, qsa::kClusterCtasWide>, &cfg);
  if (e != cudaSuccess) cudaGetLastError();
  return e == cudaSuccess && n > 0;
}

// Longest rows the decode selection gives to one 8-CTA cluster (16 cells per thread) and
// to one 16-CTA cluster (32 cells per thread); longer rows go through the multi-kernel
// selection, which spreads them over more SMs.
constexpr int kClusterMaxCells = qsa::kClusterCtas * qsa::kClusterThreads * 16;
constexpr int kClusterWideMaxCells = qsa::kClusterCtasWide * qsa::kClusterThreads * 32;

int cur_dev() {
  int dev = 0;
  cudaGetDevice(&dev);
  return dev & 63;
}

// Rows of at most kClusterMaxCells cells (launch_selection sends longer ones elsewhere).
int launch_cluster_select(const float* scores, int64_t ld, int rows, int vis0, int top_k,
                          int32_t* ids, cudaStream_t s) {
  const int vmax = vis0 + rows - 1;
  const int per_cta = qsa::kClusterCtas * qsa::kClusterThreads;
  const int need = (vmax + per_cta - 1) / per_cta;
  if (need <= 1) return launch_cluster_select_per<1, 8>(scores, ld, rows, vis0, top_k, ids, s);
  if (need <= 2) return launch_cluster_select_per<2, 8>(scores, ld, rows, vis0, top_k, ids, s);
  if (need <= 4) return launch_cluster_select_per<4, 8>(scores, ld, rows, vis0, top_k, ids, s);
  if (need <= 8) return launch_cluster_select_per<8, 8>(scores, ld, rows, vis0, top_k, ids, s);
  if (need <= 16) return launch_cluster_select_per<16, 8>(scores, ld, rows, vis0, top_k, ids, s);
  return launch_cluster_select_per<32, qsa::kClusterCtasWide>(scores, ld, rows, vis0, top_k, ids, s);
}

// The selection used by qsa_topk and the whole-step calls.  Decode-sized calls
// (a few rows, latency-bound) take one cluster per row; larger calls spread each
// row over many CTAs through the workspace, which keeps every SM busy.
int launch_selection(const float* scores, int64_t ld, int rows, int vis0, int top_k, void* ws,
                     const TopkPlan& p, int32_t* ids, cudaStream_t s) {
  const int vmax = vis0 + rows - 1;
  if (rows <= QSA_MAX_DECODE &&
      (vmax <= kClusterMaxCells || (vmax <= kClusterWideMaxCells && g_wide_cluster[cur_dev()])))
    return launch_cluster_select(scores, ld, rows, vis0, top_k, ids, s);
  return launch_topk(scores, ld, rows, vis0, top_k, ws, p, ids, s);
}

// ids == NULL: every row's list is all its visible cells (row r sees dense_vis0 + r <= top_k),
// copied to ids_fill when that is not NULL.
int launch_attn(const qsa_cache* c, int rows, const float* q, const int32_t* ids, int top_k,
                int nsplit, float scale, const float* gate, float* part, float* out, cudaStream_t s,
                int dense_vis0 = 0, int32_t* ids_fill = nullptr) {
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
  a.gate = gate;
  a.dense_vis0 = dense_vis0;
  a.ids_fill = ids_fill;
  const dim3 grid(nsplit, QSA_HKV, rows);
  cudaError_t e;
  if (rows <= QSA_MAX_DECODE) {
    if (ids) e = launch_pdl(qsa::attn_kernel<4, false>, grid, dim3(128), sizeof(qsa::AttnSmem<4>), s, a);
    else e = launch_pdl(qsa::attn_kernel<4, true>, grid, dim3(128), sizeof(qsa::AttnSmem<4>), s, a);
  } else {
    if (ids) e = launch_pdl(qsa::attn_kernel<2, false>, grid, dim3(64), sizeof(qsa::AttnSmem<2>), s, a);
    else e = launch_pdl(qsa::attn_kernel<2, true>, grid, dim3(64), sizeof(qsa::AttnSmem<2>), s, a);
  }
  return launched("attn_kernel", e);
}

int launch_merge(const float* part, int rows, int nsplit, const float* gate, float* out, cudaStream_t s) {
  return launched("merge_kernel", launch_pdl(qsa::merge_kernel, dim3(rows * QSA_HQ), dim3(256), 0, s, part,
                                             nsplit, gate, out));
}

int launch_cache_write(const qsa_cache* c, int pos0, int n, const float* k, const float* v,
                       const uint16_t* idx_key, cudaStream_t s) {
  return launched("cache_write_kernel",
                  launch_pdl(qsa::cache_write_kernel, dim3(n, QSA_HKV, 2), dim3(256), 0, s, c->k, c->v,
                             reinterpret_cast<__half*>(c->ks), reinterpret_cast<__half*>(c->vs),
                             reinterpret_cast<__half*>(c->idx_key), pos0, k, v,
                             reinterpret_cast<const __half*>(idx_key)));
}

// Scores and selection of a prompt chunk of more than 8 rows without a score matrix:
// thresholds from a sample, the candidate GEMM, the exact selection per row.
int launch_prefill_select(const qsa_cache* c, int rows, int vis0, int ncells, const uint16_t* iq,
                          const float* iw, int top_k, char* ws, const PrefillPlan& p, int32_t* ids,
                          cudaStream_t s) {
  PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  int r = tensor_map_encoder(&encode);
  if (r) return r;
  CUtensorMap tkey, tq;
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(QSA_DI), static_cast<cuuint64_t>(ncells)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(QSA_DI) * 2};
    const cuuint32_t box[2] = {64u, static_cast<cuuint32_t>(qsa::kSsCells)};
    const cuuint32_t estr[2] = {1u, 1u};
    const CUresult cr = encode(&tkey, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, c->idx_key, dims, strides, box, estr,
                               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr != CUDA_SUCCESS) return fail(QSA_ERR_CUDA, "tensor map of the keys: error %d", static_cast<int>(cr));
  }
  {
    // the queries as (token, head) rows of 64: [rows * 4][64]
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(QSA_DI), static_cast<cuuint64_t>(rows) * QSA_HI};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(QSA_DI) * 2};
    const cuuint32_t box[2] = {64u, static_cast<cuuint32_t>(qsa::kSsN)};
    const cuuint32_t estr[2] = {1u, 1u};
    const CUresult cr = encode(&tq, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<uint16_t*>(iq), dims, strides,
                               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr != CUDA_SUCCESS) return fail(QSA_ERR_CUDA, "tensor map of the queries: error %d", static_cast<int>(cr));
  }
  qsa::PrefillSel a;
  a.keys = reinterpret_cast<const __half*>(c->idx_key);
  a.iq = reinterpret_cast<const __half*>(iq);
  a.iw = iw;
  a.T = rows;
  a.vis0 = vis0;
  a.top_k = top_k;
  a.ncells = ncells;
  a.thr = reinterpret_cast<float*>(ws + p.thr);
  a.cand = reinterpret_cast<uint2*>(ws + p.cand);
  a.seg_count = reinterpret_cast<uint32_t*>(ws + p.count);
  a.n_ct = p.n_ct;
  a.items = p.items;
  a.grid = std::min(prefill_grid(p.items, p.n_ct, sm_count()), p.grid_max);
  a.per = (p.items + a.grid - 1) / a.grid;
  a.status = device_status();
  if ((r = launched("prefill_threshold_kernel",
                    launch_pdl(qsa::prefill_threshold_kernel, dim3((rows + 7) / 8), dim3(qsa::kPsThreads),
                               qsa::kScoreRowsPerCta * qsa::kBins * 4, s, a))))
    return r;
  if ((r = launched("score_select_kernel", launch_pdl(qsa::score_select_kernel, dim3(a.grid), dim3(qsa::kSsThreads),
                                                      qsa::kSsSmemBytes, s, tkey, tq, a))))
    return r;
  return launched("prefill_final_kernel", launch_pdl(qsa::prefill_final_kernel, dim3(rows), dim3(qsa::kPfThreads),
                                                     qsa::kPfSmemBytes, s, a, ids));
}

// The whole step for `rows` query rows; row r sees vis0 + r cells of ncells.  With
// `append`, the rows' own cells (the last `rows` cells, ncells - rows .. ncells - 1)
// are written first.
int run_step(const qsa_cache* c, int rows, int vis0, int ncells, const qsa_new_cells* append,
             const float* q, const uint16_t* iq, const float* iw, const float* gate, int top_k,
             int nsplit, float scale, void* ws, size_t ws_bytes, float* out, int32_t* ids_out,
             cudaStream_t s) {
  if (!q || !iq || !iw || !out) return fail(QSA_ERR_ARG, "q, iq, iw and out must not be NULL");
  if (append && (!append->k || !append->v || !append->idx_key))
    return fail(QSA_ERR_ARG, "append has a NULL array");
  if (!ws) return fail(QSA_ERR_WORKSPACE, "workspace is NULL");
  if (!aligned16(q) || !aligned16(iq) || !aligned16(iw) || !aligned16(out) || !aligned16(ws) ||
      (ids_out && !aligned16(ids_out)) || (gate && !aligned16(gate)))
    return fail(QSA_ERR_ARG, "q, iq, iw, gate, out, ids_out and ws must be 16-byte aligned");
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
  // The decode GEMV appends the new cells itself (one launch less); the dense path and the
  // prompt GEMM take them from a cache-write launch first.
  const bool gemv = rows <= qsa::kScoreRowsPerCta && vmax > top_k;
  if (append && !gemv &&
      (r = launch_cache_write(c, ncells - rows, rows, append->k, append->v, append->idx_key, s)))
    return r;
  if (vmax <= top_k) {
    // Every row sees at most top_k cells, so the selection would keep all of them in
    // order: no scores, no selection; the attention walks cells 0 .. V - 1 itself.
    if ((r = launch_attn(c, rows, q, nullptr, top_k, nsplit, scale, gate, part, out, s, vis0, ids_out)))
      return r;
  } else if (p.prefill_select) {
    if ((r = launch_prefill_select(c, rows, vis0, ncells, iq, iw, top_k, base, p.pre, ids, s))) return r;
    if ((r = launch_attn(c, rows, q, ids, top_k, nsplit, scale, gate, part, out, s))) return r;
  } else {
    if (gemv) r = launch_index_gemv(c, rows, ncells, iq, iw, scores, p.ld, append, s);
    else r = launch_index_score(c, rows, ncells, iq, iw, scores, p.ld, s);
    if (r) return r;
    if ((r = launch_selection(scores, p.ld, rows, vis0, top_k, base, p.topk, ids, s))) return r;
    if ((r = launch_attn(c, rows, q, ids, top_k, nsplit, scale, gate, part, out, s))) return r;
  }
  if (nsplit > 1 && (r = launch_merge(part, rows, nsplit, gate, out, s))) return r;
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
  if (n > QSA_MAX_ROWS) return fail(QSA_ERR_ARG, "n = %d above %d", n, QSA_MAX_ROWS);
  if ((r = launch_cache_write(cache, pos0, n, k, v, idx_key, static_cast<cudaStream_t>(stream)))) return r;
  return ok();
}

int qsa_decode(const qsa_cache* cache, int L, int n, const qsa_new_cells* append, const float* q,
               const uint16_t* iq, const float* iw, const float* gate, int top_k, int nsplit,
               float scale, void* ws, size_t ws_bytes, float* out, int32_t* ids_out, void* stream) {
  int r = check_cache(cache);
  if (r) return r;
  if (n < 1 || n > QSA_MAX_DECODE) return fail(QSA_ERR_ARG, "n = %d outside [1, 8]", n);
  if (L < n || L > cache->max_cells)
    return fail(QSA_ERR_ARG, "L = %d outside [n, max_cells = %d]", L, cache->max_cells);
  if (top_k < 1 || top_k > QSA_MAX_TOPK) return fail(QSA_ERR_ARG, "top_k = %d out of range", top_k);
  if (nsplit < 0 || nsplit > QSA_MAX_SPLITS) return fail(QSA_ERR_ARG, "nsplit = %d out of range", nsplit);
  const int ns = nsplit ? nsplit : auto_nsplit(n, top_k);
  return run_step(cache, n, L - n + 1, L, append, q, iq, iw, gate, top_k, ns, scale, ws, ws_bytes, out,
                  ids_out, static_cast<cudaStream_t>(stream));
}

int qsa_prefill_chunk(const qsa_cache* cache, int pos0, int T, const qsa_new_cells* append,
                      const float* q, const uint16_t* iq, const float* iw, const float* gate,
                      int top_k, float scale, void* ws, size_t ws_bytes, float* out,
                      int32_t* ids_out, void* stream) {
  int r = check_cache(cache);
  if (r) return r;
  if (T < 1 || pos0 < 0 || static_cast<int64_t>(pos0) + T > cache->max_cells)
    return fail(QSA_ERR_ARG, "chunk [%d, %d + %d) outside the cache of %d", pos0, pos0, T,
                cache->max_cells);
  if (T > QSA_MAX_ROWS) return fail(QSA_ERR_ARG, "T = %d above %d rows", T, QSA_MAX_ROWS);
  if (top_k < 1 || top_k > QSA_MAX_TOPK) return fail(QSA_ERR_ARG, "top_k = %d out of range", top_k);
  const int ns = auto_nsplit(T, top_k);
  return run_step(cache, T, pos0 + 1, pos0 + T, append, q, iq, iw, gate, top_k, ns, scale, ws, ws_bytes,
                  out, ids_out, static_cast<cudaStream_t>(stream));
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
  if ((r = prepare_device())) return r;
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
  if (rows < 1 || rows > QSA_MAX_ROWS || vis0 < 1 || top_k < 1 || top_k > QSA_MAX_TOPK)
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
  if ((r = launch_selection(scores, ld, rows, vis0, top_k, ws, p, ids, static_cast<cudaStream_t>(stream))))
    return r;
  return ok();
}

int qsa_attn(const qsa_cache* cache, int rows, const float* q, const int32_t* ids, int top_k,
             int nsplit, float scale, const float* gate, float* part, float* out, void* stream) {
  int r = check_cache(cache);
  if (r) return r;
  if (!q || !ids) return fail(QSA_ERR_ARG, "q and ids must not be NULL");
  if (rows < 1 || rows > QSA_MAX_ROWS || top_k < 1 || top_k > QSA_MAX_TOPK || nsplit < 1 ||
      nsplit > QSA_MAX_SPLITS)
    return fail(QSA_ERR_ARG, "rows = %d, top_k = %d, nsplit = %d out of range", rows, top_k, nsplit);
  if (nsplit == 1 && !out) return fail(QSA_ERR_ARG, "nsplit == 1 needs out");
  if (nsplit > 1 && !part) return fail(QSA_ERR_ARG, "nsplit > 1 needs part");
  if (!aligned16(q) || (out && !aligned16(out)) || (part && !aligned16(part)) || (gate && !aligned16(gate)))
    return fail(QSA_ERR_ARG, "q, gate, part and out must be 16-byte aligned");
  if ((r = prepare_device())) return r;
  if ((r = launch_attn(cache, rows, q, ids, top_k, nsplit, scale, nsplit == 1 ? gate : nullptr, part, out,
                       static_cast<cudaStream_t>(stream))))
    return r;
  return ok();
}

int qsa_merge(const float* part, int rows, int nsplit, const float* gate, float* out, void* stream) {
  if (!part || !out) return fail(QSA_ERR_ARG, "part and out must not be NULL");
  if (rows < 1 || rows > QSA_MAX_ROWS || nsplit < 1 || nsplit > QSA_MAX_SPLITS)
    return fail(QSA_ERR_ARG, "rows = %d, nsplit = %d out of range", rows, nsplit);
  int r = launch_merge(part, rows, nsplit, gate, out, static_cast<cudaStream_t>(stream));
  if (r) return r;
  return ok();
}

int qsa_device_status(int* status, void* stream) {
  if (!status) return fail(QSA_ERR_ARG, "status must not be NULL");
  int r = prepare_device();
  if (r) return r;
  uint32_t* addr = device_status();
  uint32_t host = 0u;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(&host, addr, sizeof(host), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = cudaMemsetAsync(addr, 0, sizeof(uint32_t), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return fail(QSA_ERR_CUDA, "reading the device status: %s", cudaGetErrorString(e));
  *status = static_cast<int>(host);
  return ok();
}

int qsa_selftest_wait_timeout(void* stream) {
  int r = prepare_device();
  if (r) return r;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1);
  cfg.blockDim = dim3(32);
  cfg.stream = static_cast<cudaStream_t>(stream);
  if ((r = launched("wait_selftest_kernel", cudaLaunchKernelEx(&cfg, qsa::wait_selftest_kernel, device_status()))))
    return r;
  return ok();
}

int qsa_trace_begin(int capacity, void* stream) {
  if (capacity < 1 || capacity > 4096) return fail(QSA_ERR_ARG, "trace capacity %d outside [1, 4096]", capacity);
  Trace& t = g_trace;
  while (static_cast<int>(t.ev.size()) < capacity + 1) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) {
      cudaGetLastError();
      return fail(QSA_ERR_CUDA, "cudaEventCreate failed");
    }
    t.ev.push_back(e);
  }
  t.names.assign(t.ev.size(), nullptr);
  t.stream = static_cast<cudaStream_t>(stream);
  t.n = 0;
  if (cudaEventRecord(t.ev[0], t.stream) != cudaSuccess) {
    cudaGetLastError();
    return fail(QSA_ERR_CUDA, "cudaEventRecord failed");
  }
  t.on = true;
  return ok();
}

int qsa_trace_end(int cap, int* n, float* ms, const char** names) {
  Trace& t = g_trace;
  if (!t.on) return fail(QSA_ERR_ARG, "no trace was begun on this thread");
  t.on = false;
  if (!n) return fail(QSA_ERR_ARG, "n must not be NULL");
  *n = t.n;
  if (t.n == 0) return ok();
  if (cudaEventSynchronize(t.ev[t.n]) != cudaSuccess) {
    cudaGetLastError();
    return fail(QSA_ERR_CUDA, "cudaEventSynchronize failed");
  }
  for (int i = 0; i < t.n && i < cap; ++i) {
    if (ms && cudaEventElapsedTime(&ms[i], t.ev[i], t.ev[i + 1]) != cudaSuccess) {
      cudaGetLastError();
      return fail(QSA_ERR_CUDA, "cudaEventElapsedTime failed");
    }
    if (names) names[i] = t.names[i];
  }
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
