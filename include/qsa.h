/*
 * qsa.h -- C ABI of the QSA sparse-attention step for NVIDIA B200 (sm_100a).
 *
 * The step, for each query token of a decoder layer:
 *   1. an indexer scores every cached cell the token can see,
 *   2. a top-k picks the cells to attend (one id set per token, shared by all heads),
 *   3. attention runs over only those cells of an int8 K/V cache with fp16 scales,
 *   4. partial results of context splits are merged by log-sum-exp.
 * The pages this library follows describe the same step as Metal kernels
 * (qsa_score_mm, qsa_topk, qsa_attn, qsa_merge): "opus r20 track A: MTP map
 * mlock + qsa_attn / qsa_merge decode tweaks" (sections 2-4) and "opus r15
 * track A: prompt_chunk wave zipping, fused alpha|beta GEMM, QSA PSO
 * pre-warm, 24 GB chunk 2048" (what changed, item 1).  The pages print no
 * formula for the indexer or the quantizer; the forms below are the plainest
 * reading of the workload they describe.
 *
 * Fixed shapes: 24 query heads x 256, 2 KV heads x 256 (query head h uses KV
 * head h / 12), one fp16 scale per 32 int8 values, an indexer of 4 heads x 64
 * in fp16 ("Round 5 Track C Report: Direct FP16 qcurh in qsa_prep + PromptGemm
 * Dead Buffer Removal & Layer-Local Aliasing", section 1: qcur rows of 24 x 256,
 * kcur/vcur rows of 512 floats per token, a 2051-word qids row per token).
 *
 * Conventions for every call:
 *   - Pointers are CUDA device pointers owned by the caller unless stated.
 *     The library never allocates, frees or synchronises, and keeps no state
 *     between calls apart from the launch counter, the last error string and
 *     the fixed scratch buffer of qsa_topk_static.
 *   - fp16 values travel as their IEEE binary16 bit patterns (uint16_t).
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream); every call
 *     only enqueues kernels on it and returns.  Results are ready when the
 *     stream reaches them.
 *   - Return codes: QSA_OK, or QSA_ERR_ARG (bad argument: nothing launched),
 *     QSA_ERR_WORKSPACE (workspace too small: nothing launched), QSA_ERR_CUDA
 *     (a launch failed; qsa_last_error() says which).  QSA_ERR_TIMEOUT is
 *     reported through qsa_device_status: the calls are asynchronous, so a
 *     kernel's bounded wait that expires cannot return it directly.
 *   - Arrays must be 16-byte aligned (cudaMalloc and torch allocations are).
 *   - Non-finite inputs (NaN, inf) give unspecified results.
 */
#ifndef QSA_B200_QSA_H_
#define QSA_B200_QSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define QSA_HQ 24           /* query heads */
#define QSA_D 256           /* head dim */
#define QSA_HKV 2           /* KV heads */
#define QSA_GROUP 32        /* int8 values per fp16 scale */
#define QSA_NG 8            /* scale groups per head row */
#define QSA_HI 4            /* indexer heads */
#define QSA_DI 64           /* indexer dim */
#define QSA_MAX_DECODE 8    /* decode tokens per call (MTP draft) */
#define QSA_MAX_SPLITS 64   /* context splits merged by log-sum-exp */
#define QSA_MAX_TOPK 16384  /* largest top_k */
#define QSA_MAX_CELLS (1 << 24)
#define QSA_MAX_ROWS 65535  /* query rows of one prefill, qsa_topk or qsa_attn call */
#define QSA_PART_STRIDE (2 + QSA_D) /* floats per partial: m, l, o[256] */

enum {
  QSA_OK = 0,
  QSA_ERR_ARG = 1,
  QSA_ERR_WORKSPACE = 2,
  QSA_ERR_CUDA = 3,
  QSA_ERR_TIMEOUT = 4
};

enum { QSA_MODE_DECODE = 0, QSA_MODE_PREFILL = 1 };

/*
 * The cell cache ("random int8 KV, fp16 scales": "opus r20 track A ...",
 * section 3).  Cell c holds, for KV head g:
 *   k[c][g][0..256), v[c][g][0..256)   int8 codes
 *   ks[c][g][0..8),  vs[c][g][0..8)    fp16 scales; value d of the row is
 *                                       code[d] * scale[d / 32]
 * and its indexer key idx_key[c][0..64) in fp16.  All five arrays are
 * caller-owned device memory of max_cells cells.
 */
typedef struct qsa_cache {
  int8_t* k;          /* [max_cells][2][256] */
  int8_t* v;          /* [max_cells][2][256] */
  uint16_t* ks;       /* [max_cells][2][8] fp16 */
  uint16_t* vs;       /* [max_cells][2][8] fp16 */
  uint16_t* idx_key;  /* [max_cells][64] fp16 */
  int32_t max_cells;
} qsa_cache;

/*
 * The call's own new cells (the write side of qsa_prep: "Round 5 Track C
 * Report ...", section 1, Targets 1-2, kcur / vcur rows of 2 x 256 floats per
 * token), appended by the step call itself before anything reads the cache:
 * qsa_decode writes its n tokens' cells at L - n .. L - 1, qsa_prefill_chunk
 * its T tokens' cells at pos0 .. pos0 + T - 1, exactly as qsa_cache_write
 * would (same quantizer, bit for bit).  One call then does what a cache
 * write followed by a step does, with one host crossing.  Caller-owned device
 * memory:
 *   k, v     fp32 [rows][2][256]
 *   idx_key  fp16 [rows][64]
 */
typedef struct qsa_new_cells {
  const float* k;
  const float* v;
  const uint16_t* idx_key;
} qsa_new_cells;

/*
 * Bytes of workspace qsa_decode (mode QSA_MODE_DECODE, rows = n, L = cache
 * length) or qsa_prefill_chunk (mode QSA_MODE_PREFILL, rows = T, L = pos0 + T)
 * needs for these sizes; nsplit as passed to the call (0 = automatic).
 * Returns 0 for invalid sizes.
 */
size_t qsa_workspace_bytes(int mode, int rows, int L, int top_k, int nsplit);

/*
 * Append n cells at pos0..pos0+n-1 (the write side of qsa_prep: "Round 5
 * Track C Report ...", section 1, Target 1-2, which produces kcur/vcur rows of
 * 2 x 256 floats per token).  Each group of 32 values of k / v
 * (fp32 [n][2][256]) is quantized as
 *   s = fp16_rn(max|x| / 127), saturated at 65504;
 *   code = clamp(rint(x / s), -127, 127) (half to even), all 0 when s == 0;
 * divisions and rounding in IEEE fp32.  idx_key (fp16 [n][64]) is copied.
 * Requires 0 <= pos0, 1 <= n, pos0 + n <= max_cells.
 */
int qsa_cache_write(const qsa_cache* cache, int pos0, int n, const float* k, const float* v,
                    const uint16_t* idx_key, void* stream);

/*
 * Decode step for n = 1..8 query tokens (the MTP draft of "opus r20 track A
 * ...", section 3, ntok 1..8).  Token i sees cells [0, L - n + 1 + i).
 *   append  the n tokens' own cells, written at L - n .. L - 1 first (see
 *           qsa_new_cells), or NULL when they are already in the cache
 *   q       fp32 [n][24][256]     query rows
 *   iq      fp16 [n][4][64]       indexer queries
 *   iw      fp32 [n][4]           indexer head weights
 *   gate    fp32 [n][24][256] or NULL: the output gate ("attention + gate",
 *           same page, section 3; the gate rows travel with the query rows,
 *           12288 floats per token of Q plus gate in "Round 5 Track C Report
 *           ...", section 1, Target 2): out = O * sigmoid(gate), elementwise,
 *           sigmoid(x) = 1 / (1 + exp(-x)); NULL leaves O ungated
 * Per token: score[c] = sum_h iw[h] * max(0, iq[h] . idx_key[c]) for every
 * visible c; the top_k cells of largest score (equal scores: lower index
 * first; all visible cells when fewer than top_k); then for head h
 *   s_c = scale * sum_d q[h][d] * K[c][h/12][d],  O[h] = softmax(s) . V[.][h/12]
 * over the selected cells, computed as nsplit pieces of the selected list
 * (ceil(top_k / nsplit) entries each) merged by log-sum-exp (qsa_merge,
 * same page, section 2).  nsplit = 0 lets the library choose; the result
 * does not depend on nsplit beyond rounding.  When every token sees at most
 * top_k cells (L <= top_k), all visible cells are selected: the call skips
 * the scores and the selection (the dense path for short contexts, the pages'
 * qsa_flash case) and returns the same result and ids.
 *   out      fp32 [n][24][256]
 *   ids_out  int32 [n][top_k] or NULL: the selected cells, ascending, -1 padded
 *   ws       device workspace of at least qsa_workspace_bytes(...) bytes
 * Requires 1 <= n <= 8, n <= L <= max_cells, 1 <= top_k <= QSA_MAX_TOPK,
 * 0 <= nsplit <= QSA_MAX_SPLITS.
 */
int qsa_decode(const qsa_cache* cache, int L, int n, const qsa_new_cells* append, const float* q,
               const uint16_t* iq, const float* iw, const float* gate, int top_k, int nsplit,
               float scale, void* ws, size_t ws_bytes, float* out, int32_t* ids_out, void* stream);

/*
 * Prefill step for a causal chunk of T tokens at pos0 (prompt_chunk with
 * qsa_score_mm, qsa_topk and the prompt attention: "opus r15 track A ...",
 * what changed, items 1-2; "Round 5 Track C Report ...", section 2.1).  Row t
 * sees cells [0, pos0 + t]; the chunk's own cells are written first from
 * `append`, or must already be in the cache when `append` is NULL.
 * Arguments as qsa_decode with n -> T (append rows [T], q [T][24][256],
 * iq [T][4][64], iw [T][4], gate [T][24][256] or NULL, out [T][24][256],
 * ids_out [T][top_k] or NULL).  A chunk with pos0 + T <= top_k takes the dense
 * path, as qsa_decode does.  The score GEMM of a chunk waits on mbarriers
 * (bounded): after the results are used, a caller that must know they are
 * sound checks qsa_device_status once.
 * Requires 0 <= pos0, 1 <= T <= QSA_MAX_ROWS, pos0 + T <= max_cells.
 */
int qsa_prefill_chunk(const qsa_cache* cache, int pos0, int T, const qsa_new_cells* append,
                      const float* q, const uint16_t* iq, const float* iw, const float* gate,
                      int top_k, float scale, void* ws, size_t ws_bytes, float* out,
                      int32_t* ids_out, void* stream);

/* ---- the four steps, one call each (used by the composite calls above) ---- */

/*
 * Step 1, indexer scores (qsa_score_mm; "opus r15 track A ...", item 1):
 * scores[r * ld + c] = sum_h iw[r][h] * max(0, sum_d iq[r][h][d] * idx_key[c][d])
 * for rows r < rows and cells c < ncells (fp16 products, fp32 accumulation).
 * Callers mask by visibility.  ld >= ncells, ld % 4 == 0, ncells <= max_cells.
 * More than 8 rows run the tcgen05 GEMM, whose bounded waits report through
 * qsa_device_status.
 */
int qsa_index_score(const qsa_cache* cache, int rows, int ncells, const uint16_t* iq,
                    const float* iw, float* scores, int64_t ld, void* stream);

/* Workspace bytes for qsa_topk over `rows` rows of at most L visible cells. */
size_t qsa_topk_workspace_bytes(int rows, int L, int top_k);

/*
 * Step 2, selection (qsa_topk; "opus r15 track A ...", item 1; one qids row
 * per token: "Round 5 Track C Report ...", section 1, Target 2).  Row r sees
 * scores[r * ld + c] for c < vis0 + r and gets the top_k cells of largest
 * score, equal scores going to the lower index, all visible cells when fewer
 * than top_k: ids[r][0..top_k) ascending, padded with -1.  The order is exact
 * on the fp32 values (radix select on order-preserving 32-bit keys; -0 == +0).
 * Requires 1 <= rows <= QSA_MAX_ROWS, vis0 >= 1, vis0 + rows - 1 <= ld, ld % 4 == 0.
 */
int qsa_topk(const float* scores, int64_t ld, int rows, int vis0, int top_k, void* ws,
             size_t ws_bytes, int32_t* ids, void* stream);

/*
 * Step 3, sparse attention (qsa_attn: "opus r20 track A ...", section 2).
 * For row r, head h, KV head g = h / 12, and piece j of the id list
 * ids[r][j*P .. min((j+1)*P, top_k)) with P = ceil(top_k / nsplit), entries
 * < 0 skipped:
 *   s_c = scale * sum_d q[r][h][d] * k[c][g][d] * ks[c][g][d/32]
 *   m = max_c s_c, l = sum_c exp(s_c - m), o = sum_c exp(s_c - m) * v[c][g][:] * vs[c][g][:/32]
 * nsplit == 1: out[r][h][:] = o / l (0 for an empty list), times sigmoid(gate[r][h][:])
 *              when gate (fp32 [rows][24][256]) is not NULL; part unused.
 * nsplit > 1:  part[((r * 24 + h) * nsplit + j) * 258 + {0, 1, 2..257}] = {m, l, o}
 *              (m = -inf, l = 0, o = 0 for an empty piece); out and gate unused.
 * Query and P are rounded to fp16 for the tensor cores; K/V codes are exact;
 * accumulation is fp32.  Requires 1 <= rows <= QSA_MAX_ROWS, 1 <= nsplit <= 64;
 * ids outside [0, max_cells) count as empty slots.
 */
int qsa_attn(const qsa_cache* cache, int rows, const float* q, const int32_t* ids, int top_k,
             int nsplit, float scale, const float* gate, float* part, float* out, void* stream);

/*
 * Step 4, log-sum-exp merge (qsa_merge: "opus r20 track A ...", section 2):
 * per row and head, M = max m_j over pieces with l_j > 0, e_j = exp(m_j - M),
 * L = sum_j l_j e_j and o = sum_j o_j e_j, out = o / L (0 when every piece is
 * empty), times sigmoid(gate[r][h][:]) when gate (fp32 [rows][24][256]) is not
 * NULL.  part as written by qsa_attn.
 */
int qsa_merge(const float* part, int rows, int nsplit, const float* gate, float* out, void* stream);

/*
 * Selection without a caller workspace.  The pages have no counterpart to this
 * call; it exists for callers that cannot allocate device memory when they need
 * a selection -- code running while a CUDA graph is being captured (an
 * allocation cannot be recorded into a graph), serving loops that must not pay
 * for an allocator call or its implicit device synchronisation, and runtimes
 * whose device memory is already fully owned by another allocator.
 *
 * It computes exactly what qsa_topk computes (same arguments, minus the
 * workspace), using a fixed scratch buffer of QSA_STATIC_SCRATCH_BYTES that
 * the library holds in global memory on every GPU that loads it, until the
 * process exits.  Limits: rows <= QSA_STATIC_MAX_ROWS and
 * top_k <= QSA_STATIC_MAX_TOPK; larger requests return QSA_ERR_ARG and
 * launch nothing.  It never allocates or frees memory.
 *
 * The first call on each device looks up the buffer's device address (with
 * that device current), so make that first call before any stream capture
 * that is to contain later calls.  All calls on a device share the one
 * buffer, and each call clears the parts that must start at zero: calls
 * that can run at the same time on the GPU (different streams, or threads
 * without ordering between them) race on it and must be serialised, for
 * example by issuing them on one stream.
 */
#define QSA_STATIC_MAX_ROWS 8
#define QSA_STATIC_MAX_TOPK 2048
#define QSA_STATIC_SCRATCH_BYTES 1183744
int qsa_topk_static(const float* scores, int64_t ld, int rows, int vis0, int top_k, int32_t* ids,
                    void* stream);

/*
 * Device-side failure report.  Kernels that wait on an mbarrier (the prefill
 * score GEMM) bound every wait to four seconds; on expiry they stop, drain their
 * copies, free their tensor memory and record QSA_ERR_TIMEOUT in a status word
 * of the current device.  This call copies that word into *status (QSA_OK or
 * QSA_ERR_TIMEOUT) and clears it.  Unlike the other calls it synchronises
 * `stream`.
 */
int qsa_device_status(int* status, void* stream);

/*
 * Self-test of that mechanism: enqueues one kernel that waits on a barrier
 * nothing completes; after about one second it gives up and records
 * QSA_ERR_TIMEOUT, which qsa_device_status then reports.  The context stays
 * usable.
 */
int qsa_selftest_wait_timeout(void* stream);

/*
 * Per-kernel timing of this thread's calls (the pages time each dispatch on the GPU:
 * "opus r20 track A ...", section 4).  qsa_trace_begin records a start event on
 * `stream`; until qsa_trace_end, every kernel this thread's calls launch is followed by
 * an event on that stream (so trace calls made on that stream; the events also end the
 * overlap of consecutive kernels, so the times are those of kernels run back to back).
 * qsa_trace_end stops tracing, waits for the last event (it synchronises) and returns
 * the number of launches in *n and, for the first min(*n, cap), the milliseconds from
 * the previous event in ms[i] and the kernel's name in names[i] (static strings; either
 * array may be NULL).  capacity: 1 .. 4096 launches; later ones are not timed.
 */
int qsa_trace_begin(int capacity, void* stream);
int qsa_trace_end(int cap, int* n, float* ms, const char** names);

/* Text of the last error on the calling thread ("" when none). */
const char* qsa_last_error(void);

/* Number of kernels this library has launched in this process. */
uint64_t qsa_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* QSA_B200_QSA_H_ */
