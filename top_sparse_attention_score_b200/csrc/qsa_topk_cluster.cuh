// qsa_topk_cluster.cuh -- the selection of one row by one thread-block cluster.
//
// Same result as qsa_topk.cuh (the top_k cells of largest score, equal scores to
// the lower index, ascending ids; qsa_topk of "opus r15 track A: prompt_chunk wave
// zipping, ...", what changed, item 1), organised around Blackwell's clusters:
//
//   * a cluster of 8 CTAs x 512 threads owns one row; CTA r holds the scores of
//     cells [r * chunk, (r + 1) * chunk) in registers, read once from L2/HBM;
//   * the 2048-bin coarse histogram (fp16-key bins, as in qsa_topk.cuh) is built
//     in each CTA's shared memory and reduced across the cluster through
//     distributed shared memory: CTA r sums bin slice r of all eight, then every
//     CTA finds the threshold bin from the eight slice totals;
//   * four 8-bit radix passes over the threshold bin's full 32-bit keys find the
//     exact k-th key; each pass is one cluster barrier (per-CTA 256-bin counts,
//     double-buffered, summed by every CTA);
//   * each CTA marks its selected cells (and the lowest-index ties) in a bitmap
//     of its own contiguous range and writes them in ascending order at an
//     offset summed from the other CTAs' counts.
// No global atomics, no counters to clear, no candidate lists: only hardware
// cluster barriers (which need no timeout: every CTA of a cluster is resident).
#pragma once

#include <cooperative_groups.h>

#include "qsa_common.cuh"

namespace qsa {

constexpr int kClusterCtas = 8;
constexpr int kClusterThreads = 512;
constexpr int kClusterSlice = kBins / kClusterCtas;  // 256 bins reduced by each CTA

// Scores per thread held in registers up to this many; beyond, in shared memory.
constexpr int kClusterRegPer = 32;

// grid (8, rows), cluster (8, 1, 1), block 512.  PER scores per thread: the
// cluster covers 8 * 512 * PER cells, at least the longest row.  For PER above
// kClusterRegPer the CTA's scores live in dynamic shared memory (PER * 512 floats).
template <int PER>
__global__ void __launch_bounds__(kClusterThreads) cluster_select_kernel(const float* __restrict__ scores,
                                                                         int64_t ld, int vis0, int top_k,
                                                                         int32_t* __restrict__ ids) {
  namespace cg = cooperative_groups;
  constexpr bool kInSmem = PER > kClusterRegPer;
  extern __shared__ float sv[];
  constexpr int NT = kClusterThreads;
  constexpr int CHUNK = NT * PER;
  constexpr int WORDS = CHUNK / 32;
  __shared__ uint32_t hist[kBins];
  __shared__ uint32_t slice[kClusterSlice];
  __shared__ uint32_t radix[2][256];
  __shared__ uint32_t tmp256[256];
  __shared__ uint32_t selb[WORDS];
  __shared__ uint32_t eqb[WORDS];
  __shared__ uint32_t slice_total;
  __shared__ uint32_t counts[2];  // published: selected cells without ties, cells tied at the threshold
  __shared__ uint32_t tots[kClusterCtas];
  __shared__ uint32_t scratch[33];
  __shared__ uint32_t result[2];

  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int tid = threadIdx.x;
  griddep_launch();
  griddep_wait();
  const int row = blockIdx.y;
  const int V = vis0 + row;
  int32_t* out = ids + static_cast<size_t>(row) * top_k;
  if (V <= top_k) {  // every visible cell, ascending (the whole cluster leaves together)
    if (rank == 0)
      for (int i = tid; i < top_k; i += NT) out[i] = i < V ? i : -1;
    return;
  }
  const int c0 = rank * CHUNK;
  const float* s = scores + row * ld;

  // ---- scores of this CTA's cells (element e of thread t is cell c0 + e * NT + t)
  float v[kInSmem ? 1 : PER];
#define QSA_SCORE(e) (kInSmem ? sv[(e) * NT + tid] : v[kInSmem ? 0 : (e)])
#pragma unroll
  for (int e = 0; e < PER; ++e) {
    const int c = c0 + e * NT + tid;
    const float x = c < V ? __ldcg(s + c) : 0.f;
    if constexpr (kInSmem) sv[e * NT + tid] = x;
    else v[e] = x;
  }
  for (int i = tid; i < kBins; i += NT) hist[i] = 0u;
  if (tid == 0) slice_total = 0u;
  __syncthreads();
#pragma unroll
  for (int e = 0; e < PER; ++e)
    if (c0 + e * NT + tid < V) atomicAdd(&hist[score_bin(QSA_SCORE(e))], 1u);
  cluster.sync();  // every CTA's histogram is complete

  // ---- reduce bin slice `rank` over the cluster; publish its total
  if (tid < kClusterSlice) {
    const int b = rank * kClusterSlice + tid;
    uint32_t sum = 0u;
#pragma unroll
    for (int q = 0; q < kClusterCtas; ++q) sum += cluster.map_shared_rank(hist, q)[b];
    slice[tid] = sum;
    atomicAdd(&slice_total, sum);
  }
  cluster.sync();  // slices and totals published

  // ---- threshold bin: slices from the highest (rank 7) down
  if (tid < kClusterCtas) tots[tid] = *cluster.map_shared_rank(&slice_total, tid);
  __syncthreads();
  uint32_t above = 0u;
  int qs = 0;
  for (int q = kClusterCtas - 1; q >= 0; --q) {
    if (above + tots[q] >= static_cast<uint32_t>(top_k)) {
      qs = q;
      break;
    }
    above += tots[q];
  }
  if (tid < kClusterSlice) tmp256[tid] = cluster.map_shared_rank(slice, qs)[tid];
  __syncthreads();
  uint32_t tb, above_in;
  find_threshold_bin<NT>(tmp256, kClusterSlice, static_cast<uint32_t>(top_k) - above, scratch, result, tb,
                         above_in);
  const uint32_t thr_bin = static_cast<uint32_t>(qs * kClusterSlice) + tb;
  above += above_in;

  // ---- exact threshold key among the cells of the threshold bin: 4 passes of 8 bits
  uint32_t need = static_cast<uint32_t>(top_k) - above;  // >= 1
  uint32_t prefix = 0u, mask = 0u;
#pragma unroll 1
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    uint32_t* h = radix[pass & 1];
    for (int i = tid; i < 256; i += NT) h[i] = 0u;
    __syncthreads();
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      if (c0 + e * NT + tid >= V || score_bin(QSA_SCORE(e)) != thr_bin) continue;
      const uint32_t key = score_key(QSA_SCORE(e));
      if ((key & mask) == prefix) atomicAdd(&h[(key >> shift) & 255u], 1u);
    }
    cluster.sync();  // this pass's counts are complete everywhere
    if (tid < 256) {
      uint32_t sum = 0u;
#pragma unroll
      for (int q = 0; q < kClusterCtas; ++q) sum += cluster.map_shared_rank(h, q)[tid];
      tmp256[tid] = sum;
    }
    __syncthreads();
    uint32_t digit, cnt_above;
    find_threshold_bin<NT>(tmp256, 256, need, scratch, result, digit, cnt_above);
    need -= cnt_above;
    prefix |= digit << shift;
    mask |= 255u << shift;
  }
  const uint32_t thr_key = prefix;
  const uint32_t take_eq = need;  // lowest-index cells with key == thr_key to keep

  // ---- mark this CTA's cells; publish its counts
  for (int i = tid; i < WORDS; i += NT) {
    selb[i] = 0u;
    eqb[i] = 0u;
  }
  __syncthreads();
#pragma unroll
  for (int e = 0; e < PER; ++e) {
    const int li = e * NT + tid;
    if (c0 + li >= V) continue;
    const uint32_t b = score_bin(QSA_SCORE(e));
    if (b < thr_bin) continue;
    const uint32_t key = score_key(QSA_SCORE(e));
    if (b > thr_bin || key > thr_key) atomicOr(&selb[li >> 5], 1u << (li & 31));
    else if (key == thr_key) atomicOr(&eqb[li >> 5], 1u << (li & 31));
  }
  __syncthreads();
  const int per = (WORDS + NT - 1) / NT;
  const int wb = tid * per, we = min(WORDS, wb + per);
  uint32_t nsel = 0u, neq = 0u;
  for (int i = wb; i < we; ++i) {
    nsel += __popc(selb[i]);
    neq += __popc(eqb[i]);
  }
  uint32_t tot_sel, tot_eq;
  const uint32_t sel_rank = block_exclusive_scan<NT>(nsel, scratch, tot_sel);
  const uint32_t eq_rank = block_exclusive_scan<NT>(neq, scratch, tot_eq);
  if (tid == 0) {
    counts[0] = tot_sel;
    counts[1] = tot_eq;
  }
  cluster.sync();  // counts published

  // ---- offsets from the lower-ranked CTAs; ties go to the lowest indices first
  uint32_t eq_before = 0u, out_before = 0u;
  for (int q = 0; q < rank; ++q) {
    const uint32_t* cq = cluster.map_shared_rank(counts, q);
    const uint32_t qsel = cq[0], qeq = cq[1];
    const uint32_t qtake = eq_before >= take_eq ? 0u : min(qeq, take_eq - eq_before);
    out_before += qsel + qtake;
    eq_before += qeq;
  }
  uint32_t my_take = eq_before >= take_eq ? 0u : min(tot_eq, take_eq - eq_before);
  // my eq bits in ascending order: keep the first my_take
  uint32_t r = eq_rank;
  for (int i = wb; i < we && r < my_take; ++i) {
    uint32_t b = eqb[i];
    while (b && r < my_take) {
      const uint32_t low = b & (0u - b);
      selb[i] |= low;
      b ^= low;
      ++r;
    }
  }
  // ties kept by earlier threads shift this thread's output position
  const uint32_t tie_before = min(eq_rank, my_take);
  uint32_t pos = out_before + sel_rank + tie_before;
  for (int i = wb; i < we; ++i) {
    uint32_t b = selb[i];
    while (b) {
      const int bit = __ffs(b) - 1;
      b &= b - 1u;
      if (pos < static_cast<uint32_t>(top_k)) out[pos] = c0 + i * 32 + bit;
      ++pos;
    }
  }
  cluster.sync();  // no CTA leaves while another may still read its shared memory
#undef QSA_SCORE
}

}  // namespace qsa
