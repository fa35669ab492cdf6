// qsa_topk_cluster.cuh -- the selection of one row by one thread-block cluster.
//
// Same result as qsa_topk.cuh (the top_k cells of largest score, equal scores to
// the lower index, ascending ids; qsa_topk of "opus r15 track A: prompt_chunk wave
// zipping, ...", what changed, item 1), organised around Blackwell clusters for the
// latency of a decode step:
//
//   * a cluster of 8 CTAs x 512 threads (16 CTAs for rows of more than 65536
//     cells) owns one row; CTA r holds the order-
//     preserving keys of cells [r * chunk, (r + 1) * chunk), read once from L2/HBM,
//     and their coarse bins (the top 11 bits of the key of the score's fp16
//     rounding, so a higher bin always means a strictly larger score: 2048 bins,
//     whose summed histogram every CTA reads from all the others);
//   * each CTA counts its bins in shared memory (two 16-bit counts per word);
//     after one cluster barrier every CTA sums all eight through distributed
//     shared memory and finds the threshold bin itself;
//   * each CTA lists its cells in the threshold bin (typically one to two hundred
//     in the row); after a second barrier every CTA gathers all lists and one warp
//     finds the exact k-th key over the bits the candidates do not share: up to
//     1024 candidates held in registers, one bit per step, otherwise 8-bit digits
//     counted in shared memory; it derives every CTA's output offset from the
//     gathered lists;
//   * each CTA marks its selected cells (and the lowest-index ties) in a bitmap of
//     its own contiguous range and writes them in ascending order.  A split
//     arrive/wait cluster barrier keeps every CTA's shared memory alive until the
//     others finished reading it, without a final stall.
// If the candidates overflow the gather buffers, every CTA of the cluster takes
// the same slower path: the radix passes run distributed, one cluster barrier each.
// Only hardware cluster barriers synchronise (all CTAs of a cluster are
// co-resident): no global atomics, nothing to clear between calls.
#pragma once

#include <cooperative_groups.h>

#include "qsa_common.cuh"

namespace qsa {

constexpr int kClusterCtas = 8;         // CTAs per row up to 65536 cells
constexpr int kClusterCtasWide = 16;    // CTAs per row up to 262144 cells (a non-portable cluster size)
constexpr int kClusterThreads = 512;
constexpr int kClusterRegPer = 32;       // keys per thread (registers): rows of up to 16 x 512 x 32 cells
constexpr int kClusterBins = 2048;       // coarse bins of the cluster histogram (top 11 bits of score_key16)
static_assert(kClusterBins / 2 % kClusterThreads == 0, "the histogram sum gives every thread whole words");
constexpr int kClusterCandCap = 2048;    // candidates one CTA can list
constexpr int kClusterGatherCap = 4096;  // candidates a CTA can gather from the whole cluster

// One warp, 256 bins counted from the highest: the bin where the running count
// first reaches k, and the count strictly above it (returned in every lane).
__device__ __forceinline__ void warp_threshold_256(const uint32_t* h, uint32_t k, uint32_t& bin,
                                                   uint32_t& above) {
  const int lane = threadIdx.x & 31;
  const int hi = 255 - 8 * lane;
  uint32_t local = 0u;
#pragma unroll
  for (int i = 0; i < 8; ++i) local += h[hi - i];
  uint32_t incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const uint32_t before = incl - local;
  const uint32_t m = __ballot_sync(0xffffffffu, before < k && incl >= k);
  const int f = m ? __ffs(m) - 1 : 31;
  uint32_t b = 0u, ab = 0u;
  if (lane == f) {
    uint32_t run = before;
    for (int i = 0; i < 8; ++i) {
      const uint32_t c = h[hi - i];
      if (run + c >= k) {
        b = static_cast<uint32_t>(hi - i);
        ab = run;
        break;
      }
      run += c;
    }
  }
  bin = __shfl_sync(0xffffffffu, b, f);
  above = __shfl_sync(0xffffffffu, ab, f);
}

constexpr int kWarpSelSlots = 32;  // candidates per lane the register select holds (n <= 1024)

// One warp: the need-th largest of the n gathered candidate keys (1 <= need <= n
// <= 32 * S), decided one bit at a time from the highest bit the keys do not all
// share.  Lane l holds candidates l, l + 32, ... in S registers, the empty slots
// key 0; every step runs straight-line over all S slots (a branch per slot costs
// more than its compare) and subtracts the empty slots' matches in one go.  The
// search ends early once a single candidate is left on the prefix: its key is
// the answer.  Returns the key in `thr` and, in `take`, how many candidates
// equal to it are kept (need minus the candidates above it).  The candidates of
// CTA q are the gathered range [q_off[q], q_off[q + 1]); lanes q < C
// set q_sel[q] = q_sure[q] + (those above thr) and q_eq[q] = (those equal to
// thr) from per-slot ballot words staged in words[0, 64).
template <int S, int C>
__device__ __forceinline__ void warp_select_regs(const uint32_t* gkey, const uint32_t* q_off, uint32_t n,
                                                 uint32_t need, const uint32_t* q_sure, uint32_t* q_sel,
                                                 uint32_t* q_eq, uint32_t* words, uint32_t& thr, uint32_t& take) {
  constexpr uint32_t full = 0xffffffffu;
  const uint32_t lane = threadIdx.x & 31u;
  const uint32_t mine = n > lane ? (n - lane + 31u) >> 5 : 0u;  // slots holding a key in this lane
  const uint32_t empty = S - mine;
  uint32_t k[S];
  uint32_t k_and = full, k_or = 0u;
#pragma unroll
  for (int j = 0; j < S; ++j) {
    k[j] = static_cast<uint32_t>(j) < mine ? gkey[j * 32 + lane] : 0u;
    k_and &= static_cast<uint32_t>(j) < mine ? k[j] : full;
    k_or |= k[j];
  }
  k_and = __reduce_and_sync(full, k_and);
  k_or = __reduce_or_sync(full, k_or);
  uint32_t diff = k_and ^ k_or;  // bits on which the candidates differ
  uint32_t pf = k_and, mk = ~diff, nd = need, alive = n;
  while (diff) {
    const uint32_t bit = 0x80000000u >> __clz(diff);
    diff ^= bit;
    mk |= bit;
    const uint32_t want = pf | bit;
    uint32_t c0 = 0u, c1 = 0u;
#pragma unroll
    for (int j = 0; j < S; j += 2) {
      c0 += ((k[j] ^ want) & mk) == 0u ? 1u : 0u;
      if (j + 1 < S) c1 += ((k[j + 1] ^ want) & mk) == 0u ? 1u : 0u;
    }
    const uint32_t c = __reduce_add_sync(full, c0 + c1 - ((want & mk) == 0u ? empty : 0u));
    if (nd <= c) {  // the need-th largest has this bit set
      pf = want;
      alive = c;
    } else {  // all c are above it
      nd -= c;
      alive -= c;
    }
    if (alive == 1u) {  // the one candidate left on the prefix is the answer
      uint32_t key = 0u;
      bool hit = false;
#pragma unroll
      for (int j = 0; j < S; ++j) {
        const bool h = static_cast<uint32_t>(j) < mine && ((k[j] ^ pf) & mk) == 0u;
        key = h ? k[j] : key;
        hit = hit || h;
      }
      const uint32_t who = __ballot_sync(full, hit);
      pf = __shfl_sync(full, key, __ffs(who) - 1);
      break;
    }
  }
  uint32_t w_gt = 0u, w_eq = 0u;  // lane j: the ballot words of slot j
#pragma unroll
  for (int j = 0; j < S; ++j) {
    const uint32_t base = static_cast<uint32_t>(j) * 32u;
    const uint32_t valid = n >= base + 32u ? full : (n > base ? (1u << (n - base)) - 1u : 0u);
    const uint32_t g = __ballot_sync(full, k[j] > pf) & valid;
    const uint32_t e = __ballot_sync(full, k[j] == pf) & valid;
    w_gt = lane == static_cast<uint32_t>(j) ? g : w_gt;
    w_eq = lane == static_cast<uint32_t>(j) ? e : w_eq;
  }
  words[lane] = w_gt;
  words[32 + lane] = w_eq;
  __syncwarp();
  if (lane < static_cast<uint32_t>(C)) {
    const uint32_t a = q_off[lane], b = lane + 1u < static_cast<uint32_t>(C) ? q_off[lane + 1] : n;
    uint32_t cg = 0u, ce = 0u;
    for (uint32_t w = a >> 5; a < b && w <= (b - 1u) >> 5; ++w) {
      const uint32_t lo = max(a, w * 32u) - w * 32u, hi = min(b, w * 32u + 32u) - w * 32u;
      const uint32_t m = (hi == 32u ? full : (1u << hi) - 1u) & ~((1u << lo) - 1u);
      cg += __popc(words[w] & m);
      ce += __popc(words[32 + w] & m);
    }
    q_sel[lane] = q_sure[lane] + cg;
    q_eq[lane] = ce;
  }
  thr = pf;
  take = nd;
}

__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}

template <int PER, int C>
struct ClusterSmem {
  static constexpr int kWords = kClusterThreads * PER / 32;
  uint32_t hist[kClusterBins / 2];    // two 16-bit counts per word
  uint32_t tot[kClusterBins];
  uint2 cand[kClusterCandCap];        // (key, local index)
  uint32_t gkey[kClusterGatherCap];
  uint32_t gcell[kClusterGatherCap];  // q * chunk + local index
  uint32_t selb[kWords];
  uint32_t eqb[kWords];
  uint32_t radix[2][256];
  uint32_t tmp256[256];
  uint32_t pub[4];                    // published: sure count, candidate count, selected count, tie count
  uint32_t q_sure[C], q_cand[C], q_sel[C], q_eq[C];
  uint32_t q_off[C];
  uint32_t cand_n, sure_n, misc[4];
  uint32_t scratch[33];
  uint32_t result[2];
};

template <int PER, int C>
__host__ __device__ constexpr size_t cluster_smem_bytes() {
  return sizeof(ClusterSmem<PER, C>);
}

// The selection of row blockIdx.y by this CTA of its C-CTA cluster (512 threads, shared
// memory csm_raw of cluster_smem_bytes<PER, C>()): writes the row's ids.  On return every
// CTA of the cluster has finished reading this CTA's shared memory.
template <int PER, int C>
__device__ __forceinline__ void cluster_select_row(const float* __restrict__ scores, int64_t ld, int vis0,
                                                   int top_k, int32_t* __restrict__ ids, unsigned char* csm_raw) {
  namespace cg = cooperative_groups;
  static_assert(PER <= kClusterRegPer, "keys are held in registers");
  constexpr int NT = kClusterThreads;
  constexpr int CHUNK = NT * PER;
  constexpr int WORDS = CHUNK / 32;
  ClusterSmem<PER, C>& sm = *reinterpret_cast<ClusterSmem<PER, C>*>(csm_raw);

  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int tid = threadIdx.x;
  const int lane = tid & 31;
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

  // ---- keys of this CTA's cells (element e of thread t is cell c0 + e * NT + t)
  uint32_t key[PER];
  uint32_t binpk[(PER + 1) / 2];
#define QSA_KEY(e) (key[(e)])
#define QSA_BIN(e) ((binpk[(e) >> 1] >> (16 * ((e) & 1))) & 0xffffu)
  {
    float x[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      const int c = c0 + e * NT + tid;
      x[e] = c < V ? __ldcg(s + c) : 0.f;
    }
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      key[e] = score_key(x[e]);
      const uint32_t b = score_key16(x[e]) >> 5;
      if (e & 1) binpk[e >> 1] |= b << 16;
      else binpk[e >> 1] = b;
    }
  }
  for (int i = tid; i < kClusterBins / 2; i += NT) sm.hist[i] = 0u;
  if (tid == 0) {
    sm.cand_n = 0u;
    sm.sure_n = 0u;
  }
  __syncthreads();
#pragma unroll
  for (int e = 0; e < PER; ++e)
    if (c0 + e * NT + tid < V) {
      const uint32_t b = QSA_BIN(e);
      atomicAdd(&sm.hist[b >> 1], 1u << (16 * (b & 1)));  // at most 32768 cells per CTA: no carry
    }
  cluster.sync();  // (1) every CTA's histogram is complete

  // ---- every CTA: the row's histogram (remote words of every CTA) and threshold bin
#pragma unroll
  for (int i = 0; i < kClusterBins / 2 / NT; ++i) {
    const int wi = tid + i * NT;
    uint32_t w[C];
#pragma unroll
    for (int q = 0; q < C; ++q) w[q] = cluster.map_shared_rank(sm.hist, q)[wi];
    uint32_t lo = 0u, hi = 0u;
#pragma unroll
    for (int q = 0; q < C; ++q) {
      lo += w[q] & 0xffffu;
      hi += w[q] >> 16;
    }
    sm.tot[2 * wi] = lo;
    sm.tot[2 * wi + 1] = hi;
  }
  __syncthreads();
  uint32_t thr_bin, above;
  find_threshold_bin<NT>(sm.tot, kClusterBins, static_cast<uint32_t>(top_k), sm.scratch, sm.result, thr_bin,
                         above);

  // ---- count this CTA's cells above the threshold bin; list the ones in it
  // (straight-line: per-thread counts, a warp scan, one append per warp)
  uint32_t my_sure = 0u, my_cand = 0u;
#pragma unroll
  for (int e = 0; e < PER; ++e) {
    const uint32_t b = QSA_BIN(e);
    const bool valid = c0 + e * NT + tid < V;
    my_sure += (valid && b > thr_bin) ? 1u : 0u;
    my_cand += (valid && b == thr_bin) ? 1u : 0u;
  }
  {
    uint32_t incl = my_cand;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      incl += lane >= o ? y : 0u;
    }
    const uint32_t wtot = __shfl_sync(0xffffffffu, incl, 31);
    uint32_t base = 0u;
    if (lane == 31 && wtot) base = atomicAdd(&sm.cand_n, wtot);
    uint32_t slot = __shfl_sync(0xffffffffu, base, 31) + incl - my_cand;
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      const int li = e * NT + tid;
      const bool is_cand = c0 + li < V && QSA_BIN(e) == thr_bin;
      if (is_cand && slot < static_cast<uint32_t>(kClusterCandCap))
        sm.cand[slot] = make_uint2(QSA_KEY(e), static_cast<uint32_t>(li));
      slot += is_cand ? 1u : 0u;
    }
  }
  my_sure = __reduce_add_sync(0xffffffffu, my_sure);
  if (lane == 0) atomicAdd(&sm.sure_n, my_sure);
  __syncthreads();
  if (tid == 0) {
    sm.pub[0] = sm.sure_n;
    sm.pub[1] = sm.cand_n;
  }
  cluster.sync();  // (2) lists and counts published

  if (tid < C) {
    const uint32_t* p = cluster.map_shared_rank(sm.pub, tid);
    sm.q_sure[tid] = p[0];
    sm.q_cand[tid] = p[1];
  }
  __syncthreads();
  uint32_t total_cand = 0u;
  bool fast = true;
#pragma unroll
  for (int q = 0; q < C; ++q) {
    if (tid == 0) sm.q_off[q] = total_cand;
    total_cand += sm.q_cand[q];
    fast = fast && sm.q_cand[q] <= static_cast<uint32_t>(kClusterCandCap);
  }
  fast = fast && total_cand <= static_cast<uint32_t>(kClusterGatherCap);  // the same in every CTA
  __syncthreads();

  uint32_t need = static_cast<uint32_t>(top_k) - above;  // >= 1
  uint32_t prefix = 0u, mask = 0u;
  if (fast) {
    // gather every candidate of the row; this CTA reads no remote memory after it
    for (uint32_t i = tid; i < total_cand; i += NT) {
      int q = C - 1;
      while (q > 0 && sm.q_off[q] > i) --q;
      const uint2 p = cluster.map_shared_rank(sm.cand, q)[i - sm.q_off[q]];
      sm.gkey[i] = p.x;
      sm.gcell[i] = static_cast<uint32_t>(q * CHUNK) + p.y;
    }
    cluster_arrive();
    __syncthreads();
    if (tid < 32 && total_cand <= 32u * kWarpSelSlots) {
      uint32_t pf, nd;
      if (total_cand <= 256u)
        warp_select_regs<8, C>(sm.gkey, sm.q_off, total_cand, need, sm.q_sure, sm.q_sel, sm.q_eq, sm.tmp256, pf, nd);
      else if (total_cand <= 512u)
        warp_select_regs<16, C>(sm.gkey, sm.q_off, total_cand, need, sm.q_sure, sm.q_sel, sm.q_eq, sm.tmp256, pf, nd);
      else
        warp_select_regs<kWarpSelSlots, C>(sm.gkey, sm.q_off, total_cand, need, sm.q_sure, sm.q_sel, sm.q_eq,
                                        sm.tmp256, pf, nd);
      if (lane == 0) {
        sm.misc[2] = pf;
        sm.misc[3] = nd;
      }
    } else if (tid < 32) {
      // warp 0: exact threshold key over the bits the candidates do not all share
      uint32_t k_and = 0xffffffffu, k_or = 0u;
      for (uint32_t i = lane; i < total_cand; i += 32) {
        k_and &= sm.gkey[i];
        k_or |= sm.gkey[i];
      }
      k_and = __reduce_and_sync(0xffffffffu, k_and);
      k_or = __reduce_or_sync(0xffffffffu, k_or);
      int top = 31;
      while (top >= 0 && !(((k_and ^ k_or) >> top) & 1u)) --top;  // highest differing bit, -1 if none
      uint32_t mk = top >= 31 ? 0u : (top < 0 ? 0xffffffffu : ~((2u << top) - 1u));
      uint32_t pf = k_or & mk, nd = need;
      while (top >= 0) {
        const int shift = top >= 7 ? top - 7 : 0;
        const uint32_t wm = (2u << (top - shift)) - 1u;
#pragma unroll
        for (int i = 0; i < 8; ++i) sm.tmp256[lane * 8 + i] = 0u;
        __syncwarp();
        for (uint32_t i = lane; i < total_cand; i += 32) {
          const uint32_t k = sm.gkey[i];
          if ((k & mk) == pf) atomicAdd(&sm.tmp256[(k >> shift) & wm], 1u);
        }
        __syncwarp();
        uint32_t digit, cnt_above;
        warp_threshold_256(sm.tmp256, nd, digit, cnt_above);
        __syncwarp();
        nd -= cnt_above;
        pf |= digit << shift;
        mk |= wm << shift;
        top = shift - 1;
      }
      if (lane < C) {
        sm.q_sel[lane] = sm.q_sure[lane];
        sm.q_eq[lane] = 0u;
      }
      __syncwarp();
      for (uint32_t i = lane; i < total_cand; i += 32) {
        const uint32_t k = sm.gkey[i];
        const int q = static_cast<int>(sm.gcell[i] / CHUNK);
        if (k > pf) atomicAdd(&sm.q_sel[q], 1u);
        else if (k == pf) atomicAdd(&sm.q_eq[q], 1u);
      }
      if (lane == 0) {
        sm.misc[2] = pf;
        sm.misc[3] = nd;
      }
    }
    __syncthreads();
    prefix = sm.misc[2];
    need = sm.misc[3];
  } else {
    // distributed radix passes over every CTA's own cells, one cluster barrier each
#pragma unroll 1
    for (int pass = 0; pass < 4; ++pass) {
      const int shift = 24 - 8 * pass;
      uint32_t* h = sm.radix[pass & 1];
      if (tid < 256) h[tid] = 0u;
      __syncthreads();
#pragma unroll
      for (int e = 0; e < PER; ++e) {
        if (c0 + e * NT + tid >= V || QSA_BIN(e) != thr_bin) continue;
        const uint32_t k = QSA_KEY(e);
        if ((k & mask) == prefix) atomicAdd(&h[(k >> shift) & 255u], 1u);
      }
      cluster.sync();
      if (tid < 256) {
        uint32_t sum = 0u;
#pragma unroll
        for (int q = 0; q < C; ++q) sum += cluster.map_shared_rank(h, q)[tid];
        sm.tmp256[tid] = sum;
      }
      __syncthreads();
      uint32_t digit, cnt_above;
      find_threshold_bin<NT>(sm.tmp256, 256, need, sm.scratch, sm.result, digit, cnt_above);
      need -= cnt_above;
      prefix |= digit << shift;
      mask |= 255u << shift;
    }
  }
  const uint32_t thr_key = prefix;
  const uint32_t take_eq = need;  // lowest-index cells with key == thr_key to keep

  // ---- mark this CTA's cells.  A higher key is a larger score and equal keys share a
  // bin, so the cells kept are those with key > thr_key and the ties key == thr_key.
  // Word e * (NT / 32) + w of a bitmap holds element e of warp w's 32 threads: one
  // ballot each, kept by lane e % 32 and stored once (no clearing, no atomics).
  {
    constexpr int H = (PER + 31) / 32;
    uint32_t w_sel[H], w_eq[H];
#pragma unroll
    for (int h = 0; h < H; ++h) w_sel[h] = w_eq[h] = 0u;
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      const bool valid = c0 + e * NT + tid < V;
      const uint32_t k = QSA_KEY(e);
      const uint32_t bs = __ballot_sync(0xffffffffu, valid && k > thr_key);
      const uint32_t be = __ballot_sync(0xffffffffu, valid && k == thr_key);
      w_sel[e >> 5] = lane == (e & 31) ? bs : w_sel[e >> 5];
      w_eq[e >> 5] = lane == (e & 31) ? be : w_eq[e >> 5];
    }
#pragma unroll
    for (int h = 0; h < H; ++h) {
      const int e = h * 32 + lane;
      if (e < PER) {
        sm.selb[e * (NT / 32) + (tid >> 5)] = w_sel[h];
        sm.eqb[e * (NT / 32) + (tid >> 5)] = w_eq[h];
      }
    }
  }
  __syncthreads();
  const int per = (WORDS + NT - 1) / NT;
  const int wb = tid * per, we = min(WORDS, wb + per);
  uint32_t nsel = 0u, neq = 0u;
  for (int i = wb; i < we; ++i) {
    nsel += __popc(sm.selb[i]);
    neq += __popc(sm.eqb[i]);
  }
  // one scan of both counts (each below 2^16: a CTA holds at most 32768 cells)
  uint32_t tot_pk;
  const uint32_t rank_pk = block_exclusive_scan<NT>(nsel | (neq << 16), sm.scratch, tot_pk);
  const uint32_t sel_rank = rank_pk & 0xffffu, eq_rank = rank_pk >> 16;
  const uint32_t tot_sel = tot_pk & 0xffffu, tot_eq = tot_pk >> 16;
  if (!fast) {  // the per-CTA counts come from the CTAs themselves
    if (tid == 0) {
      sm.pub[2] = tot_sel;
      sm.pub[3] = tot_eq;
    }
    cluster.sync();
    if (tid < C) {
      const uint32_t* p = cluster.map_shared_rank(sm.pub, tid);
      sm.q_sel[tid] = p[2];
      sm.q_eq[tid] = p[3];
    }
    cluster_arrive();
  }
  __syncthreads();

  // ---- offsets from the lower-ranked CTAs; ties go to the lowest indices first
  uint32_t eq_before = 0u, out_before = 0u;
  for (int q = 0; q < rank; ++q) {
    const uint32_t qtake = eq_before >= take_eq ? 0u : min(sm.q_eq[q], take_eq - eq_before);
    out_before += sm.q_sel[q] + qtake;
    eq_before += sm.q_eq[q];
  }
  const uint32_t my_take = eq_before >= take_eq ? 0u : min(tot_eq, take_eq - eq_before);
  uint32_t r = eq_rank;
  for (int i = wb; i < we && r < my_take; ++i) {
    uint32_t b = sm.eqb[i];
    while (b && r < my_take) {
      const uint32_t low = b & (0u - b);
      sm.selb[i] |= low;
      b ^= low;
      ++r;
    }
  }
  const uint32_t tie_before = min(eq_rank, my_take);  // ties kept by lower threads
  uint32_t pos = out_before + sel_rank + tie_before;
  for (int i = wb; i < we; ++i) {
    uint32_t b = sm.selb[i];
    while (b) {
      const int bit = __ffs(b) - 1;
      b &= b - 1u;
      if (pos < static_cast<uint32_t>(top_k)) out[pos] = c0 + i * 32 + bit;
      ++pos;
    }
  }
  cluster_wait();  // every CTA has finished reading this CTA's shared memory
#undef QSA_KEY
#undef QSA_BIN
}

// grid (C, rows), cluster (C, 1, 1), block 512, dynamic smem cluster_smem_bytes<PER, C>().
// PER cells per thread (held in registers): the cluster covers C * 512 * PER cells, at least
// the longest row.
template <int PER, int C>
__global__ void __launch_bounds__(kClusterThreads) cluster_select_kernel(const float* __restrict__ scores,
                                                                         int64_t ld, int vis0, int top_k,
                                                                         int32_t* __restrict__ ids) {
  extern __shared__ __align__(16) unsigned char csm_raw[];
  griddep_launch();
  griddep_wait();
  cluster_select_row<PER, C>(scores, ld, vis0, top_k, ids, csm_raw);
}

}  // namespace qsa
