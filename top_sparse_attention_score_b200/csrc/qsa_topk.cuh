// qsa_topk.cuh -- exact per-row top-k of fp32 scores, ties to the lower index.
//
// The selection step of the prompt and decode paths (qsa_topk: "opus r15 track A:
// prompt_chunk wave zipping, ...", what changed, item 1), one id set per token
// (the qids row of "Round 5 Track C Report ...", section 1, Target 2).
//
// Radix select spread over many SMs, with no CTA ever waiting on another:
//   histogram  2048-bin count of each score's coarse bin (top 11 bits of the
//              order-preserving key of its fp16 rounding), accumulated in shared
//              memory and flushed with atomics by topk_hist_kernel.  The CTA that finishes last
//              (a fence and a counter, no waiting) finds each row's threshold bin.
//   filter     topk_filter_kernel: each CTA appends the cells of its chunk above
//              the threshold bin to the row's "sure" list and the cells in it, with
//              their full 32-bit keys, to the "candidate" list.
//   final      topk_final_kernel, one CTA per row: radix-selects the exact 32-bit
//              threshold key among the candidates (four 8-bit passes), keeps the
//              lowest-index cells among equal keys, and writes the ids in ascending
//              order by compacting a bitmap of the row's cells.
// A candidate list that overflows its capacity is not lost: the final CTA then
// re-reads the score row itself for that bin.
#pragma once

#include "qsa_common.cuh"

namespace qsa {

constexpr int kTopkChunk = 4096;    // scores per hist/filter CTA
constexpr int kTopkThreads = 256;   // hist/filter block
constexpr int kMaxWindowBits = 1 << 18;  // cells per bitmap window (two 32 KB bitmaps)

// Per-row counters, zeroed before every use.
enum : int {
  kCtrSure = 0, kCtrCand = 1, kCtrHistDone = 2, kCtrThrBin = 4, kCtrAbove = 5,
  kCtrWords = 8  // words 3, 6 and 7 are spare (the layout and its size stay fixed)
};

struct TopkWs {
  uint32_t* hist;   // [rows][kBins]
  uint32_t* ctr;    // [rows][kCtrWords], then one grid-wide counter
  int32_t* sure;    // [rows][top_k]
  uint2* cand;      // [rows][cand_cap] (key, cell)
  int cand_cap;
};

__global__ void topk_zero_kernel(uint32_t* p, int64_t n) {
  griddep_launch();
  griddep_wait();
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    p[i] = 0u;
}

// Threshold bin of one row from its global histogram (copied to shared memory
// through L2 first: other CTAs wrote it).  Writes ctr[kCtrThrBin], ctr[kCtrAbove].
template <int NT>
__device__ void row_threshold(const uint32_t* ghist, uint32_t* ctr, uint32_t k, uint32_t* sh,
                              uint32_t* scratch, uint32_t* result) {
  for (int i = threadIdx.x; i < kBins; i += NT) sh[i] = __ldcg(ghist + i);
  __syncthreads();
  uint32_t thr, above;
  find_threshold_bin<NT>(sh, kBins, k, scratch, result, thr, above);
  if (threadIdx.x == 0) {
    ctr[kCtrThrBin] = thr;
    ctr[kCtrAbove] = above;
  }
  __syncthreads();
}

// True in every thread of the CTA that arrives last at `counter` (of `total`).
__device__ __forceinline__ bool last_to_arrive(uint32_t* counter, uint32_t total, uint32_t* flag) {
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) *flag = (atomicAdd(counter, 1u) == total - 1u) ? 1u : 0u;
  __syncthreads();
  const bool last = *flag != 0u;
  if (last) __threadfence();
  return last;
}

// grid: x = chunks, y = rows
__global__ void __launch_bounds__(kTopkThreads, 8) topk_hist_kernel(const float* __restrict__ scores,
                                                                 int64_t ld, int vis0, int top_k,
                                                                 TopkWs ws) {
  __shared__ uint32_t h[kBins];
  __shared__ uint32_t scratch[33];
  __shared__ uint32_t result[2];
  __shared__ uint32_t flag;
  griddep_launch();
  // Wait before anything else, even in CTAs with no work: a kernel that finished
  // without waiting would let its dependents overtake the kernels before it.
  griddep_wait();
  const int row = blockIdx.y;
  const int V = vis0 + row;
  if (V <= top_k) return;  // every visible cell is selected; no threshold needed
  for (int i = threadIdx.x; i < kBins; i += kTopkThreads) h[i] = 0u;
  __syncthreads();
  const int c0 = blockIdx.x * kTopkChunk;
  const float* s = scores + row * ld;
  if (c0 < V) {
    // all 16 scores of this thread in flight at once
    float v[16];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int c = c0 + u * (kTopkThreads * 4) + threadIdx.x * 4;
      if (c + 4 <= V) {
        const float4 x = __ldcg(reinterpret_cast<const float4*>(s + c));
        v[4 * u] = x.x; v[4 * u + 1] = x.y; v[4 * u + 2] = x.z; v[4 * u + 3] = x.w;
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) v[4 * u + e] = (c + e < V) ? __ldcg(s + c + e) : 0.f;
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (c0 + u * (kTopkThreads * 4) + threadIdx.x * 4 + e < V) atomicAdd(&h[score_bin(v[4 * u + e])], 1u);
  }
  __syncthreads();
  uint32_t* gh = ws.hist + static_cast<size_t>(row) * kBins;
  for (int i = threadIdx.x; i < kBins; i += kTopkThreads)
    if (h[i]) atomicAdd(gh + i, h[i]);
  uint32_t* ctr = ws.ctr + static_cast<size_t>(row) * kCtrWords;
  if (last_to_arrive(ctr + kCtrHistDone, gridDim.x, &flag))
    row_threshold<kTopkThreads>(gh, ctr, static_cast<uint32_t>(top_k), h, scratch, result);
}

// Append `cell` to a list with one atomic per warp; only slots below `cap` are written.
__device__ __forceinline__ void warp_append(bool pred, uint32_t* counter, int32_t* list_ids,
                                            uint2* list_pairs, uint32_t key, int cell, int cap) {
  const uint32_t m = __ballot_sync(0xffffffffu, pred);
  if (!m) return;
  const int lane = threadIdx.x & 31;
  const int leader = __ffs(m) - 1;
  uint32_t base = 0;
  if (lane == leader) base = atomicAdd(counter, static_cast<uint32_t>(__popc(m)));
  base = __shfl_sync(0xffffffffu, base, leader);
  if (pred) {
    const uint32_t pos = base + __popc(m & ((1u << lane) - 1u));
    if (static_cast<int>(pos) < cap) {
      if (list_ids) list_ids[pos] = cell;
      else list_pairs[pos] = make_uint2(key, static_cast<uint32_t>(cell));
    }
  }
}

struct SelectSmem {
  uint32_t h256[256];
  uint32_t scratch[33];
  uint32_t result[2];
  uint32_t flag;
};

// The exact selection of one row by one CTA of NT threads, once its sure and
// candidate lists are complete.  `bits` is 2 * win_bits / 32 words of shared memory.
template <int NT>
__device__ void final_select(const float* __restrict__ s, int V, int top_k, const uint32_t* ctr,
                             const int32_t* sure, const uint2* cand, int cand_cap, uint32_t* bits,
                             int win_bits, SelectSmem& sm, int32_t* __restrict__ out) {
  const int tid = threadIdx.x;
  uint32_t* selb = bits;
  uint32_t* eqb = bits + win_bits / 32;
  const uint32_t thr_bin = __ldcg(ctr + kCtrThrBin);
  const uint32_t n_sure = __ldcg(ctr + kCtrSure);
  const uint32_t n_cand_all = __ldcg(ctr + kCtrCand);
  const bool overflow = n_cand_all > static_cast<uint32_t>(cand_cap);
  const int n_src = overflow ? V : static_cast<int>(n_cand_all);

  // Bits every candidate shares need no radix pass (they all sit in one coarse
  // bin, so the top byte is usually common): AND and OR of the candidate keys.
  uint32_t k_and = 0xffffffffu, k_or = 0u;
  for (int i = tid; i < n_src; i += NT) {
    uint32_t key;
    if (overflow) {
      const float v = __ldcg(s + i);
      if (score_bin(v) != thr_bin) continue;
      key = score_key(v);
    } else {
      key = __ldcg(&cand[i].x);
    }
    k_and &= key;
    k_or |= key;
  }
  k_and = __reduce_and_sync(0xffffffffu, k_and);
  k_or = __reduce_or_sync(0xffffffffu, k_or);
  if (tid == 0) {
    sm.result[0] = 0xffffffffu;
    sm.result[1] = 0u;
  }
  __syncthreads();
  if ((tid & 31) == 0) {
    atomicAnd(&sm.result[0], k_and);
    atomicOr(&sm.result[1], k_or);
  }
  __syncthreads();
  const uint32_t same = ~(sm.result[0] ^ sm.result[1]);
  const uint32_t common = sm.result[1];
  __syncthreads();
  int top = 31;
  while (top >= 0 && ((same >> top) & 1u)) --top;  // highest differing bit, -1 if none
  uint32_t mask = top >= 31 ? 0u : (top < 0 ? 0xffffffffu : ~((2u << top) - 1u));
  uint32_t prefix = common & mask;

  // Exact threshold key among the candidates: 8-bit passes over the differing bits.
  uint32_t need = static_cast<uint32_t>(top_k) - n_sure;  // >= 1
  while (top >= 0) {
    const int shift = top >= 7 ? top - 7 : 0;
    const uint32_t width_mask = (2u << (top - shift)) - 1u;
    for (int i = tid; i < 256; i += NT) sm.h256[i] = 0u;
    __syncthreads();
    for (int i = tid; i < n_src; i += NT) {
      uint32_t key;
      if (overflow) {
        const float v = __ldcg(s + i);
        if (score_bin(v) != thr_bin) continue;
        key = score_key(v);
      } else {
        key = __ldcg(&cand[i].x);
      }
      if ((key & mask) == prefix) atomicAdd(&sm.h256[(key >> shift) & width_mask], 1u);
    }
    __syncthreads();
    uint32_t digit, cnt_above;
    find_threshold_bin<NT>(sm.h256, 256, need, sm.scratch, sm.result, digit, cnt_above);
    need -= cnt_above;
    prefix |= digit << shift;
    mask |= width_mask << shift;
    top = shift - 1;
  }
  const uint32_t thr_key = prefix;
  const uint32_t take_eq = need;  // lowest-index cells with key == thr_key to keep

  uint32_t out_base = 0u, eq_taken = 0u;
  for (int w0 = 0; w0 < V; w0 += win_bits) {
    const int wn = min(win_bits, V - w0);
    const int words = (wn + 31) >> 5;
    for (int i = tid; i < words; i += NT) {
      selb[i] = 0u;
      eqb[i] = 0u;
    }
    __syncthreads();
    for (uint32_t i = tid; i < n_sure; i += NT) {
      const int c = __ldcg(sure + i) - w0;
      if (c >= 0 && c < wn) atomicOr(&selb[c >> 5], 1u << (c & 31));
    }
    if (overflow) {
      for (int i = w0 + tid; i < w0 + wn; i += NT) {
        const float v = __ldcg(s + i);
        if (score_bin(v) != thr_bin) continue;
        const uint32_t key = score_key(v);
        const int c = i - w0;
        if (key > thr_key) atomicOr(&selb[c >> 5], 1u << (c & 31));
        else if (key == thr_key) atomicOr(&eqb[c >> 5], 1u << (c & 31));
      }
    } else {
      for (int i = tid; i < n_src; i += NT) {
        const uint2 p = __ldcg(cand + i);
        const int c = static_cast<int>(p.y) - w0;
        if (c < 0 || c >= wn) continue;
        if (p.x > thr_key) atomicOr(&selb[c >> 5], 1u << (c & 31));
        else if (p.x == thr_key) atomicOr(&eqb[c >> 5], 1u << (c & 31));
      }
    }
    __syncthreads();
    const int per = (words + NT - 1) / NT;
    const int wb = tid * per, we = min(words, wb + per);
    uint32_t cnt = 0u;
    for (int i = wb; i < we; ++i) cnt += __popc(eqb[i]);
    uint32_t tot;
    uint32_t rank = eq_taken + block_exclusive_scan<NT>(cnt, sm.scratch, tot);
    for (int i = wb; i < we && rank < take_eq; ++i) {
      uint32_t b = eqb[i];
      while (b && rank < take_eq) {
        const uint32_t low = b & (0u - b);
        selb[i] |= low;
        b ^= low;
        ++rank;
      }
    }
    eq_taken += tot;
    __syncthreads();
    cnt = 0u;
    for (int i = wb; i < we; ++i) cnt += __popc(selb[i]);
    uint32_t pos = out_base + block_exclusive_scan<NT>(cnt, sm.scratch, tot);
    for (int i = wb; i < we; ++i) {
      uint32_t b = selb[i];
      while (b) {
        const int bit = __ffs(b) - 1;
        b &= b - 1u;
        if (pos < static_cast<uint32_t>(top_k)) out[pos] = w0 + i * 32 + bit;
        ++pos;
      }
    }
    out_base += tot;
    __syncthreads();
  }
  for (uint32_t i = out_base + tid; i < static_cast<uint32_t>(top_k); i += NT) out[i] = -1;
}

// grid: x = chunks (of the longest row), y = rows; block kTopkThreads.
// Appends each chunk's cells above the threshold bin to the sure list and the
// cells in it (with their 32-bit keys) to the candidate list.  The CTA counts
// its cells first and reserves its slots with one global atomic per list, so no
// warp waits on an atomic round trip per hit.
__global__ void __launch_bounds__(kTopkThreads, 8) topk_filter_kernel(const float* __restrict__ scores,
                                                                      int64_t ld, int vis0, int top_k,
                                                                      TopkWs ws) {
  __shared__ uint32_t warp_n[2][kTopkThreads / 32];
  __shared__ uint32_t base_g[2];
  griddep_launch();
  griddep_wait();
  const int row = blockIdx.y;
  const int V = vis0 + row;
  if (V <= top_k) return;
  const int c0 = blockIdx.x * kTopkChunk;
  if (c0 >= V) return;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t* ctr = ws.ctr + static_cast<size_t>(row) * kCtrWords;
  const float* s = scores + row * ld;
  int32_t* sure = ws.sure + static_cast<size_t>(row) * top_k;
  uint2* cand = ws.cand + static_cast<size_t>(row) * ws.cand_cap;
  const uint32_t thr = __ldcg(ctr + kCtrThrBin);
  // all 16 scores of this thread in flight at once
  float v[16];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int c = c0 + u * (kTopkThreads * 4) + threadIdx.x * 4;
    if (c + 4 <= V) {
      const float4 x = __ldcg(reinterpret_cast<const float4*>(s + c));
      v[4 * u] = x.x; v[4 * u + 1] = x.y; v[4 * u + 2] = x.z; v[4 * u + 3] = x.w;
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) v[4 * u + e] = (c + e < V) ? __ldcg(s + c + e) : 0.f;
    }
  }
  // classify: bit e of `up` / `eq` marks element e above / in the threshold bin
  uint32_t up = 0u, eq = 0u;
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const int c = c0 + (e >> 2) * (kTopkThreads * 4) + threadIdx.x * 4 + (e & 3);
    if (c >= V) continue;
    const uint32_t b = score_bin(v[e]);
    up |= (b > thr ? 1u : 0u) << e;
    eq |= (b == thr ? 1u : 0u) << e;
  }
  const uint32_t nu = __popc(up), ne = __popc(eq);
  // per-warp exclusive offsets, then per-CTA offsets, then one global atomic per list
  uint32_t xu = nu, xe = ne;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t yu = __shfl_up_sync(0xffffffffu, xu, o);
    const uint32_t ye = __shfl_up_sync(0xffffffffu, xe, o);
    if (lane >= o) {
      xu += yu;
      xe += ye;
    }
  }
  if (lane == 31) {
    warp_n[0][warp] = xu;
    warp_n[1][warp] = xe;
  }
  __syncthreads();
  if (threadIdx.x < 2) {
    uint32_t tot = 0u;
    for (int w = 0; w < kTopkThreads / 32; ++w) {
      const uint32_t n = warp_n[threadIdx.x][w];
      warp_n[threadIdx.x][w] = tot;
      tot += n;
    }
    base_g[threadIdx.x] = tot ? atomicAdd(ctr + (threadIdx.x == 0 ? kCtrSure : kCtrCand), tot) : 0u;
  }
  __syncthreads();
  uint32_t pu = base_g[0] + warp_n[0][warp] + xu - nu;
  uint32_t pe = base_g[1] + warp_n[1][warp] + xe - ne;
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const int c = c0 + (e >> 2) * (kTopkThreads * 4) + threadIdx.x * 4 + (e & 3);
    if ((up >> e) & 1u) {
      if (pu < static_cast<uint32_t>(top_k)) sure[pu] = c;
      ++pu;
    } else if ((eq >> e) & 1u) {
      if (pe < static_cast<uint32_t>(ws.cand_cap)) cand[pe] = make_uint2(score_key(v[e]), static_cast<uint32_t>(c));
      ++pe;
    }
  }
}

constexpr int kFinalThreads = 1024;

// One CTA per row once the lists are complete; dynamic smem: two bitmaps of
// win_bits / 32 words.
__global__ void __launch_bounds__(kFinalThreads) topk_final_kernel(const float* __restrict__ scores,
                                                                   int64_t ld, int vis0, int top_k,
                                                                   TopkWs ws, int win_bits,
                                                                   int32_t* __restrict__ ids) {
  extern __shared__ uint32_t bits[];
  __shared__ SelectSmem sm;
  griddep_launch();
  griddep_wait();
  const int row = blockIdx.x;
  const int V = vis0 + row;
  int32_t* out = ids + static_cast<size_t>(row) * top_k;
  if (V <= top_k) {  // every visible cell, ascending
    for (int i = threadIdx.x; i < top_k; i += kFinalThreads) out[i] = i < V ? i : -1;
    return;
  }
  final_select<kFinalThreads>(scores + row * ld, V, top_k, ws.ctr + static_cast<size_t>(row) * kCtrWords,
                              ws.sure + static_cast<size_t>(row) * top_k,
                              ws.cand + static_cast<size_t>(row) * ws.cand_cap, ws.cand_cap, bits, win_bits,
                              sm, out);
}

}  // namespace qsa
