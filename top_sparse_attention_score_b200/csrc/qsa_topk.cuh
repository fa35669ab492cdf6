// qsa_topk.cuh -- exact per-row top-k of fp32 scores, ties to the lower index.
//
// The selection step of the prompt and decode paths (qsa_topk: "opus r15 track A:
// prompt_chunk wave zipping, ...", what changed, item 1), one id set per token
// (the qids row of "Round 5 Track C Report ...", section 1, Target 2).
//
// Radix select in three launches, so every row spreads over many SMs:
//   hist   (many CTAs per row) 2048-bin histogram of each score's coarse bin
//          (top 11 bits of its fp16 key) in shared memory, flushed with atomics;
//   filter (many CTAs per row) each CTA finds the bin holding the k-th score,
//          appends cells of higher bins to the row's "sure" list and cells of
//          that bin, with their full 32-bit keys, to the "candidate" list
//          (warp-aggregated atomics);
//   final  (one CTA per row) radix-selects the exact 32-bit threshold key
//          among the candidates (four 8-bit passes with shared histograms),
//          takes the lowest-index cells among equal keys, and emits the ids in
//          ascending order by compacting a bitmap of the row's cells.
// A candidate list that overflows its capacity is not lost: the final pass
// then re-reads the score row itself for that bin.
#pragma once

#include "qsa_common.cuh"

namespace qsa {

constexpr int kTopkChunk = 4096;   // scores per hist/filter CTA
constexpr int kTopkThreads = 256;  // hist/filter block
constexpr int kFinalThreads = 1024;
constexpr int kMaxWindowBits = 1 << 19;  // cells per bitmap window (two 64 KB bitmaps)

struct TopkWs {
  uint32_t* hist;   // [rows][kBins]
  uint32_t* ctr;    // [rows][4]: n_sure, n_cand
  int32_t* sure;    // [rows][top_k]
  uint2* cand;      // [rows][cand_cap] (key, cell)
  int cand_cap;
};

__global__ void topk_zero_kernel(uint32_t* p, int64_t n) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    p[i] = 0u;
}

// grid: x = chunks, y = rows
__global__ void __launch_bounds__(kTopkThreads) topk_hist_kernel(const float* __restrict__ scores,
                                                                 int64_t ld, int vis0, int top_k,
                                                                 TopkWs ws) {
  __shared__ uint32_t h[kBins];
  const int row = blockIdx.y;
  const int V = vis0 + row;
  if (V <= top_k) return;
  const int c0 = blockIdx.x * kTopkChunk;
  if (c0 >= V) return;
  const int c1 = min(V, c0 + kTopkChunk);
  for (int i = threadIdx.x; i < kBins; i += kTopkThreads) h[i] = 0u;
  __syncthreads();
  const float* s = scores + row * ld;
  for (int c = c0 + threadIdx.x * 4; c < c1; c += kTopkThreads * 4) {
    if (c + 4 <= c1) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(s + c));
      atomicAdd(&h[score_bin(v.x)], 1u);
      atomicAdd(&h[score_bin(v.y)], 1u);
      atomicAdd(&h[score_bin(v.z)], 1u);
      atomicAdd(&h[score_bin(v.w)], 1u);
    } else {
      for (int e = c; e < c1; ++e) atomicAdd(&h[score_bin(s[e])], 1u);
    }
  }
  __syncthreads();
  uint32_t* gh = ws.hist + static_cast<size_t>(row) * kBins;
  for (int i = threadIdx.x; i < kBins; i += kTopkThreads)
    if (h[i]) atomicAdd(gh + i, h[i]);
}

// Append `cell` to a list with one atomic per warp.  Returns nothing; writes
// only slots below `cap`.
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

// grid: x = chunks, y = rows
__global__ void __launch_bounds__(kTopkThreads) topk_filter_kernel(const float* __restrict__ scores,
                                                                   int64_t ld, int vis0, int top_k,
                                                                   TopkWs ws) {
  __shared__ uint32_t scratch[33];
  __shared__ uint32_t result[2];
  const int row = blockIdx.y;
  const int V = vis0 + row;
  if (V <= top_k) return;
  const int c0 = blockIdx.x * kTopkChunk;
  if (c0 >= V) return;
  const int c1 = min(V, c0 + kTopkChunk);
  uint32_t thr, above;
  find_threshold_bin<kTopkThreads>(ws.hist + static_cast<size_t>(row) * kBins, kBins,
                                   static_cast<uint32_t>(top_k), scratch, result, thr, above);
  const float* s = scores + row * ld;
  uint32_t* ctr = ws.ctr + static_cast<size_t>(row) * 4;
  int32_t* sure = ws.sure + static_cast<size_t>(row) * top_k;
  uint2* cand = ws.cand + static_cast<size_t>(row) * ws.cand_cap;
  // Every lane walks the chunk in lockstep so the warp-wide ballots line up.
  for (int base = c0; base < c1; base += kTopkThreads) {
    const int c = base + threadIdx.x;
    const bool in = c < c1;
    const float v = in ? s[c] : 0.f;
    const uint32_t b = in ? score_bin(v) : 0u;
    warp_append(in && b > thr, ctr + 0, sure, nullptr, 0u, c, top_k);
    warp_append(in && b == thr, ctr + 1, nullptr, cand, score_key(v), c, ws.cand_cap);
  }
}

// One CTA per row.  Dynamic shared memory: two bitmaps of win_bits / 32 words
// (win_bits a multiple of 32, at most kMaxWindowBits).
__global__ void __launch_bounds__(kFinalThreads) topk_final_kernel(const float* __restrict__ scores,
                                                                   int64_t ld, int vis0, int top_k,
                                                                   TopkWs ws, int win_bits,
                                                                   int32_t* __restrict__ ids) {
  extern __shared__ uint32_t bitmaps[];
  uint32_t* selb = bitmaps;
  uint32_t* eqb = bitmaps + win_bits / 32;
  __shared__ uint32_t h256[256];
  __shared__ uint32_t scratch[33];
  __shared__ uint32_t result[2];
  const int row = blockIdx.x;
  const int V = vis0 + row;
  const int tid = threadIdx.x;
  int32_t* out = ids + static_cast<size_t>(row) * top_k;

  if (V <= top_k) {  // every visible cell, ascending
    for (int i = tid; i < top_k; i += kFinalThreads) out[i] = i < V ? i : -1;
    return;
  }
  const float* s = scores + row * ld;
  uint32_t thr_bin, above;
  find_threshold_bin<kFinalThreads>(ws.hist + static_cast<size_t>(row) * kBins, kBins,
                                    static_cast<uint32_t>(top_k), scratch, result, thr_bin,
                                    above);
  const uint32_t* ctr = ws.ctr + static_cast<size_t>(row) * 4;
  const uint32_t n_sure = ctr[0];
  const uint32_t n_cand_all = ctr[1];
  const bool overflow = n_cand_all > static_cast<uint32_t>(ws.cand_cap);
  const int n_src = overflow ? V : static_cast<int>(n_cand_all);
  const int32_t* sure = ws.sure + static_cast<size_t>(row) * top_k;
  const uint2* cand = ws.cand + static_cast<size_t>(row) * ws.cand_cap;
  (void)above;

  // Exact threshold key among the candidates: 4 passes of 8 bits.
  uint32_t need = static_cast<uint32_t>(top_k) - n_sure;  // >= 1
  uint32_t prefix = 0u, mask = 0u;
  for (int shift = 24; shift >= 0; shift -= 8) {
    if (tid < 256) h256[tid] = 0u;
    __syncthreads();
    for (int i = tid; i < n_src; i += kFinalThreads) {
      uint32_t key;
      if (overflow) {
        const float v = s[i];
        if (score_bin(v) != thr_bin) continue;
        key = score_key(v);
      } else {
        key = cand[i].x;
      }
      if ((key & mask) == prefix) atomicAdd(&h256[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    uint32_t digit, cnt_above;
    find_threshold_bin<kFinalThreads>(h256, 256, need, scratch, result, digit, cnt_above);
    need -= cnt_above;
    prefix |= digit << shift;
    mask |= 255u << shift;
  }
  const uint32_t thr_key = prefix;
  const uint32_t take_eq = need;  // lowest-index cells with key == thr_key to take

  // Bitmap windows over the row's cells, emitted in ascending order.
  uint32_t out_base = 0u, eq_taken = 0u;
  for (int w0 = 0; w0 < V; w0 += win_bits) {
    const int wn = min(win_bits, V - w0);
    const int words = (wn + 31) >> 5;
    for (int i = tid; i < words; i += kFinalThreads) {
      selb[i] = 0u;
      eqb[i] = 0u;
    }
    __syncthreads();
    for (uint32_t i = tid; i < n_sure; i += kFinalThreads) {
      const int c = sure[i] - w0;
      if (c >= 0 && c < wn) atomicOr(&selb[c >> 5], 1u << (c & 31));
    }
    if (overflow) {
      for (int i = w0 + tid; i < w0 + wn; i += kFinalThreads) {
        const float v = s[i];
        if (score_bin(v) != thr_bin) continue;
        const uint32_t key = score_key(v);
        const int c = i - w0;
        if (key > thr_key) atomicOr(&selb[c >> 5], 1u << (c & 31));
        else if (key == thr_key) atomicOr(&eqb[c >> 5], 1u << (c & 31));
      }
    } else {
      for (int i = tid; i < n_src; i += kFinalThreads) {
        const uint2 p = cand[i];
        const int c = static_cast<int>(p.y) - w0;
        if (c < 0 || c >= wn) continue;
        if (p.x > thr_key) atomicOr(&selb[c >> 5], 1u << (c & 31));
        else if (p.x == thr_key) atomicOr(&eqb[c >> 5], 1u << (c & 31));
      }
    }
    __syncthreads();
    // Each thread owns a contiguous run of words.
    const int per = (words + kFinalThreads - 1) / kFinalThreads;
    const int wb = tid * per, we = min(words, wb + per);
    // Ties at the threshold: keep the lowest-index take_eq cells overall.
    uint32_t cnt = 0u;
    for (int i = wb; i < we; ++i) cnt += __popc(eqb[i]);
    uint32_t tot;
    uint32_t rank = eq_taken + block_exclusive_scan<kFinalThreads>(cnt, scratch, tot);
    for (int i = wb; i < we && rank < take_eq; ++i) {
      uint32_t bits = eqb[i];
      while (bits && rank < take_eq) {
        const uint32_t low = bits & (0u - bits);
        selb[i] |= low;
        bits ^= low;
        ++rank;
      }
    }
    eq_taken += tot;
    __syncthreads();
    cnt = 0u;
    for (int i = wb; i < we; ++i) cnt += __popc(selb[i]);
    uint32_t pos = out_base + block_exclusive_scan<kFinalThreads>(cnt, scratch, tot);
    for (int i = wb; i < we; ++i) {
      uint32_t bits = selb[i];
      while (bits) {
        const int b = __ffs(bits) - 1;
        bits &= bits - 1u;
        if (pos < static_cast<uint32_t>(top_k)) out[pos] = w0 + i * 32 + b;
        ++pos;
      }
    }
    out_base += tot;
    __syncthreads();
  }
  for (uint32_t i = out_base + tid; i < static_cast<uint32_t>(top_k); i += kFinalThreads) out[i] = -1;
}

}  // namespace qsa
