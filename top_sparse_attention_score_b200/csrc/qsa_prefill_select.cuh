// qsa_prefill_select.cuh -- a prompt chunk's selection without the T x L score matrix.
//
// qsa_score_mm followed by qsa_topk ("opus r15 track A: prompt_chunk wave zipping, ...",
// what changed, item 1) for a chunk of T tokens, row t seeing cells [0, vis0 + t):
//
//   1. prefill_threshold_kernel -- each row scores every R-th visible cell (R = 16, or
//      more for rows of over 8192 x 16 cells; the decode GEMV) into a histogram of coarse
//      bins and takes as its candidate threshold the lower edge of the bin where the
//      sample's count from the top reaches a margin above top_k / R: a score that, by the
//      sample, clearly more than top_k cells reach.
//   2. score_select_kernel -- the tcgen05 GEMM of every (cell, token) score with the cells
//      as the 128 M rows and 64 tokens x 4 indexer heads as the N = 256 columns, so one
//      TMEM lane holds a cell's 16 head products for 4 tokens and the ReLU-weighted head
//      sum needs no data exchange.  The epilogue keeps only the candidates -- visible
//      cells whose score reaches the row's threshold -- as (order key, cell) pairs in
//      per-(CTA, token block) lists; nothing of size T x L is written.
//   3. prefill_final_kernel -- per row, the exact top_k among the candidates: radix select
//      on the 32-bit order keys, the lowest cell index among equal keys, ids ascending.
//      The candidates are exactly the visible cells at or above the threshold, so a row
//      with at least top_k of them has its whole top_k among them (every other cell
//      scores below the threshold, hence below the k-th candidate).  A row with fewer
//      candidates, or more than its lists hold, is selected exactly by the same CTA
//      from scores it recomputes: radix passes over all its cells.  Slower, never wrong.
#pragma once

#include "qsa_index_score.cuh"
#include "qsa_sm100.cuh"
#include "qsa_topk.cuh"

namespace qsa {

constexpr int kPsStride = 16;        // smallest sample stride of the threshold pass
constexpr int kPsSamples = 8192;     // samples per row the stride grows to keep (longer rows)
constexpr int kPsThreads = 256;      // threshold CTA: 8 warps over 8 rows
constexpr int kSsCells = 128;        // GEMM M: cells per tile
constexpr int kSsTokens = 64;        // tokens per tile
constexpr int kSsN = kSsTokens * kHI;  // GEMM N: (token, head) columns
constexpr int kSsStages = 6;         // key-tile ring
constexpr int kSsEpiWarps = 16;      // 4 TMEM lane quadrants x 4 column quarters
constexpr int kSsThreads = (2 + kSsEpiWarps) * 32;
constexpr int kSsKeyBytes = kSsCells * kDI * 2;  // 16 KB
constexpr int kSsQBytes = kSsN * kDI * 2;        // 32 KB
constexpr int kSsCapPerTile = 16;    // candidate slots per (token, cell tile) of a list
constexpr int kSsCapSlack = 64;
constexpr int kSsTable = 8;          // words per token of an epilogue warp's table
constexpr int kSsSmemBytes = kSsQBytes + kSsStages * kSsKeyBytes + kSsEpiWarps * 16 * kSsTable * 4 +
                             2 * kSsTokens * 4 + kSsEpiWarps * 16 * 32 * 4 /*scores*/ +
                             kSsEpiWarps * 16 * 4 /*ballots*/ + 512 /*barriers*/ + 1024 /*align*/;
static_assert(kSsSmemBytes > 114 * 1024, "one GEMM CTA per SM (it allocates all 512 TMEM columns)");
constexpr int kPfThreads = 512;      // final kernel (two CTAs per SM)
constexpr int kPfCand = 8192;        // candidates a final CTA holds in shared memory
constexpr int kPfWinBits = 65536;    // cells per bitmap window
constexpr int kPfMaxSegs = 64;       // lists one row may span
constexpr int kPfSmemBytes = kPfCand * 8 + 2 * (kPfWinBits / 32) * 4;

struct PrefillSel {
  const __half* keys;   // the cache's indexer keys [ncells][64]
  const __half* iq;     // [T][4][64]
  const float* iw;      // [T][4]
  int T;
  int vis0;             // cells row 0 sees (row t sees vis0 + t)
  int top_k;
  int ncells;
  float* thr;           // [T] candidate threshold: a visible cell is a candidate iff score >= thr[t]
  uint2* cand;          // candidate lists (order key, cell), see ss_list_base
  uint32_t* seg_count;  // [grid][2][64] entries appended to each list (may exceed its capacity)
  int n_ct;             // cell tiles (ceil(ncells / 128))
  int items;            // token blocks x cell tiles
  int per;              // items per GEMM CTA (<= n_ct, so a CTA meets at most two token blocks)
  int grid;             // GEMM CTAs
  uint32_t* status;     // device status word (bounded waits)
};

// ---- candidate list geometry (the same on host and device)
//
// GEMM CTA b owns items [b * per, min(items, (b + 1) * per)); the part in its first token
// block is its segment 0, the rest (if any) segment 1.  Segment s keeps one list per token
// of its block, of capacity kSsCapPerTile * (tiles in the segment) + kSsCapSlack.

__host__ __device__ inline int ss_cap(int tiles) { return kSsCapPerTile * tiles + kSsCapSlack; }

__host__ __device__ inline size_t ss_cta_entries(int per) {
  return static_cast<size_t>(kSsTokens) * (kSsCapPerTile * per + 2 * kSsCapSlack);
}

// Tiles of CTA b's two segments.
__host__ __device__ inline void ss_segments(int b, int per, int items, int n_ct, int& tiles0, int& tiles1) {
  const int it0 = b * per, it1 = min(items, it0 + per);
  const int end0 = min(it1, (it0 / n_ct + 1) * n_ct);
  tiles0 = max(0, end0 - it0);
  tiles1 = max(0, it1 - end0);
}

// First entry of the list of token `tl` (0..63) in segment s of CTA b.
__host__ __device__ inline size_t ss_list_base(int b, int s, int tl, int per, int tiles0, int tiles1) {
  const size_t seg = static_cast<size_t>(b) * ss_cta_entries(per) +
                     (s ? static_cast<size_t>(kSsTokens) * ss_cap(tiles0) : 0);
  return seg + static_cast<size_t>(tl) * ss_cap(s ? tiles1 : tiles0);
}

// Cells the last token of block tb sees, and the block's live cell tiles (the rest are
// beyond every token's horizon and skipped).
__device__ __forceinline__ int ss_live_tiles(const PrefillSel& a, int tb) {
  const int vmax = a.vis0 + min(a.T, (tb + 1) * kSsTokens) - 1;
  return min(a.n_ct, (vmax + kSsCells - 1) / kSsCells);
}

// Inverse of score_key.
__device__ __forceinline__ float key_float(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k ^ 0x80000000u) : ~k);
}

// A float below every value whose coarse bin (score_bin) is `bin` or higher: the bin's
// lowest fp16 value, moved down by 65536 fp32 steps (more than half an fp16 step, so
// every fp32 value that rounds into the bin stays above it).
__device__ __forceinline__ float bin_floor(uint32_t bin) {
  const uint32_t k16 = bin << 5;
  const uint32_t b16 = (k16 & 0x8000u) ? (k16 ^ 0x8000u) : (~k16 & 0xffffu);
  const uint32_t k32 = score_key(__half2float(__ushort_as_half(static_cast<unsigned short>(b16))));
  return key_float(k32 > 65536u ? k32 - 65536u : 0u);
}

// One warp over `nbins` (a multiple of 32) bins counted from the highest: the bin where
// the running count first reaches k (0 if the total stays below k).
__device__ __forceinline__ uint32_t warp_find_bin(const uint32_t* h, int nbins, uint32_t k) {
  const int lane = threadIdx.x & 31;
  const int per = nbins / 32;
  const int hi = nbins - 1 - per * lane;
  uint32_t local = 0u;
  for (int i = 0; i < per; ++i) local += h[hi - i];
  uint32_t incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const uint32_t before = incl - local;
  const uint32_t m = __ballot_sync(0xffffffffu, before < k && incl >= k);
  uint32_t bin = 0u;
  if (m && lane == __ffs(m) - 1) {
    uint32_t run = before;
    for (int i = 0; i < per; ++i) {
      run += h[hi - i];
      if (run >= k) {
        bin = static_cast<uint32_t>(hi - i);
        break;
      }
    }
  }
  return m ? __shfl_sync(0xffffffffu, bin, __ffs(m) - 1) : 0u;
}

// ---------------------------------------------------------------- 1. thresholds

// grid: ceil(T / 8); block: kPsThreads; dynamic smem: 8 x kBins x 4 bytes.
__global__ void __launch_bounds__(kPsThreads) prefill_threshold_kernel(PrefillSel a) {
  extern __shared__ uint32_t ps_hist[];  // [8][kBins]
  __shared__ __align__(16) uint32_t s_iq[kScoreRowsPerCta * kHI * kScoreIqWords];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int rb = blockIdx.x * kScoreRowsPerCta;
  griddep_launch();
  griddep_wait();  // the chunk's own keys may come from the cache write before this kernel
  for (int i = threadIdx.x; i < kScoreRowsPerCta * kBins; i += kPsThreads) ps_hist[i] = 0u;
  gemv_stage_q<kPsThreads>(s_iq, a.iq, rb, a.T);
  __syncthreads();
  GemvQ Q;
  gemv_load_q(Q, s_iq);
  float w[4][2];
  gemv_load_w(w, a.iw, rb, a.T);
  const int nrows = min(kScoreRowsPerCta, a.T - rb);
  const int nj = (nrows + 1) >> 1;
  const int vmax = a.vis0 + rb + nrows - 1;               // cells the block's last row sees
  const int R = max(kPsStride, (vmax + kPsSamples - 1) / kPsSamples);  // sample stride
  const int ns = (vmax + R - 1) / R;                      // sampled cells j * R < vmax
  constexpr int kStep = (kPsThreads / 32) * 16;  // samples the CTA's warps take per round
  auto key = [&](int s) {
    return s < ns ? reinterpret_cast<const uint4*>(a.keys + static_cast<size_t>(s) * R * kDI) : nullptr;
  };
  // the keys of the next two rounds are in flight while one round is scored
  GemvKeys K0 = gemv_load_keys(key(warp * 16 + g), key(warp * 16 + g + 8));
  GemvKeys K1 = gemv_load_keys(key(warp * 16 + kStep + g), key(warp * 16 + kStep + g + 8));
  for (int base = warp * 16; base < ns; base += kStep) {
    const int s0 = base + g, s1 = base + g + 8;
    const GemvKeys K2 = gemv_load_keys(key(base + 2 * kStep + g), key(base + 2 * kStep + g + 8));
    float sc[4];
    gemv_mma(Q, K0, w, nj, sc);
    K0 = K1;
    K1 = K2;
    const int slot = (t & 1) ? s1 : s0;
    const int cell = slot * R;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int r = 2 * j + (t >> 1);
      if (j < nj && r < nrows && slot < ns && cell < a.vis0 + rb + r)
        atomicAdd(&ps_hist[r * kBins + score_bin(sc[j])], 1u);
    }
  }
  __syncthreads();
  if (warp < nrows) {  // one warp per row
    const int row = rb + warp;
    const int V = a.vis0 + row;
    float thr;
    if (V <= a.top_k) {
      thr = INFINITY;  // every visible cell is selected: no candidates needed
    } else {
      const int nsr = (V + R - 1) / R;  // this row's samples
      const float e = static_cast<float>(a.top_k) / R;
      const int need = static_cast<int>(ceilf(e + 6.f * sqrtf(e))) + 16;
      if (nsr <= need) thr = -INFINITY;  // too few samples to judge: every visible cell
      else thr = bin_floor(warp_find_bin(ps_hist + warp * kBins, kBins, static_cast<uint32_t>(need)));
    }
    if (lane == 0) a.thr[row] = thr;
  }
}

// ---------------------------------------------------------------- 2. scores and candidates

struct __align__(8) SsBarriers {
  uint64_t key_full[kSsStages];
  uint64_t key_empty[kSsStages];
  uint64_t q_full;
  uint64_t q_empty;
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t seg_done[2];   // every epilogue warp finished appending to segment s
  uint64_t drain;
  uint32_t tmem_base;
  uint32_t abort;
};

// fp32 accumulate, fp16 A (keys) and B (queries), both K-major, M = 128, N = 256.
constexpr uint32_t kSsIdesc = umma_idesc_f16(kSsCells, kSsN, false, false);

// grid: a.grid (persistent, one CTA per SM); block: kSsThreads; dynamic smem: kSsSmemBytes.
// Warp 0 issues the TMA loads, warp 1 owns TMEM and issues the MMAs, warps 2..17 are the
// epilogue: warp w reads TMEM lanes 32 (w % 4) .. + 31 (cells) and columns
// 64 ((w - 2) / 4) .. + 63 (16 tokens x 4 heads).
__global__ void __launch_bounds__(kSsThreads, 1)
    score_select_kernel(const __grid_constant__ CUtensorMap tmap_key, const __grid_constant__ CUtensorMap tmap_q,
                        PrefillSel a) {
  extern __shared__ __align__(1024) unsigned char ss_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(ss_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* sQ = base;                                  // 256 (token, head) rows x 128 B
  unsigned char* sK = base + kSsQBytes;                      // stages x 128 cells x 128 B
  float* table = reinterpret_cast<float*>(sK + kSsStages * kSsKeyBytes);  // [16 warps][16 tokens][8]
  uint32_t* cnt = reinterpret_cast<uint32_t*>(table + kSsEpiWarps * 16 * kSsTable);  // [2][64]
  float* stage = reinterpret_cast<float*>(cnt + 2 * kSsTokens);  // [16 warps][16 tokens][32 lanes] scores
  uint32_t* ballots = reinterpret_cast<uint32_t*>(stage + kSsEpiWarps * 16 * 32);  // [16 warps][16 tokens]
  SsBarriers& bar = *reinterpret_cast<SsBarriers*>(ballots + kSsEpiWarps * 16);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.x;
  const int it0 = min(a.items, b * a.per);
  const int it1 = min(a.items, it0 + a.per);
  const int tb0 = it0 / a.n_ct;
  int tiles0, tiles1;
  ss_segments(b, a.per, a.items, a.n_ct, tiles0, tiles1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSsStages; ++s) {
      mbar_init(&bar.key_full[s], 1);
      mbar_init(&bar.key_empty[s], 1);
    }
    mbar_init(&bar.q_full, 1);
    mbar_init(&bar.q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar.acc_full[i], 1);
      mbar_init(&bar.acc_empty[i], kSsEpiWarps);
      mbar_init(&bar.seg_done[i], kSsEpiWarps);
    }
    mbar_init(&bar.drain, 1);
    bar.abort = 0u;
    mbar_init_fence();
  }
  for (int i = threadIdx.x; i < 2 * kSsTokens; i += kSsThreads) cnt[i] = 0u;
  if (warp == 1) tmem_alloc(&bar.tmem_base, 512u);  // two accumulators of 256 columns
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar.tmem_base;
  griddep_launch();
  griddep_wait();  // thresholds come from the kernel before; keys may come from a cache write

  if (warp == 0) {
    // ---------------- TMA producer
    if (lane == 0) {
      int cur_tb = -1, q_loads = 0, li = 0;
      bool ok = true;
      for (int it = it0; it < it1 && ok; ++it) {
        const int tb = it / a.n_ct, ct = it % a.n_ct;
        if (ct >= ss_live_tiles(a, tb)) continue;
        if (tb != cur_tb) {
          if (q_loads > 0) ok = mbar_wait(&bar.q_empty, (q_loads - 1) & 1, &bar.abort, a.status);
          if (!ok) break;
          mbar_expect_tx(&bar.q_full, kSsQBytes);
          tma_load_2d(sQ, &tmap_q, 0, tb * kSsN, &bar.q_full);
          cur_tb = tb;
          ++q_loads;
        }
        const int s = li % kSsStages, round = li / kSsStages;
        ok = mbar_wait(&bar.key_empty[s], (round & 1) ^ 1, &bar.abort, a.status);
        if (!ok) break;
        mbar_expect_tx(&bar.key_full[s], kSsKeyBytes);
        tma_load_2d(sK + s * kSsKeyBytes, &tmap_key, 0, ct * kSsCells, &bar.key_full[s]);
        ++li;
      }
      if (!ok) {  // drain copies still in flight before the CTA leaves
        for (int i = max(0, li - kSsStages); i < li; ++i)
          mbar_drain_wait(&bar.key_full[i % kSsStages], (i / kSsStages) & 1);
        if (q_loads > 0) mbar_drain_wait(&bar.q_full, (q_loads - 1) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      int cur_tb = -1, q_loads = 0, li = 0;
      bool ok = true;
      for (int it = it0; it < it1 && ok; ++it) {
        const int tb = it / a.n_ct, ct = it % a.n_ct;
        const int live = ss_live_tiles(a, tb);
        if (ct >= live) continue;
        if (tb != cur_tb) {
          ok = mbar_wait(&bar.q_full, q_loads & 1, &bar.abort, a.status);
          if (!ok) break;
          cur_tb = tb;
          ++q_loads;
        }
        const int s = li % kSsStages, round = li / kSsStages;
        const int buf = li & 1, bround = li >> 1;
        ok = mbar_wait(&bar.key_full[s], round & 1, &bar.abort, a.status) &&
             mbar_wait(&bar.acc_empty[buf], (bround & 1) ^ 1, &bar.abort, a.status);
        if (!ok) break;
        tc_fence_after();
        const uint32_t ka = smem_u32(sK + s * kSsKeyBytes), qa = smem_u32(sQ);
        const uint32_t d = tmem + static_cast<uint32_t>(buf * kSsN);
#pragma unroll
        for (int ks = 0; ks < kDI / 16; ++ks)
          umma_f16(d, umma_desc_k_sw128(ka + ks * 32, 1024), umma_desc_k_sw128(qa + ks * 32, 1024), kSsIdesc,
                   ks > 0 ? 1u : 0u);
        umma_commit(&bar.key_empty[s]);    // the key stage is free once these MMAs finish
        umma_commit(&bar.acc_full[buf]);   // the accumulator is ready for the epilogue
        // the query block is free after the block's last live tile in this CTA's range
        const int next = it + 1;
        if (next >= it1 || next / a.n_ct != tb || next % a.n_ct >= live) umma_commit(&bar.q_empty);
        ++li;
      }
      umma_commit(&bar.drain);  // every MMA this thread issued has completed once it fires
      mbar_drain_wait(&bar.drain, 0);
    }
    __syncwarp();
  } else {
    // ---------------- epilogue
    const int e = warp - 2;
    const int quad = warp & 3;            // TMEM lanes 32 quad .. + 31: this warp's cells
    const int cq = e >> 2;                // columns 64 cq .. + 63: tokens 16 cq .. + 15 of the block
    float* tab = table + e * 16 * kSsTable;
    float* stw = stage + e * 16 * 32;  // this warp's scores, [token][lane]
    uint32_t* balw = ballots + e * 16;  // this warp's ballots, [token]
    int cur_tb = -1, li = 0;
    bool ok = true;
    for (int it = it0; it < it1 && ok; ++it) {
      const int tb = it / a.n_ct, ct = it % a.n_ct;
      if (tb != cur_tb) {
        if (cur_tb >= 0) {  // segment 0 is complete for this warp
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar.seg_done[0]);
        }
        // this warp's 16 tokens: weights, threshold, visible cells (0 past the chunk)
        if (lane < 16) {
          const int tok = tb * kSsTokens + 16 * cq + lane;
          const bool in = tok < a.T;
          const float4 wv = in ? __ldg(reinterpret_cast<const float4*>(a.iw) + tok) : make_float4(0.f, 0.f, 0.f, 0.f);
          float* r = tab + lane * kSsTable;
          r[0] = wv.x;
          r[1] = wv.y;
          r[2] = wv.z;
          r[3] = wv.w;
          r[4] = in ? __ldcg(a.thr + tok) : INFINITY;
          r[5] = __int_as_float(in ? a.vis0 + tok : 0);
          // first entry of this token's list in the block's segment
          const size_t lb = ss_list_base(b, tb - tb0, 16 * cq + lane, a.per, tiles0, tiles1);
          r[6] = __uint_as_float(static_cast<uint32_t>(lb));
          r[7] = __uint_as_float(static_cast<uint32_t>(lb >> 32));
        }
        __syncwarp();
        cur_tb = tb;
      }
      if (ct >= ss_live_tiles(a, tb)) continue;
      const int seg = tb - tb0;
      const int cap = ss_cap(seg ? tiles1 : tiles0);
      const int buf = li & 1, bround = li >> 1;
      ++li;
      if (!mbar_wait_warp(&bar.acc_full[buf], bround & 1, &bar.abort, a.status)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int cell = ct * kSsCells + quad * 32 + lane;
      uint32_t* seg_cnt = cnt + seg * kSsTokens;
      // Scores of the warp's 32 cells for its 16 tokens (two TMEM loads of 8 tokens x 4
      // heads), two tokens at a time in packed fp32 (the same fma chain per token), staged in
      // shared memory for the candidate writes; each token's ballot of candidates goes to
      // shared memory too (lane t reads token t's), every lane keeps the set of tokens its
      // cell is a candidate of.
      uint32_t mine = 0u;
      uint32_t rr[2][16];
#pragma unroll
      for (int tp = 0; tp < 8; ++tp) {
        if ((tp & 3) == 0) {  // columns of tokens 2 tp .. 2 tp + 7
#pragma unroll
          for (int c = 0; c < 2; ++c)
            tmem_ld16(tmem + (static_cast<uint32_t>(quad * 32) << 16) +
                          static_cast<uint32_t>(buf * kSsN + 64 * cq + 16 * (2 * (tp >> 2) + c)),
                      rr[c]);
          tmem_ld_wait();
          if (tp == 4) {  // the accumulator is in registers: hand it back to the MMA warp
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar.acc_empty[buf]);
          }
        }
        const int ta = 2 * tp, tb2 = ta + 1;
        const float4 wa = *reinterpret_cast<const float4*>(tab + ta * kSsTable);
        const float4 wb = *reinterpret_cast<const float4*>(tab + tb2 * kSsTable);
        const uint32_t* da = &rr[(ta >> 2) & 1][(ta & 3) * 4];
        const uint32_t* db = &rr[(tb2 >> 2) & 1][(tb2 & 3) * 4];
        float2 x = __fmul2_rn(make_float2(wa.x, wb.x), make_float2(fmaxf(__uint_as_float(da[0]), 0.f),
                                                                   fmaxf(__uint_as_float(db[0]), 0.f)));
        x = __ffma2_rn(make_float2(wa.y, wb.y),
                       make_float2(fmaxf(__uint_as_float(da[1]), 0.f), fmaxf(__uint_as_float(db[1]), 0.f)), x);
        x = __ffma2_rn(make_float2(wa.z, wb.z),
                       make_float2(fmaxf(__uint_as_float(da[2]), 0.f), fmaxf(__uint_as_float(db[2]), 0.f)), x);
        x = __ffma2_rn(make_float2(wa.w, wb.w),
                       make_float2(fmaxf(__uint_as_float(da[3]), 0.f), fmaxf(__uint_as_float(db[3]), 0.f)), x);
        stw[ta * 32 + lane] = x.x;
        stw[tb2 * 32 + lane] = x.y;
        const float2 ta_tv = *reinterpret_cast<const float2*>(tab + ta * kSsTable + 4);   // threshold, V
        const float2 tb_tv = *reinterpret_cast<const float2*>(tab + tb2 * kSsTable + 4);
        const bool ha = cell < __float_as_int(ta_tv.y) && x.x >= ta_tv.x;
        const bool hb = cell < __float_as_int(tb_tv.y) && x.y >= tb_tv.x;
        const uint32_t ma = __ballot_sync(0xffffffffu, ha), mb = __ballot_sync(0xffffffffu, hb);
        if (lane == 0) {
          balw[ta] = ma;
          balw[tb2] = mb;
        }
        mine |= (ha ? 1u : 0u) << ta;
        mine |= (hb ? 1u : 0u) << tb2;
      }
      __syncwarp();
      const uint32_t my_hits = lane < 16 ? balw[lane] : 0u;
      // one round of shared-memory atomics reserves every token's slots
      uint32_t my_base = 0u;
      if (lane < 16 && my_hits) my_base = atomicAdd(&seg_cnt[16 * cq + lane], static_cast<uint32_t>(__popc(my_hits)));
      const uint32_t below = (1u << lane) - 1u;
      // each lane writes its own candidates, one token per step (as many steps as the most
      // any lane has)
      while (__any_sync(0xffffffffu, mine != 0u)) {
        const int tl = mine ? __ffs(mine) - 1 : 0;
        const uint32_t m = __shfl_sync(0xffffffffu, my_hits, tl);
        const uint32_t base = __shfl_sync(0xffffffffu, my_base, tl);
        if (mine) {
          mine &= mine - 1u;
          const uint32_t slot = base + __popc(m & below);
          if (slot < static_cast<uint32_t>(cap)) {
            const float v = stw[tl * 32 + lane];
            const uint2 lb2 = *reinterpret_cast<const uint2*>(tab + tl * kSsTable + 6);
            const size_t lb = (static_cast<size_t>(lb2.y) << 32) | lb2.x;
            a.cand[lb + slot] = make_uint2(score_key(v), static_cast<uint32_t>(cell));
          }
        }
      }
    }
    // the last segment is complete for this warp
    __syncwarp();
    if (lane == 0 && cur_tb >= 0) mbar_arrive(&bar.seg_done[cur_tb - tb0]);
    // warp 2 publishes each segment's counts once every epilogue warp is done with it
    if (e == 0 && cur_tb >= 0) {
      for (int s = 0; s <= cur_tb - tb0; ++s) {
        if (!mbar_wait_warp(&bar.seg_done[s], 0, &bar.abort, a.status)) break;
        for (int i = lane; i < kSsTokens; i += 32)
          a.seg_count[(static_cast<size_t>(b) * 2 + s) * kSsTokens + i] = cnt[s * kSsTokens + i];
      }
    }
    (void)ok;
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512u);
}

// ---------------------------------------------------------------- 3. exact selection

// Exact radix select over n keys in shared memory: the key of the need-th largest
// (thr) and how many keys equal to it are kept (take).  NT threads.
template <int NT>
__device__ void smem_radix_select(const uint32_t* keys, int n, uint32_t need, SelectSmem& sm, uint32_t& thr,
                                  uint32_t& take) {
  const int tid = threadIdx.x;
  uint32_t k_and = 0xffffffffu, k_or = 0u;
  for (int i = tid; i < n; i += NT) {
    k_and &= keys[i];
    k_or |= keys[i];
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
  while (top >= 0) {
    const int shift = top >= 7 ? top - 7 : 0;
    const uint32_t wm = (2u << (top - shift)) - 1u;
    for (int i = tid; i < 256; i += NT) sm.h256[i] = 0u;
    __syncthreads();
    for (int i = tid; i < n; i += NT) {
      const uint32_t k = keys[i];
      if ((k & mask) == prefix) atomicAdd(&sm.h256[(k >> shift) & wm], 1u);
    }
    __syncthreads();
    uint32_t digit, above;
    find_threshold_bin<NT>(sm.h256, 256, need, sm.scratch, sm.result, digit, above);
    need -= above;
    prefix |= digit << shift;
    mask |= wm << shift;
    top = shift - 1;
  }
  thr = prefix;
  take = need;
}

// Ascending ids of the selected cells from the window bitmaps of [w0, w0 + wn): the
// selected (selb) plus the first `take_eq - eq_taken` ties (eqb) in index order.
template <int NT>
__device__ void emit_window(uint32_t* selb, const uint32_t* eqb, int w0, int wn, uint32_t take_eq,
                            uint32_t& eq_taken, uint32_t& out_base, int top_k, SelectSmem& sm,
                            int32_t* __restrict__ out) {
  const int tid = threadIdx.x;
  const int words = (wn + 31) >> 5;
  const int per = (words + NT - 1) / NT;
  const int wb = tid * per, we = min(words, wb + per);
  uint32_t c = 0u;
  for (int i = wb; i < we; ++i) c += __popc(eqb[i]);
  uint32_t tot;
  uint32_t rank = eq_taken + block_exclusive_scan<NT>(c, sm.scratch, tot);
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
  c = 0u;
  for (int i = wb; i < we; ++i) c += __popc(selb[i]);
  uint32_t pos = out_base + block_exclusive_scan<NT>(c, sm.scratch, tot);
  for (int i = wb; i < we; ++i) {
    uint32_t bits = selb[i];
    while (bits) {
      const int bit = __ffs(bits) - 1;
      bits &= bits - 1u;
      if (pos < static_cast<uint32_t>(top_k)) out[pos] = w0 + i * 32 + bit;
      ++pos;
    }
  }
  out_base += tot;
  __syncthreads();
}

// Scores of one row recomputed for 16 cells per warp step (the decode GEMV's arithmetic).
// For lanes t < 2 (the row's lanes), `sc` is the score of cell `base + g + 8 t`.
struct RowGemv {
  GemvQ Q;
  float w[4][2];
};

__device__ __forceinline__ float row_score(const RowGemv& R, const __half* keys, int base, int V, int& cell) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int c0 = base + g, c1 = base + g + 8;
  float sc[4];
  gemv_scores(R.Q, c0 < V ? reinterpret_cast<const uint4*>(keys + static_cast<size_t>(c0) * kDI) : nullptr,
              c1 < V ? reinterpret_cast<const uint4*>(keys + static_cast<size_t>(c1) * kDI) : nullptr, R.w, 1, sc);
  cell = (t & 1) ? c1 : c0;
  if (t >= 2 || cell >= V) cell = -1;  // lanes t >= 2 hold the (empty) second row
  return sc[0];
}

// grid: T; block: kPfThreads; dynamic smem: kPfSmemBytes.
__global__ void __launch_bounds__(kPfThreads, 2) prefill_final_kernel(PrefillSel a, int32_t* __restrict__ ids) {
  extern __shared__ uint32_t pf_smem[];
  uint32_t* ckey = pf_smem;                  // [kPfCand]
  uint32_t* ccell = ckey + kPfCand;          // [kPfCand]
  uint32_t* selb = ccell + kPfCand;          // [kPfWinBits / 32]
  uint32_t* eqb = selb + kPfWinBits / 32;    // [kPfWinBits / 32]
  __shared__ SelectSmem sm;
  __shared__ uint32_t seg_off[kPfMaxSegs + 1];
  __shared__ uint64_t seg_base[kPfMaxSegs];
  __shared__ uint32_t s_bad;
  __shared__ __align__(16) uint32_t s_iq[kScoreRowsPerCta * kHI * kScoreIqWords];
  constexpr int NT = kPfThreads;
  const int tid = threadIdx.x;
  griddep_launch();
  griddep_wait();  // the lists and counts come from the GEMM
  const int row = blockIdx.x;
  const int V = a.vis0 + row;
  int32_t* out = ids + static_cast<size_t>(row) * a.top_k;
  if (V <= a.top_k) {  // every visible cell, ascending
    for (int i = tid; i < a.top_k; i += NT) out[i] = i < V ? i : -1;
    return;
  }
  const int tb = row / kSsTokens, tl = row % kSsTokens;
  const int last_cta = (a.items - 1) / a.per;
  const int b_lo = (tb * a.n_ct) / a.per;
  const int b_hi = min(last_cta, ((tb + 1) * a.n_ct - 1) / a.per);
  const int nseg = b_hi - b_lo + 1;
  if (tid == 0) s_bad = nseg > kPfMaxSegs ? 1u : 0u;
  __syncthreads();
  if (tid < nseg && tid < kPfMaxSegs) {
    const int bb = b_lo + tid;
    int t0, t1;
    ss_segments(bb, a.per, a.items, a.n_ct, t0, t1);
    const int s = tb - (bb * a.per) / a.n_ct;
    const uint32_t n = __ldcg(a.seg_count + (static_cast<size_t>(bb) * 2 + s) * kSsTokens + tl);
    if (n > static_cast<uint32_t>(ss_cap(s ? t1 : t0))) atomicOr(&s_bad, 1u);  // a list overflowed
    seg_base[tid] = ss_list_base(bb, s, tl, a.per, t0, t1);
    seg_off[tid + 1] = n;
  }
  __syncthreads();
  if (tid == 0 && !s_bad) {
    seg_off[0] = 0u;
    for (int i = 0; i < nseg; ++i) seg_off[i + 1] += seg_off[i];
    const uint32_t total = seg_off[nseg];
    if (total < static_cast<uint32_t>(a.top_k) || total > static_cast<uint32_t>(kPfCand)) s_bad = 1u;
  }
  __syncthreads();

  uint32_t thr_key, take_eq;
  if (!s_bad) {
    // ---- the candidates: load, select exactly, emit in index order
    const int n = static_cast<int>(seg_off[nseg]);
    constexpr int kBatch = 8;  // loads in flight per thread before their stores
    for (int i0 = tid; i0 < n; i0 += NT * kBatch) {
      uint2 p[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int i = i0 + u * NT;
        if (i < n) {
          int s = 0;
          while (seg_off[s + 1] <= static_cast<uint32_t>(i)) ++s;
          p[u] = __ldcg(a.cand + seg_base[s] + (i - seg_off[s]));
        }
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int i = i0 + u * NT;
        if (i < n) {
          ckey[i] = p[u].x;
          ccell[i] = p[u].y;
        }
      }
    }
    __syncthreads();
    smem_radix_select<NT>(ckey, n, static_cast<uint32_t>(a.top_k), sm, thr_key, take_eq);
    uint32_t out_base = 0u, eq_taken = 0u;
    for (int w0 = 0; w0 < V; w0 += kPfWinBits) {
      const int wn = min(kPfWinBits, V - w0);
      const int words = (wn + 31) >> 5;
      for (int i = tid; i < words; i += NT) {
        selb[i] = 0u;
        eqb[i] = 0u;
      }
      __syncthreads();
      for (int i = tid; i < n; i += NT) {
        const int c = static_cast<int>(ccell[i]) - w0;
        if (c < 0 || c >= wn) continue;
        if (ckey[i] > thr_key) atomicOr(&selb[c >> 5], 1u << (c & 31));
        else if (ckey[i] == thr_key) atomicOr(&eqb[c >> 5], 1u << (c & 31));
      }
      __syncthreads();
      emit_window<NT>(selb, eqb, w0, wn, take_eq, eq_taken, out_base, a.top_k, sm, out);
    }
    for (uint32_t i = out_base + tid; i < static_cast<uint32_t>(a.top_k); i += NT) out[i] = -1;
    return;
  }

  // ---- fallback: exact radix select over every visible cell, scores recomputed per pass
  gemv_stage_q<NT>(s_iq, a.iq, row, row + 1);  // this row alone (the block's other rows zero)
  __syncthreads();
  RowGemv R;
  gemv_load_q(R.Q, s_iq);
  gemv_load_w(R.w, a.iw, row, row + 1);
  const int warp = tid >> 5;
  uint32_t prefix = 0u, mask = 0u, need = static_cast<uint32_t>(a.top_k);
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += NT) sm.h256[i] = 0u;
    __syncthreads();
    for (int base = warp * 16; base < V; base += (NT / 32) * 16) {
      int cell;
      const float sc = row_score(R, a.keys, base, V, cell);
      const uint32_t k = score_key(sc);
      if (cell >= 0 && (k & mask) == prefix) atomicAdd(&sm.h256[(k >> shift) & 255u], 1u);
    }
    __syncthreads();
    uint32_t digit, above;
    find_threshold_bin<NT>(sm.h256, 256, need, sm.scratch, sm.result, digit, above);
    need -= above;
    prefix |= digit << shift;
    mask |= 255u << shift;
  }
  thr_key = prefix;
  take_eq = need;
  uint32_t out_base = 0u, eq_taken = 0u;
  for (int w0 = 0; w0 < V; w0 += kPfWinBits) {
    const int wn = min(kPfWinBits, V - w0);
    const int words = (wn + 31) >> 5;
    for (int i = tid; i < words; i += NT) {
      selb[i] = 0u;
      eqb[i] = 0u;
    }
    __syncthreads();
    for (int base = w0 + warp * 16; base < w0 + wn; base += (NT / 32) * 16) {
      int cell;
      const float sc = row_score(R, a.keys, base, w0 + wn, cell);
      if (cell < 0) continue;
      const uint32_t k = score_key(sc);
      const int c = cell - w0;
      if (k > thr_key) atomicOr(&selb[c >> 5], 1u << (c & 31));
      else if (k == thr_key) atomicOr(&eqb[c >> 5], 1u << (c & 31));
    }
    __syncthreads();
    emit_window<NT>(selb, eqb, w0, wn, take_eq, eq_taken, out_base, a.top_k, sm, out);
  }
  for (uint32_t i = out_base + tid; i < static_cast<uint32_t>(a.top_k); i += NT) out[i] = -1;
}

}  // namespace qsa
