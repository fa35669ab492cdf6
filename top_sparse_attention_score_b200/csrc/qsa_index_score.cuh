// qsa_index_score.cuh -- indexer scores of every cell for a block of query rows.
//
// score[r][c] = sum_h w[r][h] * max(0, sum_d iq[r][h][d] * key[c][d]), 4 heads x 64 dims,
// the indexer of "opus r20 track A: MTP map mlock + qsa_attn / qsa_merge decode tweaks"
// (section 3, "indexer q") in the matrix form the prompt path calls qsa_score_mm
// ("opus r15 track A: prompt_chunk wave zipping, ...", what changed, item 1).
//
// Tensor-core GEMV/GEMM on mma.sync m16n8k16: the 16 A rows are cells (keys
// streamed once from HBM with 16-byte loads that use every sector), the N
// columns are (row, head) pairs, K = 64.  Products of fp16 are exact in fp32,
// and every cell runs the same instruction sequence, so equal keys always get
// bit-equal scores (the selection's tie rule relies on that).
//
// A decode call that appends its own cells hands them to this kernel: extra CTAs
// quantize the new cells into the cache (the cache write's arithmetic), and the
// scoring CTAs read the new cells' keys from the caller's buffer, since the cache
// copies are written by other CTAs of the same launch.
#pragma once

#include "qsa_cache_write.cuh"
#include "qsa_common.cuh"

namespace qsa {

constexpr int kScoreCellsPerWarp = 16;
constexpr int kScoreWarps = 4;
constexpr int kScoreCellsPerCta = kScoreCellsPerWarp * kScoreWarps;
constexpr int kScoreRowsPerCta = 8;  // 8 rows x 4 heads = 32 columns = 4 n-tiles

// Cells appended by the same call: cells [from, from + n) of the cache get the
// quantized k / v rows and the keys given here.
struct ScoreAppend {
  const float* k;      // [n][2][256] fp32
  const float* v;      // [n][2][256] fp32
  const __half* key;   // [n][64] fp16
  int8_t* kc;          // the cache arrays
  int8_t* vc;
  __half* ks;
  __half* vs;
  __half* idx_key;
  int from;
  int n;               // 0: nothing appended
};

// Staged (row, head) queries are 34 words apart (64 fp16 + 4 of padding, fewer bank
// conflicts); every access is an 8-byte one at an even word.
constexpr int kScoreIqWords = 34;

// ---- one warp's 16-cell step of the GEMV, shared with the prompt selection kernels
//
// K index <-> dim mapping (the contraction may permute dims as long as A and B
// agree): thread t owns dims [8t, 8t+8) and [32+8t, 32+8t+8) of each key; k-step
// ks covers, for thread t, dims d0..d0+3 with d0 = 32*(ks/2) + 8t + 4*(ks%2):
// k-index 2t,2t+1 <-> d0,d0+1 and 2t+8,2t+9 <-> d0+2,d0+3.  N columns: n-tile j
// holds rows 2j, 2j+1 of the block (4 heads each).

struct GemvQ {
  uint32_t b[4][4][2];  // B fragments of the 8 x 4 staged (row, head) queries
};

// From the block's queries staged as kScoreIqWords-word rows per (row, head).
__device__ __forceinline__ void gemv_load_q(GemvQ& Q, const uint32_t* s_iq) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int rh = (2 * j + (g >> 2)) * kHI + (g & 3);  // (row 2j + g/4, head g%4)
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      const int d0 = 32 * (ks >> 1) + 8 * t + 4 * (ks & 1);
      const uint2 v = *reinterpret_cast<const uint2*>(&s_iq[rh * kScoreIqWords + d0 / 2]);
      Q.b[j][ks][0] = v.x;
      Q.b[j][ks][1] = v.y;
    }
  }
}

// Head weights this lane applies: w[j] = weights of heads 2(t%2), 2(t%2)+1 of row rb + 2j + t/2.
__device__ __forceinline__ void gemv_load_w(float (&w)[4][2], const float* __restrict__ iw, int rb, int rows) {
  const int t = threadIdx.x & 3;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int row = rb + 2 * j + (t >> 1), h0 = 2 * (t & 1);
    const bool ok = row < rows;
    w[j][0] = ok ? __ldg(iw + row * kHI + h0) : 0.f;
    w[j][1] = ok ? __ldg(iw + row * kHI + h0 + 1) : 0.f;
  }
}

// This lane's parts of the warp's 16 keys: cell slot g (k0) and slot g + 8 (k1).
struct GemvKeys {
  uint4 a0h0, a0h1, a1h0, a1h1;
};

// Key rows k0 and k1 (NULL for no cell: zeros).
__device__ __forceinline__ GemvKeys gemv_load_keys(const uint4* k0, const uint4* k1) {
  const int t = threadIdx.x & 3;
  GemvKeys K;
  K.a0h0 = K.a0h1 = K.a1h0 = K.a1h1 = make_uint4(0, 0, 0, 0);
  if (k0) {
    K.a0h0 = __ldg(k0 + t);
    K.a0h1 = __ldg(k0 + 4 + t);
  }
  if (k1) {
    K.a1h0 = __ldg(k1 + t);
    K.a1h1 = __ldg(k1 + 4 + t);
  }
  return K;
}

// Scores of the warp's 16 cells for n-tiles j < nj (warp-uniform).  sc[j] = score of
// (row 2j + t/2 of the block, cell slot g + 8 (t % 2)).  The ReLU-weighted head sum
// runs in the same order on every lane, so equal keys always get bit-equal scores.
__device__ __forceinline__ void gemv_mma(const GemvQ& Q, const GemvKeys& K, const float (&w)[4][2], int nj,
                                         float (&sc)[4]) {
  const int t = threadIdx.x & 3;
  uint32_t a[4][4];
  a[0][0] = K.a0h0.x; a[0][2] = K.a0h0.y; a[0][1] = K.a1h0.x; a[0][3] = K.a1h0.y;
  a[1][0] = K.a0h0.z; a[1][2] = K.a0h0.w; a[1][1] = K.a1h0.z; a[1][3] = K.a1h0.w;
  a[2][0] = K.a0h1.x; a[2][2] = K.a0h1.y; a[2][1] = K.a1h1.x; a[2][3] = K.a1h1.y;
  a[3][0] = K.a0h1.z; a[3][2] = K.a0h1.w; a[3][1] = K.a1h1.z; a[3][3] = K.a1h1.w;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    sc[j] = 0.f;
    if (j >= nj) continue;  // warp-uniform
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) mma_f16_16816(acc, a[ks], Q.b[j][ks][0], Q.b[j][ks][1]);
    // columns 2t, 2t+1 of n-tile j: row 2j + t/2, heads 2(t%2), 2(t%2)+1
    const float pg = w[j][0] * fmaxf(acc[0], 0.f) + w[j][1] * fmaxf(acc[1], 0.f);
    const float p8 = w[j][0] * fmaxf(acc[2], 0.f) + w[j][1] * fmaxf(acc[3], 0.f);
    const float og = __shfl_xor_sync(0xffffffffu, pg, 1);
    const float o8 = __shfl_xor_sync(0xffffffffu, p8, 1);
    // heads {0,1} + heads {2,3} in the same order on both lanes of the pair
    sc[j] = (t & 1) ? (o8 + p8) : (pg + og);
  }
}

// Both steps at once: key rows k0 (cell slot g) and k1 (slot g + 8), NULL for no cell.
__device__ __forceinline__ void gemv_scores(const GemvQ& Q, const uint4* k0, const uint4* k1,
                                            const float (&w)[4][2], int nj, float (&sc)[4]) {
  gemv_mma(Q, gemv_load_keys(k0, k1), w, nj, sc);
}

// Stage the queries of rows [rb, rb + 8) (fewer past `rows`; zeros there) with 16-byte loads.
template <int NT>
__device__ __forceinline__ void gemv_stage_q(uint32_t* s_iq, const __half* __restrict__ iq, int rb, int rows) {
  const int nrow = min(kScoreRowsPerCta, rows - rb);
  const uint4* src = reinterpret_cast<const uint4*>(iq + static_cast<size_t>(rb) * kHI * kDI);
  for (int i = threadIdx.x; i < kScoreRowsPerCta * kHI * 8; i += NT) {  // 8 chunks of 16 B per (row, head)
    const int rh = i >> 3, ch = i & 7;
    const uint4 v = rh < nrow * kHI ? __ldg(src + i) : make_uint4(0, 0, 0, 0);
    uint32_t* dst = &s_iq[rh * kScoreIqWords + ch * 4];
    *reinterpret_cast<uint2*>(dst) = make_uint2(v.x, v.y);
    *reinterpret_cast<uint2*>(dst + 2) = make_uint2(v.z, v.w);
  }
}

// Scoring CTAs of the decode GEMV for `ncells` cells: enough that every SM runs a few
// warps, each of which then walks many 16-cell groups with the next group's keys in
// flight while it multiplies the current one.
constexpr int kScoreGroupsPerWarp = 2;
__host__ __device__ inline int score_ctas_for(int ncells, int sms) {
  const int groups = (ncells + kScoreCellsPerWarp - 1) / kScoreCellsPerWarp;
  const int want = (groups + kScoreWarps * kScoreGroupsPerWarp - 1) / (kScoreWarps * kScoreGroupsPerWarp);
  return max(1, min(want, 4 * sms));
}

// grid: x = score_ctas + 4 * app.n, y = ceil(rows / 8); block: 128 threads.
__global__ void __launch_bounds__(128) index_score_kernel(const __half* __restrict__ keys,
                                                          int ncells,
                                                          const __half* __restrict__ iq,
                                                          const float* __restrict__ iw, int rows,
                                                          float* __restrict__ scores, int64_t ld,
                                                          ScoreAppend app, int score_ctas) {
  // the block's (row, head) queries, 8 x 4 x 64 fp16, staged once with 16-byte loads
  __shared__ __align__(16) uint32_t s_iq[kScoreRowsPerCta * kHI * kScoreIqWords];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int rb = blockIdx.y * kScoreRowsPerCta;
  griddep_launch();
  if (static_cast<int>(blockIdx.x) >= score_ctas) {
    // quantizer CTA: one (new cell, KV head, K or V) row of 256 values
    griddep_wait();  // earlier kernels on the stream may still read the cells rewritten here
    if (blockIdx.y != 0) return;
    const int j = blockIdx.x - score_ctas;
    const int i = j >> 2, kvh = (j >> 1) & 1, which = j & 1;
    const size_t row = (static_cast<size_t>(app.from) + i) * kHKV + kvh;
    quantize_row((which ? app.v : app.k) + (static_cast<size_t>(i) * kHKV + kvh) * kD,
                 (which ? app.vc : app.kc) + row * kD, (which ? app.vs : app.ks) + row * kNG, 128);
    if (kvh == 0 && which == 0 && threadIdx.x < kDI)
      app.idx_key[(static_cast<size_t>(app.from) + i) * kDI + threadIdx.x] =
          app.key[static_cast<size_t>(i) * kDI + threadIdx.x];
    return;
  }
  // Everything read before the grid-dependency wait is data no kernel of this library
  // writes while a dependent may already run: the caller's queries and weights, the
  // appended cells' keys (the caller's buffer) and the cache's keys (written only by the
  // cache write, which lets its dependents start only once it has completed).  So the
  // first loads overlap the previous kernel's tail; the score stores wait for it (the
  // previous call's selection may still read the scores).
  gemv_stage_q<128>(s_iq, iq, rb, rows);
  float w[4][2];
  gemv_load_w(w, iw, rb, rows);
  const int nj = (min(rows - rb, kScoreRowsPerCta) + 1) >> 1;
  // key of cell c: the cache, or the caller's buffer for the cells this call appends
  auto key_row = [&](int c) -> const uint4* {
    if (c >= ncells) return nullptr;
    return reinterpret_cast<const uint4*>(
        c >= app.from && c < app.from + app.n ? app.key + static_cast<size_t>(c - app.from) * kDI
                                               : keys + static_cast<size_t>(c) * kDI);
  };
  const int groups = (ncells + kScoreCellsPerWarp - 1) / kScoreCellsPerWarp;
  const int step = score_ctas * kScoreWarps;
  int grp = blockIdx.x * kScoreWarps + warp;
  // the keys of this warp's next two groups are in flight while one group is scored (rows of
  // many cells give each warp several groups)
  auto load = [&](int gr) {
    GemvKeys K;
    if (gr < groups) K = gemv_load_keys(key_row(gr * 16 + g), key_row(gr * 16 + g + 8));
    return K;
  };
  GemvKeys K0 = load(grp), K1 = load(grp + step);
  __syncthreads();
  GemvQ Q;
  gemv_load_q(Q, s_iq);
  griddep_wait();
  for (; grp < groups; grp += step) {
    const GemvKeys K2 = load(grp + 2 * step);
    float sc[4];
    gemv_mma(Q, K0, w, nj, sc);
    const int c = grp * 16 + g + 8 * (t & 1);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int row = rb + 2 * j + (t >> 1);
      if (j < nj && row < rows && c < ncells) scores[row * ld + c] = sc[j];
    }
    K0 = K1;
    K1 = K2;
  }
}

}  // namespace qsa
