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
#pragma once

#include "qsa_common.cuh"

namespace qsa {

constexpr int kScoreCellsPerWarp = 16;
constexpr int kScoreWarps = 4;
constexpr int kScoreCellsPerCta = kScoreCellsPerWarp * kScoreWarps;
constexpr int kScoreRowsPerCta = 8;  // 8 rows x 4 heads = 32 columns = 4 n-tiles

// grid: x = ceil(ncells / 64), y = ceil(rows / 8); block: 128 threads.
__global__ void __launch_bounds__(128) index_score_kernel(const __half* __restrict__ keys,
                                                          int ncells,
                                                          const __half* __restrict__ iq,
                                                          const float* __restrict__ iw, int rows,
                                                          float* __restrict__ scores, int64_t ld) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int cb = blockIdx.x * kScoreCellsPerCta + warp * kScoreCellsPerWarp;
  const int rb = blockIdx.y * kScoreRowsPerCta;
  griddep_launch();
  griddep_wait();  // keys may have just been written, scores may still be read by earlier kernels
  if (cb >= ncells) return;

  // K index <-> dim mapping (the contraction may permute dims as long as A and
  // B agree): thread t owns dims [8t, 8t+8) and [32+8t, 32+8t+8) of each key;
  // k-step ks covers, for thread t, dims d0..d0+3 with
  // d0 = 32*(ks/2) + 8t + 4*(ks%2): k-index 2t,2t+1 <-> d0,d0+1 and 2t+8,2t+9 <-> d0+2,d0+3.
  uint32_t b[4][4][2];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int row = rb + 2 * j + (g >> 2), head = g & 3;
    const bool ok = row < rows;
    const __half* src = iq + (static_cast<size_t>(ok ? row : 0) * kHI + head) * kDI;
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      const int d0 = 32 * (ks >> 1) + 8 * t + 4 * (ks & 1);
      b[j][ks][0] = ok ? *reinterpret_cast<const uint32_t*>(src + d0) : 0u;
      b[j][ks][1] = ok ? *reinterpret_cast<const uint32_t*>(src + d0 + 2) : 0u;
    }
  }

  const int c0 = cb + g, c1 = cb + g + 8;
  uint4 a0h0 = make_uint4(0, 0, 0, 0), a0h1 = a0h0, a1h0 = a0h0, a1h1 = a0h0;
  if (c0 < ncells) {
    const uint4* p = reinterpret_cast<const uint4*>(keys + static_cast<size_t>(c0) * kDI);
    a0h0 = __ldg(p + t);
    a0h1 = __ldg(p + 4 + t);
  }
  if (c1 < ncells) {
    const uint4* p = reinterpret_cast<const uint4*>(keys + static_cast<size_t>(c1) * kDI);
    a1h0 = __ldg(p + t);
    a1h1 = __ldg(p + 4 + t);
  }
  uint32_t a[4][4];
  a[0][0] = a0h0.x; a[0][2] = a0h0.y; a[0][1] = a1h0.x; a[0][3] = a1h0.y;
  a[1][0] = a0h0.z; a[1][2] = a0h0.w; a[1][1] = a1h0.z; a[1][3] = a1h0.w;
  a[2][0] = a0h1.x; a[2][2] = a0h1.y; a[2][1] = a1h1.x; a[2][3] = a1h1.y;
  a[3][0] = a0h1.z; a[3][2] = a0h1.w; a[3][1] = a1h1.z; a[3][3] = a1h1.w;

#pragma unroll
  for (int j = 0; j < 4; ++j) {
    if (rb + 2 * j >= rows) break;  // warp-uniform: n-tile j holds rows rb+2j, rb+2j+1
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) mma_f16_16816(acc, a[ks], b[j][ks][0], b[j][ks][1]);
    // columns 2t, 2t+1 of n-tile j: row rb + 2j + t/2, heads 2(t%2), 2(t%2)+1
    const int row = rb + 2 * j + (t >> 1);
    const int h0 = 2 * (t & 1);
    const bool rok = row < rows;
    const float w0 = rok ? __ldg(iw + row * kHI + h0) : 0.f;
    const float w1 = rok ? __ldg(iw + row * kHI + h0 + 1) : 0.f;
    const float pg = w0 * fmaxf(acc[0], 0.f) + w1 * fmaxf(acc[1], 0.f);
    const float p8 = w0 * fmaxf(acc[2], 0.f) + w1 * fmaxf(acc[3], 0.f);
    const float og = __shfl_xor_sync(0xffffffffu, pg, 1);
    const float o8 = __shfl_xor_sync(0xffffffffu, p8, 1);
    // heads {0,1} + heads {2,3} in the same order on both lanes of the pair
    const float sg = (t & 1) ? (og + pg) : (pg + og);
    const float s8 = (t & 1) ? (o8 + p8) : (p8 + o8);
    if (rok) {
      if ((t & 1) == 0) {
        if (c0 < ncells) scores[row * ld + c0] = sg;
      } else {
        if (c1 < ncells) scores[row * ld + c1] = s8;
      }
    }
  }
}

}  // namespace qsa
