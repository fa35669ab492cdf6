// qsa_merge.cuh -- log-sum-exp merge of split partials, with the optional output gate.
//
// The merge of qsa_merge ("opus r20 track A: MTP map mlock + qsa_attn / qsa_merge decode
// tweaks", section 2) rests on the log-sum-exp identity: piece j reports its maximum
// logit m_j, its weight sum l_j and its unnormalised output o_j, all relative to m_j;
// rescaled to the common maximum M = max_j m_j by e_j = exp(m_j - M), the pieces add
// up to L = sum_j l_j e_j and O = sum_j o_j e_j, and the attention output is O / L.
// Pieces without cells (l_j = 0) contribute nothing and do not set M.
//
// The optional gate multiplies the result by sigmoid(gate) elementwise ("attention +
// gate" in the same page's section 3).
//
// One CTA per (row, head), one thread per output dim.  Warp 0 reduces the piece
// statistics (two pieces per lane, warp-shuffle maximum and sum); every thread has
// its dim's 64 possible o_j loads in flight before the weights are known.
#pragma once

#include "qsa_common.cuh"

namespace qsa {

// grid: rows * 24 (one CTA per row and head); block: 256 threads (one per dim).
__global__ void __launch_bounds__(256) merge_kernel(const float* __restrict__ part, int nsplit,
                                                    const float* __restrict__ gate,
                                                    float* __restrict__ out) {
  __shared__ float s_e[64];  // e_j, 0 for empty pieces
  __shared__ float s_inv;    // 1 / L, 0 when every piece is empty
  const int tid = threadIdx.x;
  const size_t rh = blockIdx.x;
  const float* base = part + rh * nsplit * kPart;
  griddep_launch();
  griddep_wait();  // the partials come from the attention kernel
  float ov[64];
#pragma unroll
  for (int j = 0; j < 64; ++j) ov[j] = j < nsplit ? __ldcg(base + j * kPart + 2 + tid) : 0.f;
  const float g = gate ? __ldg(gate + rh * kD + tid) : 0.f;
  if (tid < 32) {
    float m[2], l[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int j = tid + 32 * u;
      m[u] = j < nsplit ? __ldcg(base + j * kPart) : -INFINITY;
      l[u] = j < nsplit ? __ldcg(base + j * kPart + 1) : 0.f;
    }
    float M = fmaxf(l[0] > 0.f ? m[0] : -INFINITY, l[1] > 0.f ? m[1] : -INFINITY);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float e[2], L = 0.f;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      e[u] = l[u] > 0.f ? expf(m[u] - M) : 0.f;
      L = fmaf(l[u], e[u], L);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
    s_e[tid] = e[0];
    s_e[tid + 32] = e[1];
    if (tid == 0) s_inv = L > 0.f ? 1.f / L : 0.f;
  }
  __syncthreads();
  float o = 0.f;
#pragma unroll
  for (int j = 0; j < 64; ++j)
    if (j < nsplit) o = fmaf(ov[j], s_e[j], o);
  float r = o * s_inv;
  if (gate) r *= gate_factor(g);
  out[rh * kD + tid] = r;
}

}  // namespace qsa
