// qsa_merge.cuh -- log-sum-exp merge of split partials.
//
// qsa_merge of "opus r20 track A: MTP map mlock + qsa_attn / qsa_merge decode tweaks",
// section 2: the chunk maxima are loaded once, M = max_k m_k, e_k = exp(m_k - M) is
// computed once per piece, L = sum_k l_k e_k is summed with fma in piece order by one
// thread, every thread accumulates o = sum_k o_k e_k with fma in piece order for its
// dim, and the result is o / L.  Pieces with l = 0 (no cells) are skipped.
#pragma once

#include "qsa_common.cuh"

namespace qsa {

// grid: rows * 24 (one CTA per row and head); block: 256 threads (one per dim).
__global__ void __launch_bounds__(256) merge_kernel(const float* __restrict__ part, int nsplit,
                                                    float* __restrict__ out) {
  __shared__ float sm[64], sl[64], se[64];
  __shared__ float sL;
  const int tid = threadIdx.x;
  const float* base = part + static_cast<size_t>(blockIdx.x) * nsplit * kPart;
  griddep_launch();
  griddep_wait();  // the partials come from the attention kernel
  // every o_j of this dim in flight at once (nsplit <= 64)
  float ov[64];
#pragma unroll
  for (int j = 0; j < 64; ++j) ov[j] = j < nsplit ? __ldcg(base + j * kPart + 2 + tid) : 0.f;
  if (tid < nsplit) {
    sm[tid] = __ldcg(base + tid * kPart + 0);
    sl[tid] = __ldcg(base + tid * kPart + 1);
  }
  __syncthreads();
  float M = -INFINITY;
  for (int j = 0; j < nsplit; ++j)
    if (sl[j] > 0.f) M = fmaxf(M, sm[j]);
  if (tid < nsplit) se[tid] = sl[tid] > 0.f ? expf(sm[tid] - M) : 0.f;
  __syncthreads();
  if (tid == 0) {
    float L = 0.f;
    for (int j = 0; j < nsplit; ++j) L = fmaf(sl[j], se[j], L);
    sL = L;
  }
  float o = 0.f;
#pragma unroll
  for (int j = 0; j < 64; ++j)
    if (j < nsplit) o = fmaf(ov[j], se[j], o);
  __syncthreads();
  out[static_cast<size_t>(blockIdx.x) * kD + tid] = sL > 0.f ? o / sL : 0.f;
}

}  // namespace qsa
