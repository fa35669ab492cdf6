// qsa_cache_write.cuh -- quantize and append cells to the int8 K/V cache.
//
// The write side of the prompt prep ("Round 5 Track C Report ...", section 1,
// Target 1-2: kcur/vcur rows of 2 x 256 floats per token) into "int8 KV, fp16
// scales" ("opus r20 track A ...", section 3).  Per group of 32 values (one warp):
//   s = fp16_rn(max|x| / 127) saturated at 65504; code = clamp(rint(x / s), -127, 127),
//   all codes 0 when s == 0.  Division and rounding are IEEE fp32 (round to nearest,
//   ties to even), so the codes are exact integers of a fixed rule.
#pragma once

#include "qsa_common.cuh"

namespace qsa {

// One group of 32 values, one per lane of a warp: returns this lane's code and, in
// `scale`, the group's fp16 scale.
__device__ __forceinline__ int8_t quantize_lane(float x, __half& scale) {
  float amax = fabsf(x);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  __half s = __float2half_rn(__fdiv_rn(amax, 127.0f));
  float sf = __half2float(s);
  if (!(sf <= 65504.0f)) {
    s = __ushort_as_half(0x7bff);
    sf = 65504.0f;
  }
  int code = 0;
  if (sf != 0.0f) code = max(-127, min(127, __float2int_rn(__fdiv_rn(x, sf))));
  scale = s;
  return static_cast<int8_t>(code);
}

// Quantize the 256 values of one (cell, KV head) row of K or V with `nthreads`
// threads (a multiple of 32, at most 256) and store codes and scales.
__device__ __forceinline__ void quantize_row(const float* __restrict__ src, int8_t* __restrict__ codes,
                                             __half* __restrict__ scales, int nthreads) {
  const int lane = threadIdx.x & 31;
  for (int d = static_cast<int>(threadIdx.x); d < kD; d += nthreads) {
    __half s;
    codes[d] = quantize_lane(__ldg(src + d), s);
    if (lane == 0) scales[d / kGroup] = s;
  }
}

// grid: (n, 2 KV heads, 2 = {K, V}); block: 256 threads = 8 groups of 32.
__global__ void __launch_bounds__(256) cache_write_kernel(int8_t* __restrict__ kc, int8_t* __restrict__ vc,
                                                          __half* __restrict__ ks, __half* __restrict__ vs,
                                                          __half* __restrict__ idx_key, int pos0,
                                                          const float* __restrict__ k,
                                                          const float* __restrict__ v,
                                                          const __half* __restrict__ key) {
  const int i = blockIdx.x, g = blockIdx.y, which = blockIdx.z;
  const int tid = threadIdx.x;
  const size_t cell = static_cast<size_t>(pos0) + i;
  // No early launch of dependents: a dependent may read cache keys before its own
  // grid-dependency wait (the decode score kernel does), so it starts only once every
  // cell here is written.
  griddep_wait();  // earlier kernels on the stream may still read the cells rewritten here
  const size_t row = cell * kHKV + g;
  quantize_row((which ? v : k) + (static_cast<size_t>(i) * kHKV + g) * kD, (which ? vc : kc) + row * kD,
               (which ? vs : ks) + row * kNG, 256);
  if (g == 0 && which == 0 && tid < kDI) idx_key[cell * kDI + tid] = key[static_cast<size_t>(i) * kDI + tid];
}

}  // namespace qsa
