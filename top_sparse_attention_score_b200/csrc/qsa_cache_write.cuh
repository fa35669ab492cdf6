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

// grid: (n, 2 KV heads, 2 = {K, V}); block: 256 threads = 8 groups of 32.
__global__ void __launch_bounds__(256) cache_write_kernel(int8_t* __restrict__ kc, int8_t* __restrict__ vc,
                                                          __half* __restrict__ ks, __half* __restrict__ vs,
                                                          __half* __restrict__ idx_key, int pos0,
                                                          const float* __restrict__ k,
                                                          const float* __restrict__ v,
                                                          const __half* __restrict__ key) {
  const int i = blockIdx.x, g = blockIdx.y, which = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, grp = tid >> 5;
  const size_t cell = static_cast<size_t>(pos0) + i;
  griddep_launch();
  griddep_wait();  // earlier kernels on the stream may still read the cells rewritten here
  const float x = __ldg((which ? v : k) + (static_cast<size_t>(i) * kHKV + g) * kD + tid);
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
  (which ? vc : kc)[(cell * kHKV + g) * kD + tid] = static_cast<int8_t>(code);
  if (lane == 0) (which ? vs : ks)[(cell * kHKV + g) * kNG + grp] = s;
  if (g == 0 && which == 0 && tid < kDI) idx_key[cell * kDI + tid] = key[static_cast<size_t>(i) * kDI + tid];
}

}  // namespace qsa
