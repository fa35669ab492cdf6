// qsa_common.cuh -- shapes and small device helpers shared by the QSA kernels.
#pragma once

#include <cuda_fp16.h>
#include <cstdint>

namespace qsa {

constexpr int kHQ = 24;        // query heads
constexpr int kD = 256;        // head dim
constexpr int kHKV = 2;        // KV heads
constexpr int kQPerKV = 12;    // query heads per KV head
constexpr int kGroup = 32;     // int8 values per fp16 scale
constexpr int kNG = 8;         // scale groups per head row
constexpr int kHI = 4;         // indexer heads
constexpr int kDI = 64;        // indexer dim
constexpr int kPart = 2 + kD;  // floats per split partial {m, l, o[256]}
constexpr int kBins = 2048;    // coarse histogram bins of the selection

// D = A(16x16, row) * B(16x8, col) + D with fp16 inputs and fp32 accumulators.
// Fragment layout (g = lane / 4, t = lane % 4):
//   a0 = A[g][2t..2t+1], a1 = A[g+8][2t..2t+1], a2 = A[g][2t+8..2t+9], a3 = A[g+8][2t+8..2t+9]
//   b0 = B[2t..2t+1][g], b1 = B[2t+8..2t+9][g]
//   c0 = C[g][2t], c1 = C[g][2t+1], c2 = C[g+8][2t], c3 = C[g+8][2t+1]
__device__ __forceinline__ void mma_f16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                              uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Two int8 codes -> exact fp16 pair.  `x` holds bytes already XORed with 0x80
// (so byte = code + 128); `sel` picks the two bytes (byte_perm selector with
// 0x4 in the odd nibbles).  0x64yy is the fp16 1024 + yy, so subtracting
// 1152 = 1024 + 128 leaves the code exactly.
__device__ __forceinline__ uint32_t i8x2_to_h2(uint32_t x, uint32_t sel) {
  const uint32_t h = __byte_perm(x, 0x64646464u, sel);
  const __half2 r = __hsub2(*reinterpret_cast<const __half2*>(&h), __half2half2(__ushort_as_half(0x6480)));
  return *reinterpret_cast<const uint32_t*>(&r);
}

// The same two bytes as fp16 1152 + code (exact; the caller removes the 1152).
__device__ __forceinline__ uint32_t i8x2_to_h2_biased(uint32_t x, uint32_t sel) {
  return __byte_perm(x, 0x64646464u, sel);
}

// The output gate ("attention + gate"): the attention output is multiplied
// elementwise by sigmoid(g) = 1 / (1 + exp(-g)).
__device__ __forceinline__ float gate_factor(float g) { return 1.f / (1.f + expf(-g)); }

// Order-preserving 32-bit key of an fp32 score: larger value -> larger key,
// -0 mapped to +0 so the two compare equal.
__device__ __forceinline__ uint32_t score_key(float f) {
  uint32_t b = __float_as_uint(f);
  if ((b << 1) == 0u) b = 0u;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// 16-bit order-preserving key of a score's fp16 rounding (-0 mapped to +0).
// fp32 -> fp16 round-to-nearest never reverses an order, so a bin made of this
// key's top bits always holds strictly larger scores than every lower bin.
__device__ __forceinline__ uint32_t score_key16(float f) {
  uint32_t b = __half_as_ushort(__float2half_rn(f));
  if ((b & 0x7fffu) == 0u) b = 0u;
  return (b & 0x8000u) ? (~b & 0xffffu) : (b | 0x8000u);
}

// Coarse bin of a score: the top 11 bits of score_key16 (2048 bins).
__device__ __forceinline__ uint32_t score_bin(float f) { return score_key16(f) >> 5; }

// Exclusive prefix sum over the block (NT threads, NT % 32 == 0, NT <= 1024).
// `scratch` is 33 words of shared memory; `total` receives the block sum.
template <int NT>
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t* scratch,
                                                         uint32_t& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) scratch[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = lane < NT / 32 ? scratch[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    scratch[lane] = w;
  }
  __syncthreads();
  const uint32_t base = warp ? scratch[warp - 1] : 0u;
  total = scratch[NT / 32 - 1];
  __syncthreads();
  return base + x - v;
}

// Over `nbins` bins held in shared or global memory, bins taken from the
// highest down: find the bin `thr` where the running count first reaches
// `k`, and the count strictly above it.  Every thread returns the answer.
// Requires nbins % NT == 0 or NT % nbins == 0.  If the total is below k,
// thr = 0 and `above` is the total minus bin 0.
template <int NT>
__device__ __forceinline__ void find_threshold_bin(const uint32_t* hist, int nbins, uint32_t k,
                                                   uint32_t* scratch, uint32_t* result,
                                                   uint32_t& thr, uint32_t& above) {
  const int per = nbins >= NT ? nbins / NT : 1;
  const bool owner = static_cast<int>(threadIdx.x) * per < nbins;
  const int hi = nbins - 1 - static_cast<int>(threadIdx.x) * per;  // bins hi, hi-1, ..., hi-per+1
  uint32_t local = 0;
  if (owner)
    for (int i = 0; i < per; ++i) local += hist[hi - i];
  uint32_t total;
  const uint32_t before = block_exclusive_scan<NT>(local, scratch, total);
  if (threadIdx.x == 0) {
    result[0] = 0u;
    result[1] = total - hist[0];
  }
  __syncthreads();
  if (owner && before < k && before + local >= k) {
    uint32_t run = before;
    for (int i = 0; i < per; ++i) {
      const uint32_t h = hist[hi - i];
      if (run + h >= k) {
        result[0] = static_cast<uint32_t>(hi - i);
        result[1] = run;
        break;
      }
      run += h;
    }
  }
  __syncthreads();
  thr = result[0];
  above = result[1];
  __syncthreads();
}

// Programmatic dependent launch: a kernel launched with programmatic stream
// serialisation may start while its predecessor drains.  It must call
// griddep_wait() before touching memory the predecessor reads or writes, and
// every CTA must call it before exiting (the ordering is transitive only if
// no kernel completes ahead of its predecessor); griddep_launch() lets its own
// dependent start launching early.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void griddep_launch() { asm volatile("griddepcontrol.launch_dependents;\n" ::); }

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, bool valid) {
  const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  const int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem), "r"(n));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

}  // namespace qsa
