// qsa_score_gemm.cuh -- prefill indexer scores as a tcgen05 / TMEM GEMM fed by TMA.
//
// The prompt path's qsa_score_mm ("opus r15 track A: prompt_chunk wave zipping, ...",
// what changed, item 1): for T query tokens and L cells,
//   score[t][c] = sum_h w[t][h] * max(0, sum_d iq[t][h][d] * key[c][d])   (4 heads x 64, fp16)
// is four [T x 64] x [64 x L] products followed by a ReLU-weighted sum over heads.
//
// sm_100a design (one persistent CTA per SM, 19 warps):
//   * a tile is 128 tokens x 64 cells.  For each head h one tcgen05.mma chain
//     (M = 128, N = 64, four K = 16 steps) writes D_h = iq_h . key^T into its own
//     64 TMEM columns, so token t's four head products sit in TMEM lane t at the
//     same column: the epilogue combines them without any data exchange;
//   * the 128 tokens' queries (4 heads x 128 x 64 fp16 = 64 KB) stay in shared
//     memory while a CTA sweeps its cells; key tiles (64 x 64 fp16 = 8 KB) stream
//     in through a 4-stage TMA ring, both with the 128-byte swizzle the UMMA
//     K-major descriptors describe;
//   * warp 0 issues TMA loads, warp 1 owns TMEM and issues the MMAs (one
//     thread), warps 2..17 are the epilogue (four per TMEM lane quadrant, 16
//     columns each), warp 18 issues TMA stores.  The epilogue writes each score
//     tile into a double-buffered shared stage in the 128-byte-swizzled layout,
//     and the stores move whole 128-byte row segments to global memory;  TMEM holds two 256-column accumulators, so
//     the epilogue of tile i overlaps the MMAs of tile i + 1;
//   * every wait on an mbarrier is bounded (four seconds of %globaltimer): on
//     expiry the CTA records QSA_ERR_TIMEOUT in `status`, every role stops,
//     in-flight copies and MMAs are drained (again with a bound) and TMEM is freed.
#pragma once

#include "qsa_sm100.cuh"

namespace qsa {

constexpr int kGemmTokens = 128;     // M
constexpr int kGemmCells = 64;       // N per head
constexpr int kGemmStages = 4;       // key-tile ring
constexpr int kGemmEpiWarps = 16;
constexpr int kGemmStoreWarp = 2 + kGemmEpiWarps;           // issues the TMA stores
constexpr int kGemmThreads = (3 + kGemmEpiWarps) * 32;
constexpr int kGemmABytes = kHI * kGemmTokens * kDI * 2;   // 64 KB
constexpr int kGemmBBytes = kGemmCells * kDI * 2;           // 8 KB
constexpr int kGemmCHalfBytes = kGemmTokens * 32 * 4;       // 16 KB: 128 rows x 32 fp32 scores
constexpr int kGemmSmemBytes = kGemmABytes + kGemmStages * kGemmBBytes + 4 * kGemmCHalfBytes +
                               1024 /*barriers*/ + 1024 /*align*/;
// More shared memory than two CTAs could share, so one CTA owns an SM and its
// TMEM (the CTA allocates all 512 columns).
constexpr int kGemmSmemRequest = kGemmSmemBytes;
static_assert(kGemmSmemRequest > 114 * 1024, "one GEMM CTA per SM");

struct GemmArgs {
  const float* iw;     // [T][4]
  float* scores;       // [T][ld]
  int64_t ld;
  int T;
  int ncells;
  uint32_t* status;    // 0, or QSA_ERR_TIMEOUT after a wait expired
};

struct __align__(8) GemmBarriers {
  uint64_t b_full[kGemmStages];
  uint64_t b_empty[kGemmStages];
  uint64_t a_full;
  uint64_t a_empty;
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t stage_full[2];   // epilogue warps wrote a score tile into the staging buffer
  uint64_t stage_free[2];   // the TMA store finished reading that buffer
  uint64_t drain;
  uint32_t tmem_base;
  uint32_t abort;
};

// Instruction descriptor: fp32 accumulate, fp16 A and B, both K-major, M = 128, N = 64.
constexpr uint32_t kGemmIdesc = umma_idesc_f16(kGemmTokens, kGemmCells, false, false);

// A K-major operand here is a stack of 8-row atoms of 1024 bytes.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr) { return umma_desc_k_sw128(saddr, 1024); }

// grid: number of SMs (persistent); block: kGemmThreads; dynamic smem: kGemmSmemRequest.
__global__ void __launch_bounds__(kGemmThreads, 1)
    score_gemm_kernel(const __grid_constant__ CUtensorMap tmap_key,
                      const __grid_constant__ CUtensorMap tmap_iq,
                      const __grid_constant__ CUtensorMap tmap_out, GemmArgs a) {
  extern __shared__ __align__(1024) unsigned char gsm_raw[];
  unsigned char* gsm = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(gsm_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* sA = gsm;                                   // 4 heads x 16 KB
  unsigned char* sB = gsm + kGemmABytes;                     // stages x 8 KB
  unsigned char* sC = sB + kGemmStages * kGemmBBytes;        // 2 buffers x 2 halves x 16 KB
  GemmBarriers& gb = *reinterpret_cast<GemmBarriers*>(sC + 4 * kGemmCHalfBytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntb = (a.T + kGemmTokens - 1) / kGemmTokens;
  const int nct = (a.ncells + kGemmCells - 1) / kGemmCells;
  const int items = ntb * nct;
  const int per = (items + gridDim.x - 1) / gridDim.x;
  const int it0 = min(items, static_cast<int>(blockIdx.x) * per);
  const int it1 = min(items, it0 + per);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGemmStages; ++s) {
      mbar_init(&gb.b_full[s], 1);
      mbar_init(&gb.b_empty[s], 1);
    }
    mbar_init(&gb.a_full, 1);
    mbar_init(&gb.a_empty, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&gb.acc_full[b], 1);
      mbar_init(&gb.acc_empty[b], kGemmEpiWarps);
      mbar_init(&gb.stage_full[b], kGemmEpiWarps);
      mbar_init(&gb.stage_free[b], 1);
    }
    mbar_init(&gb.drain, 1);
    gb.abort = 0u;
    mbar_init_fence();
  }
  if (warp == 1) tmem_alloc(&gb.tmem_base, 512u);  // two accumulators of 4 heads x 64 columns
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = gb.tmem_base;
  griddep_launch();
  griddep_wait();  // keys and queries may come from kernels before this one

  if (warp == 0) {
    // ---------------- TMA producer
    if (lane == 0) {
      int cur_tb = -1, a_loads = 0, issued = 0;
      bool ok = true;
      for (int it = it0; it < it1 && ok; ++it) {
        const int tb = it / nct, ct = it % nct;
        if (tb != cur_tb) {
          if (a_loads > 0) ok = mbar_wait(&gb.a_empty, (a_loads - 1) & 1, &gb.abort, a.status);
          if (!ok) break;
          mbar_expect_tx(&gb.a_full, kGemmABytes);
          for (int h = 0; h < kHI; ++h)
            tma_load_3d(sA + h * (kGemmTokens * kDI * 2), &tmap_iq, 0, h, tb * kGemmTokens, &gb.a_full);
          cur_tb = tb;
          ++a_loads;
        }
        const int li = it - it0, s = li % kGemmStages, round = li / kGemmStages;
        ok = mbar_wait(&gb.b_empty[s], (round & 1) ^ 1, &gb.abort, a.status);
        if (!ok) break;
        mbar_expect_tx(&gb.b_full[s], kGemmBBytes);
        tma_load_2d(sB + s * kGemmBBytes, &tmap_key, 0, ct * kGemmCells, &gb.b_full[s]);
        issued = li + 1;
      }
      if (!ok) {  // drain copies still in flight before the CTA leaves
        for (int li = max(0, issued - kGemmStages); li < issued; ++li)
          mbar_drain_wait(&gb.b_full[li % kGemmStages], (li / kGemmStages) & 1);
        if (a_loads > 0) mbar_drain_wait(&gb.a_full, (a_loads - 1) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      int cur_tb = -1, a_loads = 0;
      bool ok = true;
      for (int it = it0; it < it1 && ok; ++it) {
        const int tb = it / nct;
        const int li = it - it0, s = li % kGemmStages, round = li / kGemmStages;
        const int buf = li & 1, bround = li >> 1;
        if (tb != cur_tb) {
          ok = mbar_wait(&gb.a_full, a_loads & 1, &gb.abort, a.status);
          if (!ok) break;
          cur_tb = tb;
          ++a_loads;
        }
        ok = mbar_wait(&gb.b_full[s], round & 1, &gb.abort, a.status) &&
             mbar_wait(&gb.acc_empty[buf], (bround & 1) ^ 1, &gb.abort, a.status);
        if (!ok) break;
        tc_fence_after();
        const uint32_t b0 = smem_u32(sB + s * kGemmBBytes);
#pragma unroll
        for (int h = 0; h < kHI; ++h) {
          const uint32_t a0 = smem_u32(sA + h * (kGemmTokens * kDI * 2));
          const uint32_t d = tmem + static_cast<uint32_t>(buf * 256 + h * kGemmCells);
#pragma unroll
          for (int ks = 0; ks < kDI / 16; ++ks)
            umma_f16(d, umma_desc_sw128(a0 + ks * 32), umma_desc_sw128(b0 + ks * 32), kGemmIdesc, ks > 0 ? 1u : 0u);
        }
        umma_commit(&gb.b_empty[s]);       // the key stage is free once these MMAs finish
        umma_commit(&gb.acc_full[buf]);    // the accumulator is ready for the epilogue
        const bool last_of_tb = (it + 1 == it1) || ((it + 1) / nct != tb);
        if (last_of_tb) umma_commit(&gb.a_empty);
      }
      // every MMA this thread issued has completed once `drain` fires
      umma_commit(&gb.drain);
      mbar_drain_wait(&gb.drain, 0);
    }
    __syncwarp();
  } else if (warp == kGemmStoreWarp) {
    // ---------------- TMA stores of the staged score tiles (two 32-column boxes each)
    if (lane == 0) {
      for (int it = it0; it < it1; ++it) {
        const int tb = it / nct, ct = it % nct;
        const int li = it - it0, sb = li & 1;
        if (!mbar_wait(&gb.stage_full[sb], (li >> 1) & 1, &gb.abort, a.status)) break;
        for (int h = 0; h < 2; ++h)  // a box past the last column has nothing to write
          if (ct * kGemmCells + 32 * h < a.ncells)
            tma_store_2d(&tmap_out, ct * kGemmCells + 32 * h, tb * kGemmTokens,
                         sC + (sb * 2 + h) * kGemmCHalfBytes);
        bulk_commit();
        // the previous tile's buffer is free once its store has read it
        bulk_wait_read<1>();
        if (li > 0) mbar_arrive(&gb.stage_free[sb ^ 1]);
      }
      bulk_wait_all();  // every store of this CTA has landed in global memory
    }
    __syncwarp();
  } else {
    // ---------------- epilogue: 16 warps; warp w reads TMEM lanes 32 * (w % 4) ...
    const int quad = warp & 3;
    const int colq = (warp - 2) >> 2;  // columns [16 * colq, 16 * colq + 16) of each head
    const int r = quad * 32 + lane;    // tile row of this thread
    int cur_tb = -1;
    float w[kHI] = {0.f, 0.f, 0.f, 0.f};
    for (int it = it0; it < it1; ++it) {
      const int tb = it / nct;
      const int li = it - it0, buf = li & 1, bround = li >> 1;
      const int row = tb * kGemmTokens + r;
      if (tb != cur_tb) {
#pragma unroll
        for (int h = 0; h < kHI; ++h) w[h] = row < a.T ? __ldg(a.iw + row * kHI + h) : 0.f;
        cur_tb = tb;
      }
      // one lane waits, the warp follows it (the TMEM loads below are warp-collective)
      if (!mbar_wait_warp(&gb.acc_full[buf], bround & 1, &gb.abort, a.status)) break;
      tc_fence_after();
      const int col = colq * 16;
      uint32_t rr[kHI][16];
#pragma unroll
      for (int h = 0; h < kHI; ++h)
        tmem_ld16(tmem + (static_cast<uint32_t>(quad * 32) << 16) +
                      static_cast<uint32_t>(buf * 256 + h * kGemmCells + col),
                  rr[h]);
      tmem_ld_wait();
      // the accumulator is in registers: hand it back to the MMA warp now
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&gb.acc_empty[buf]);
      float sc[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        float sacc = w[0] * fmaxf(__uint_as_float(rr[0][j]), 0.f);
        sacc = fmaf(w[1], fmaxf(__uint_as_float(rr[1][j]), 0.f), sacc);
        sacc = fmaf(w[2], fmaxf(__uint_as_float(rr[2][j]), 0.f), sacc);
        sc[j] = fmaf(w[3], fmaxf(__uint_as_float(rr[3][j]), 0.f), sacc);
      }
      // stage the scores: buffer li & 1, half colq / 2, 128-byte rows with 16-byte
      // chunk c stored at c ^ (row % 8) (the layout the TMA store's 128-byte swizzle reads)
      const int sb = li & 1;
      if (!mbar_wait_warp(&gb.stage_free[sb], ((li >> 1) & 1) ^ 1, &gb.abort, a.status)) break;
      unsigned char* half = sC + (sb * 2 + (colq >> 1)) * kGemmCHalfBytes + r * 128;
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const int chunk = ((colq & 1) * 4 + jj) ^ (r & 7);
        *reinterpret_cast<float4*>(half + chunk * 16) =
            make_float4(sc[4 * jj], sc[4 * jj + 1], sc[4 * jj + 2], sc[4 * jj + 3]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&gb.stage_full[sb]);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512u);
}

// Self-test of the bounded wait: one thread waits on a barrier that nothing
// completes and must give up after the limit, recording the timeout.
__global__ void wait_selftest_kernel(uint32_t* status) {
  __shared__ GemmBarriers gb;
  if (threadIdx.x == 0) {
    mbar_init(&gb.drain, 1);
    gb.abort = 0u;
    mbar_init_fence();
    mbar_wait(&gb.drain, 0, &gb.abort, status, kSelftestLimitNs);
  }
}

}  // namespace qsa
