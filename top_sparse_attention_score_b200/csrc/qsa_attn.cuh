// qsa_attn.cuh -- sparse attention over the selected cells of an int8 K/V cache.
//
// qsa_attn of "opus r20 track A: MTP map mlock + qsa_attn / qsa_merge decode tweaks",
// section 2 (max-subtracted softmax over the selected cells, then a weighted sum of V),
// on "random int8 KV, fp16 scales" (section 3), written for sm_100a:
//
//  * one CTA per (row, KV head, split); the 12 query heads of the KV head are the
//    16 rows of mma.sync m16n8k16 tiles (rows 12..15 zero), so QK^T and PV run on
//    tensor cores instead of 6144 fp32 FMAs per gathered cell;
//  * cells are gathered 32 at a time with cp.async (16-byte copies of whole
//    256-byte K/V rows and their scales) into a double-buffered shared-memory
//    ring, so the next block's gathers are in flight while one computes; each
//    block's ids are loaded a block before its gathers are issued;
//  * W warps split the 256 dims (W = 2 for prompt chunks, 4 for decode): each
//    computes a partial QK^T over its dims, the partials are summed through shared
//    memory in a fixed order (every warp gets bit-equal scores), each warp runs the
//    same online softmax and accumulates P.V for its own dims;
//  * int8 codes become fp16 exactly by byte-permute with the 0x6400 exponent, which
//    gives 1152 + code.  For K the 1152 stays in: each 32-dim group's accumulator
//    starts at -1152 times the group's sum of fp16 q, and the per-32 K scale
//    multiplies the group's partial product in fp32 after the MMA.  For V the 1152
//    is subtracted (the two cells of a B register interleaved by one byte-permute
//    per four pairs) and the per-32 V scale multiplies the fp16 V operand.  Q and P
//    are fp16, the weights 2^x from the hardware ex2;
//  * the reference maximum of the online softmax moves only when a block
//    exceeds it by more than 2^8, so P stays <= 256 and most blocks skip the
//    rescale of O; split partials are reported against the true maximum;
//  * a second instantiation (kAll) serves rows that see at most top_k cells:
//    the selection would keep all of them, so list position p is cell p and
//    no ids are read (the whole-step calls then launch no score or selection).
#pragma once

#include "qsa_common.cuh"

namespace qsa {

constexpr int kAttnCells = 32;    // cells per pipeline block
constexpr int kAttnKStride = 288; // bytes per K row in shared memory (72 words: conflict-free 8-byte reads)
constexpr int kAttnVStride = 272; // bytes per V row in shared memory (68 words: conflict-free 4-byte reads)

struct __align__(16) AttnStage {
  int8_t k[kAttnCells * kAttnKStride];
  int8_t v[kAttnCells * kAttnVStride];
  __half ks[kAttnCells * kNG];
  __half vs[kAttnCells * kNG];
  int valid[kAttnCells];
};

constexpr int kAttnStages = 2;

// 2^x by the hardware approximation (ex2.approx.ftz: subnormal results flush to zero; the
// weights it feeds are rounded to fp16 and never exceed 2^8, so nothing below 2^-126 matters).
__device__ __forceinline__ float attn_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
constexpr float kAttnShift = 8.f;      // log2 margin before the reference maximum moves
constexpr float kAttnNoMax = -1.0e30f;  // reference maximum before the first valid cell

// W warps split the 256 dims (W = 4 for the latency of decode, 2 for the
// throughput of prefill: half the duplicated softmax and score-reduction work).
template <int W>
struct AttnSmem {
  AttnStage st[kAttnStages];
  float4 red[W][4][32];  // [warp][n-tile][lane] partial scores
};

struct AttnArgs {
  const int8_t* k;
  const int8_t* v;
  const __half* ks;
  const __half* vs;
  const float* q;     // [rows][24][256]
  const int* ids;     // [rows][top_k]; NULL: row r's list is cells 0 .. dense_vis0 + r - 1, -1 padded
  int top_k;
  int max_cells;      // ids outside [0, max_cells) are treated as empty slots
  int nsplit;
  int piece;          // ceil(top_k / nsplit)
  float scale_log2;   // softmax scale * log2(e)
  float* part;        // [rows][24][nsplit][258] when nsplit > 1
  float* out;         // [rows][24][256] when nsplit == 1
  const float* gate;  // [rows][24][256] or NULL: out *= sigmoid(gate) when nsplit == 1
  int dense_vis0;     // ids == NULL: cells row 0 sees (row r sees dense_vis0 + r <= top_k)
  int* ids_fill;      // ids == NULL: optional [rows][top_k] copy of the implicit lists
};

// Cell of list position p < end: ids[p], or with the implicit list (kAll) p itself below dv.
template <bool kAll>
__device__ __forceinline__ int attn_cell(const int* rid, int dv, int p, int end) {
  if (p >= end) return -1;
  if constexpr (kAll) return p < dv ? p : -1;
  else return __ldg(rid + p);
}

// ---- the pieces of attn_kernel

// Online-softmax state of one W-warp group for one (row, KV head): the reference
// maximum (log2 units) of P, finite from the start so a block with no valid cell gives
// exp2(-inf - m_run) = 0 without a guard; the true maximum; the weight sum; and this
// warp's O accumulators (rows g and g + 8 of the 16-row tiles).
template <int W>
struct AttnState {
  static constexpr int GW = kNG / W;  // scale groups (32 dims each) per warp
  float m_run[2], m_top[2], l_run[2];
  float o[GW][4][4];
  __device__ __forceinline__ void init() {
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      m_run[r] = kAttnNoMax;
      m_top[r] = -INFINITY;
      l_run[r] = 0.f;
    }
#pragma unroll
    for (int gi = 0; gi < GW; ++gi)
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int c = 0; c < 4; ++c) o[gi][i][c] = 0.f;
  }
};

// Q fragments for warp `warp` of a W-warp group, its kNG / W scale groups of dims, prescaled
// by sl = scale * log2(e).  q0 points at the KV head's first query head of the row.
// Within group qg, thread t covers dims 32qg + 8t + 4s + {0..3} in sub-step s:
// k-index 2t,2t+1 <-> +0,+1 and 2t+8,2t+9 <-> +2,+3 (the same map as the K loads).
template <int W>
__device__ __forceinline__ void attn_load_q(uint32_t (&aq)[kNG / W][2][4], const float* q0, float sl, int warp) {
  constexpr int GW = kNG / W;
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const float* qg0 = q0 + g * kD;
  const float* q8 = qg0 + 8 * kD;
  const bool has8 = g + 8 < kQPerKV;
#pragma unroll
  for (int gi = 0; gi < GW; ++gi)
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      const int d0 = 32 * (GW * warp + gi) + 8 * t + 4 * s;
      const float4 x = __ldg(reinterpret_cast<const float4*>(qg0 + d0));
      aq[gi][s][0] = pack_half2(x.x * sl, x.y * sl);
      aq[gi][s][2] = pack_half2(x.z * sl, x.w * sl);
      if (has8) {
        const float4 y = __ldg(reinterpret_cast<const float4*>(q8 + d0));
        aq[gi][s][1] = pack_half2(y.x * sl, y.y * sl);
        aq[gi][s][3] = pack_half2(y.z * sl, y.w * sl);
      } else {
        aq[gi][s][1] = 0u;
        aq[gi][s][3] = 0u;
      }
    }
}

// The cells one thread gathers of a 32-cell block: chunk u (K and V rows) is cell
// (tid + NT u) / 16, the scales' cell is tid % 32 (for tid < 64).
template <int NT>
struct AttnIds {
  static constexpr int kChunks = 512 / NT;
  int chunk[kChunks];
  int scale;
};

// The ids of one block (cell_of(i): list slot i), loaded a block before its gather.
template <int NT, class CellOf>
__device__ __forceinline__ void attn_load_ids(AttnIds<NT>& ids, int tid, CellOf cell_of) {
#pragma unroll
  for (int u = 0; u < AttnIds<NT>::kChunks; ++u) ids.chunk[u] = cell_of((tid + NT * u) >> 4);
  ids.scale = tid < 2 * kAttnCells ? cell_of(tid & 31) : -1;
}

// The K codes enter the QK^T tiles as fp16 1152 + code (one byte-permute, no subtraction):
// each group's accumulator starts at -1152 times the group's sum of fp16 q instead, for rows g
// (kb[gi][0]) and g + 8 (kb[gi][1]).  The sums are of the fp16 fragments the MMAs read, over
// the quad's 32 dims of the group.
template <int W>
__device__ __forceinline__ void attn_k_bias(float (&kb)[kNG / W][2], const uint32_t (&aq)[kNG / W][2][4]) {
#pragma unroll
  for (int gi = 0; gi < kNG / W; ++gi)
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      float sum = 0.f;
#pragma unroll
      for (int s = 0; s < 2; ++s)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&aq[gi][s][r + 2 * h]));
          sum += f.x + f.y;
        }
      sum += __shfl_xor_sync(0xffffffffu, sum, 1);
      sum += __shfl_xor_sync(0xffffffffu, sum, 2);
      kb[gi][r] = -1152.f * sum;
    }
}

// Gather one block of 32 cells into `st` with NT threads (tid = 0 .. NT - 1): slot i holds
// the cell of ids, an empty slot for one < 0 or >= max_cells.
template <int NT>
__device__ __forceinline__ void attn_gather(AttnStage& st, const AttnArgs& a, int kvh, int tid,
                                            const AttnIds<NT>& ids) {
  // K and V rows: 32 cells x 16 chunks of 16 bytes each, 512 / NT + 512 / NT per thread.
#pragma unroll
  for (int u = 0; u < AttnIds<NT>::kChunks; ++u) {
    const int chunk = tid + NT * u;
    const int i = chunk >> 4, part = chunk & 15;
    int cell = ids.chunk[u];
    const bool ok = cell >= 0 && cell < a.max_cells;
    if (!ok) cell = 0;
    const size_t row = (static_cast<size_t>(cell) * kHKV + kvh) * kD + part * 16;
    cp_async16(st.k + i * kAttnKStride + part * 16, a.k + row, ok);
    cp_async16(st.v + i * kAttnVStride + part * 16, a.v + row, ok);
  }
  if (tid < 2 * kAttnCells) {  // scales: 64 rows of 16 bytes
    const int i = tid & 31;
    int cell = ids.scale;
    const bool ok = cell >= 0 && cell < a.max_cells;
    if (tid < kAttnCells) st.valid[i] = ok;
    if (!ok) cell = 0;
    const size_t srow = (static_cast<size_t>(cell) * kHKV + kvh) * kNG;
    if (tid < kAttnCells) cp_async16(st.ks + i * kNG, a.ks + srow, ok);
    else cp_async16(st.vs + i * kNG, a.vs + srow, ok);
  }
}

// N consecutive fp16 scales (N = 2 or 4, 4N-byte aligned) as floats, in one shared load.
template <int N>
__device__ __forceinline__ void attn_load_scales(const __half* p, float (&f)[N]) {
  if constexpr (N == 4) {
    const uint2 w = *reinterpret_cast<const uint2*>(p);
    const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&w.x));
    const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&w.y));
    f[0] = a.x;
    f[1] = a.y;
    f[2] = b.x;
    f[3] = b.y;
  } else {
    static_assert(N == 2, "two or four scales");
    const float2 a = __half22float2(*reinterpret_cast<const __half2*>(p));
    f[0] = a.x;
    f[1] = a.y;
  }
}

// One gathered block through the online softmax, for warp `warp` of a W-warp group:
// partial QK^T over the warp's dims, the group's partial scores summed through `red`
// (every warp in the same order, so all agree bit for bit), masking, the running
// maximum, the weights and P.V into the warp's O.  `sync` is the group's barrier.
template <int W, class Sync>
__device__ __forceinline__ void attn_block(const AttnStage& st, float4 (*red)[4][32],
                                           const uint32_t (&aq)[kNG / W][2][4], const float (&kb)[kNG / W][2],
                                           AttnState<W>& S, int warp, Sync sync) {
  constexpr int GW = kNG / W;
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const uint32_t valid = __ballot_sync(0xffffffffu, st.valid[lane] != 0);  // bit c: slot c holds a cell

  // ---- partial scores over this warp's dims
  float s[4][4];
#pragma unroll
  for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
    for (int c = 0; c < 4; ++c) s[nt][c] = 0.f;
    const int8_t* krow = st.k + (8 * nt + g) * kAttnKStride;
    // the K scales of this warp's groups for cells 8 nt + 2t and 8 nt + 2t + 1, one load each
    float ksa[GW], ksb[GW];
    attn_load_scales<GW>(st.ks + (8 * nt + 2 * t) * kNG + GW * warp, ksa);
    attn_load_scales<GW>(st.ks + (8 * nt + 2 * t + 1) * kNG + GW * warp, ksb);
#pragma unroll
    for (int gi = 0; gi < GW; ++gi) {
      const int qg = GW * warp + gi;
      const uint2 kw = *reinterpret_cast<const uint2*>(krow + 32 * qg + 8 * t);
      const uint32_t x0 = kw.x ^ 0x80808080u, x1 = kw.y ^ 0x80808080u;
      float acc[4] = {kb[gi][0], kb[gi][0], kb[gi][1], kb[gi][1]};
      mma_f16_16816(acc, aq[gi][0], i8x2_to_h2_biased(x0, 0x4140u), i8x2_to_h2_biased(x0, 0x4342u));
      mma_f16_16816(acc, aq[gi][1], i8x2_to_h2_biased(x1, 0x4140u), i8x2_to_h2_biased(x1, 0x4342u));
      const float2 sc = make_float2(ksa[gi], ksb[gi]);
      s[nt][0] = fmaf(sc.x, acc[0], s[nt][0]);
      s[nt][1] = fmaf(sc.y, acc[1], s[nt][1]);
      s[nt][2] = fmaf(sc.x, acc[2], s[nt][2]);
      s[nt][3] = fmaf(sc.y, acc[3], s[nt][3]);
    }
    red[warp][nt][lane] = make_float4(s[nt][0], s[nt][1], s[nt][2], s[nt][3]);
  }
  sync();
  // ---- full scores (same summation order in every warp), masked
  float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
  for (int nt = 0; nt < 4; ++nt) {
    float4 r;
    if constexpr (W == 2) {  // own partial + the other warp's (a + b == b + a: both warps agree)
      const float4 y = red[warp ^ 1][nt][lane];
      r = make_float4(s[nt][0] + y.x, s[nt][1] + y.y, s[nt][2] + y.z, s[nt][3] + y.w);
    } else {
      r = red[0][nt][lane];
#pragma unroll
      for (int w = 1; w < W; ++w) {
        const float4 y = red[w][nt][lane];
        r.x += y.x;
        r.y += y.y;
        r.z += y.z;
        r.w += y.w;
      }
    }
    const bool v0 = (valid >> (8 * nt + 2 * t)) & 1u, v1 = (valid >> (8 * nt + 2 * t + 1)) & 1u;
    s[nt][0] = v0 ? r.x : -INFINITY;
    s[nt][1] = v1 ? r.y : -INFINITY;
    s[nt][2] = v0 ? r.z : -INFINITY;
    s[nt][3] = v1 ? r.w : -INFINITY;
    mx[0] = fmaxf(mx[0], fmaxf(s[nt][0], s[nt][1]));
    mx[1] = fmaxf(mx[1], fmaxf(s[nt][2], s[nt][3]));
  }
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
    mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
  }
  // The reference maximum m_run moves only when a block exceeds it by more
  // than 2^8 (P <= 256 in fp16), so most blocks skip the rescale of O; the
  // true maximum m_top is kept for the split partials.
#pragma unroll
  for (int r = 0; r < 2; ++r) S.m_top[r] = fmaxf(S.m_top[r], mx[r]);
  if (__any_sync(0xffffffffu, mx[0] > S.m_run[0] + kAttnShift || mx[1] > S.m_run[1] + kAttnShift)) {
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const float mnew = fmaxf(S.m_run[r], mx[r]);
      const float alpha = attn_exp2(S.m_run[r] - mnew);
      S.l_run[r] *= alpha;
      S.m_run[r] = mnew;
#pragma unroll
      for (int gi = 0; gi < GW; ++gi)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          S.o[gi][i][2 * r] *= alpha;
          S.o[gi][i][2 * r + 1] *= alpha;
        }
    }
  }
  float rs[2] = {0.f, 0.f};
#pragma unroll
  for (int nt = 0; nt < 4; ++nt)
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int r = c >> 1;
      const float p = attn_exp2(s[nt][c] - S.m_run[r]);
      s[nt][c] = p;
      rs[r] += p;
    }
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    rs[r] += __shfl_xor_sync(0xffffffffu, rs[r], 1);
    rs[r] += __shfl_xor_sync(0xffffffffu, rs[r], 2);
    S.l_run[r] += rs[r];
  }

  // ---- P.V for this warp's dims; P's k-index j <-> cell 16*s2 + j
#pragma unroll
  for (int s2 = 0; s2 < 2; ++s2) {
    uint32_t pa[4];
    pa[0] = pack_half2(s[2 * s2][0], s[2 * s2][1]);
    pa[1] = pack_half2(s[2 * s2][2], s[2 * s2][3]);
    pa[2] = pack_half2(s[2 * s2 + 1][0], s[2 * s2 + 1][1]);
    pa[3] = pack_half2(s[2 * s2 + 1][2], s[2 * s2 + 1][3]);
    const int cA = 16 * s2 + 2 * t;  // cells of k-index 2t, 2t+1, 2t+8, 2t+9
    // their V scales for this warp's groups: one load per cell (two fp16 per word)
    uint32_t vsw[4][(GW + 1) / 2];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const __half* p = st.vs + (cA + (k & 1) + 8 * (k >> 1)) * kNG + GW * warp;
      if constexpr (GW == 4) {
        const uint2 w = *reinterpret_cast<const uint2*>(p);
        vsw[k][0] = w.x;
        vsw[k][1] = w.y;
      } else {
        vsw[k][0] = *reinterpret_cast<const uint32_t*>(p);
      }
    }
#pragma unroll
    for (int gi = 0; gi < GW; ++gi) {
      const int qg = GW * warp + gi;
      // column g of n-tile i is dim 32qg + 4g + i
      const int8_t* vb = st.v + 32 * qg + 4 * g;
      const uint32_t wA = *reinterpret_cast<const uint32_t*>(vb + cA * kAttnVStride) ^ 0x80808080u;
      const uint32_t wB = *reinterpret_cast<const uint32_t*>(vb + (cA + 1) * kAttnVStride) ^ 0x80808080u;
      const uint32_t wC = *reinterpret_cast<const uint32_t*>(vb + (cA + 8) * kAttnVStride) ^ 0x80808080u;
      const uint32_t wD = *reinterpret_cast<const uint32_t*>(vb + (cA + 9) * kAttnVStride) ^ 0x80808080u;
      const uint32_t hsel = (gi & 1) ? 0x7632u : 0x5410u;  // the group's fp16 of two cells' words
      const uint32_t uAB = __byte_perm(vsw[0][gi >> 1], vsw[1][gi >> 1], hsel);
      const uint32_t uCD = __byte_perm(vsw[2][gi >> 1], vsw[3][gi >> 1], hsel);
      const __half2 sAB = *reinterpret_cast<const __half2*>(&uAB);
      const __half2 sCD = *reinterpret_cast<const __half2*>(&uCD);
      // the two cells' bytes interleaved once: [A0 B0 A1 B1] and [A2 B2 A3 B3]
      const uint32_t ab[2] = {__byte_perm(wA, wB, 0x5140u), __byte_perm(wA, wB, 0x7362u)};
      const uint32_t cd[2] = {__byte_perm(wC, wD, 0x5140u), __byte_perm(wC, wD, 0x7362u)};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t sel = (i & 1) ? 0x4342u : 0x4140u;
        uint32_t b0 = i8x2_to_h2(ab[i >> 1], sel);
        uint32_t b1 = i8x2_to_h2(cd[i >> 1], sel);
        const __half2 h0 = __hmul2(*reinterpret_cast<const __half2*>(&b0), sAB);
        const __half2 h1 = __hmul2(*reinterpret_cast<const __half2*>(&b1), sCD);
        mma_f16_16816(S.o[gi][i], pa, *reinterpret_cast<const uint32_t*>(&h0),
                      *reinterpret_cast<const uint32_t*>(&h1));
      }
    }
  }
}

// grid: (nsplit, 2, rows); block: 32 * W threads; dynamic smem: sizeof(AttnSmem<W>).
// kAll: a.ids is NULL and every row's list is all its visible cells.
template <int W, bool kAll>
__global__ void __launch_bounds__(32 * W) attn_kernel(AttnArgs a) {
  constexpr int NT = 32 * W;
  constexpr int GW = kNG / W;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  AttnSmem<W>& sm = *reinterpret_cast<AttnSmem<W>*>(smem_raw);
  const int split = blockIdx.x, kvh = blockIdx.y, row = blockIdx.z;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int beg = min(a.top_k, split * a.piece);
  const int end = min(a.top_k, beg + a.piece);
  const int* rid = kAll ? nullptr : a.ids + static_cast<size_t>(row) * a.top_k;
  const int dv = kAll ? a.dense_vis0 + row : 0;  // implicit list: every visible cell
  const int nblk = (end - beg + kAttnCells - 1) / kAttnCells;
  griddep_launch();

  uint32_t aq[GW][2][4];
  attn_load_q<W>(aq, a.q + (static_cast<size_t>(row) * kHQ + kvh * kQPerKV) * kD, a.scale_log2, warp);
  float kb[GW][2];
  attn_k_bias<W>(kb, aq);

  // The ids come from the selection kernel: wait for it before the first gather.
  griddep_wait();
  if constexpr (kAll) {
    if (a.ids_fill && kvh == 0)  // this piece of the implicit list, for the caller
      for (int p = beg + static_cast<int>(threadIdx.x); p < end; p += NT)
        a.ids_fill[static_cast<size_t>(row) * a.top_k + p] = p < dv ? p : -1;
  }
  // a block's ids are loaded one block before its gather is issued (the first two blocks'
  // together, so the second gather does not wait for its ids)
  AttnIds<NT> ids;
  auto load_ids = [&](AttnIds<NT>& dst, int blk) {
    const int p0 = beg + blk * kAttnCells;
    attn_load_ids<NT>(dst, static_cast<int>(threadIdx.x),
                      [&](int i) { return attn_cell<kAll>(rid, dv, p0 + i, end); });
  };
  static_assert(kAttnStages == 2, "the id prefetch below assumes a double-buffered ring");
  if (nblk > 0) {
    AttnIds<NT> ids0;
    load_ids(ids0, 0);
    if (nblk > 1) load_ids(ids, 1);
    attn_gather<NT>(sm.st[0], a, kvh, static_cast<int>(threadIdx.x), ids0);
  }
  cp_async_commit();

  AttnState<W> S;
  S.init();
  for (int b = 0; b < nblk; ++b) {
    // block b has landed for every thread, and every warp has finished block b - 1 (its
    // stage and the partial-score exchange are free again)
    cp_async_wait<0>();
    __syncthreads();
    // refill the stage block b - 1 used
    const int nb = b + 1;
    if (nb < nblk) attn_gather<NT>(sm.st[nb % kAttnStages], a, kvh, static_cast<int>(threadIdx.x), ids);
    cp_async_commit();
    if (nb + 1 < nblk) load_ids(ids, nb + 1);
    attn_block<W>(sm.st[b % kAttnStages], sm.red, aq, kb, S, warp, [] { __syncthreads(); });
  }
  cp_async_wait<0>();

  // ---- epilogue: rows g (heads 12kvh + g) and g + 8 (heads 12kvh + g + 8, g < 4)
  // C element (row, col 2t) of n-tile i, group qg is dim 32qg + 8t + i; col 2t+1 is +4.
  const float kLn2 = 0.6931471805599453f;
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int hr = g + 8 * r;
    if (hr >= kQPerKV) continue;
    const int head = kvh * kQPerKV + hr;
    const size_t rh = static_cast<size_t>(row) * kHQ + head;
#pragma unroll
    for (int gi = 0; gi < GW; ++gi) {
      const int dbase = 32 * (GW * warp + gi) + 8 * t;
      float4 lo = make_float4(S.o[gi][0][2 * r], S.o[gi][1][2 * r], S.o[gi][2][2 * r], S.o[gi][3][2 * r]);
      float4 hi = make_float4(S.o[gi][0][2 * r + 1], S.o[gi][1][2 * r + 1], S.o[gi][2][2 * r + 1],
                              S.o[gi][3][2 * r + 1]);
      if (a.nsplit == 1) {
        const float inv = S.l_run[r] > 0.f ? 1.f / S.l_run[r] : 0.f;
        lo.x *= inv; lo.y *= inv; lo.z *= inv; lo.w *= inv;
        hi.x *= inv; hi.y *= inv; hi.z *= inv; hi.w *= inv;
        if (a.gate) {
          const float4 ga = __ldg(reinterpret_cast<const float4*>(a.gate + rh * kD + dbase));
          const float4 gb = __ldg(reinterpret_cast<const float4*>(a.gate + rh * kD + dbase + 4));
          lo.x *= gate_factor(ga.x); lo.y *= gate_factor(ga.y); lo.z *= gate_factor(ga.z); lo.w *= gate_factor(ga.w);
          hi.x *= gate_factor(gb.x); hi.y *= gate_factor(gb.y); hi.z *= gate_factor(gb.z); hi.w *= gate_factor(gb.w);
        }
        float* dst = a.out + rh * kD + dbase;
        *reinterpret_cast<float4*>(dst) = lo;
        *reinterpret_cast<float4*>(dst + 4) = hi;
      } else {  // partials relative to the true maximum
        const float corr = (S.m_top[r] == -INFINITY) ? 0.f : attn_exp2(S.m_run[r] - S.m_top[r]);
        lo.x *= corr; lo.y *= corr; lo.z *= corr; lo.w *= corr;
        hi.x *= corr; hi.y *= corr; hi.z *= corr; hi.w *= corr;
        float* dst = a.part + (rh * a.nsplit + split) * kPart;
        *reinterpret_cast<float2*>(dst + 2 + dbase) = make_float2(lo.x, lo.y);
        *reinterpret_cast<float2*>(dst + 2 + dbase + 2) = make_float2(lo.z, lo.w);
        *reinterpret_cast<float2*>(dst + 2 + dbase + 4) = make_float2(hi.x, hi.y);
        *reinterpret_cast<float2*>(dst + 2 + dbase + 6) = make_float2(hi.z, hi.w);
        if (warp == 0 && t == 0) {
          dst[0] = S.m_top[r] == -INFINITY ? -INFINITY : S.m_top[r] * kLn2;
          dst[1] = S.l_run[r] * corr;
        }
      }
    }
  }
}

}  // namespace qsa
