// Router logits, routing (softmax / top-k / gates / stable ranks) and the scan
// that turns per-chunk expert histograms into counts, capacity cuts, padded
// segment offsets and the Switch balance statistic.
//
// Sources: Zero to Frontier 13.1 "Why MoE", "The MoE layer" (r = x W_r, TopK,
// gates = softmax over the kept logits); kevinluzbetak "Mixture-Of-Experts",
// routing paragraph (softmax over all, top-k, renormalise) and balancing list
// (E * sum_i f_i P_i); AI Engineering Illustrated "Mixture of Experts", "The
// router is small but it decides everything" (router in float32) and "The
// safety valve is a capacity limit".
#pragma once
#include "common.cuh"
#include <math.h>

namespace moe {

// ---------------------------------------------------------------------------
// SIMT fp32 "TN" GEMM: C[m, n] = sum_k A[m, k] * B[e][n, k], both operands
// K-contiguous, fp32 FMA accumulation (no TF32). Used for the fp32 layer's
// expert products, where the rows of A are grouped per expert in
// ROW_TILE-padded segments; grid z selects the routed or the shared group.
// ---------------------------------------------------------------------------
enum { EPI_SWIGLU = 1, EPI_SCALE = 2 };

struct SimtGroup {
  const void* A;            // [rows, K]
  const void* B0;           // expert e at B0 + e * b_stride  ([N, K] each)
  const void* B1;           // second operand of the SwiGLU (up projection)
  int64_t b_stride;         // elements between experts
  void* C;                  // [rows, N]
  const float* row_scale;   // EPI_SCALE: multiplier per row (NULL = 1)
  const int32_t* tile_start;// grouped rows: [E + 1] segment starts in ROW_TILE units; NULL = dense
  int E;
  int64_t rows;             // dense: number of valid rows
  int N, K;
  int active;               // 0: this grid z-slice does nothing
};

constexpr int SG_BM = 64, SG_BN = 64, SG_BK = 32;

template <typename TA>
__device__ __forceinline__ void load4(const TA* p, float* f);
template <>
__device__ __forceinline__ void load4<float>(const float* p, float* f) {
  float4 v = *reinterpret_cast<const float4*>(p);
  f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
}
template <>
__device__ __forceinline__ void load4<__nv_bfloat16>(const __nv_bfloat16* p, float* f) {
  uint2 v = *reinterpret_cast<const uint2*>(p);
  float2 a = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&v.x));
  float2 b = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&v.y));
  f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y;
}

// 64x64 output tile per 256-thread block, 4x4 outputs per thread, K tiles of
// 32 staged in shared memory; the next tile's global loads are issued before
// the current tile is consumed. Each K tile is summed into a fresh partial
// that is then added to the running total (blocked summation), which keeps
// the rounding error of a long dot product well below one sequential chain.
template <typename TA, typename TB, typename TC, int EPI>
__global__ void __launch_bounds__(256) simt_gemm_kernel(SimtGroup g0, SimtGroup g1) {
  pdl_wait();
  pdl_launch_dependents();
  const SimtGroup g = blockIdx.z == 0 ? g0 : g1;
  if (!g.active) return;
  const int k_len = g.K;
  const int k_begin = 0;
  const int n0 = blockIdx.x * SG_BN;
  const int64_t m0 = (int64_t)blockIdx.y * SG_BM;
  if (n0 >= g.N) return;
  int e = 0;
  int64_t m_end;
  if (g.tile_start) {
    const int64_t total = (int64_t)g.tile_start[g.E] * ROW_TILE;
    if (m0 >= total) return;
    int lo = 0, hi = g.E - 1;  // last expert whose segment starts at or before m0
    while (lo < hi) {
      int mid = (lo + hi + 1) >> 1;
      if ((int64_t)g.tile_start[mid] * ROW_TILE <= m0) lo = mid; else hi = mid - 1;
    }
    e = lo;
    m_end = (int64_t)g.tile_start[e + 1] * ROW_TILE;
  } else {
    if (m0 >= g.rows) return;
    m_end = g.rows;
  }
  constexpr int NB = (EPI == EPI_SWIGLU) ? 2 : 1;
  __shared__ __align__(16) float As[SG_BK][SG_BM + 4];
  __shared__ __align__(16) float Bs[NB][SG_BK][SG_BN + 4];

  const int tid = threadIdx.x;
  const int lr = tid >> 2, lk = (tid & 3) * 8;  // row within the tile, first of 8 K elements
  const int ty = tid >> 4, tx = tid & 15;
  const TA* A = reinterpret_cast<const TA*>(g.A);
  const TB* Bp[2] = {reinterpret_cast<const TB*>(g.B0) + (int64_t)e * g.b_stride,
                     NB == 2 ? reinterpret_cast<const TB*>(g.B1) + (int64_t)e * g.b_stride : nullptr};
  float acc[NB][4][4];
#pragma unroll
  for (int b = 0; b < NB; ++b)
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[b][i][j] = 0.f;

  const int64_t arow = m0 + lr;
  const int brow = n0 + lr;
  const bool a_ok = arow < m_end, b_ok = brow < g.N;
  float fa[8], fb[NB][8];
  auto fetch = [&](int k0) {
#pragma unroll
    for (int i = 0; i < 8; ++i) fa[i] = 0.f;
    if (a_ok) {
      load4<TA>(A + arow * g.K + k0 + lk, fa);
      load4<TA>(A + arow * g.K + k0 + lk + 4, fa + 4);
    }
#pragma unroll
    for (int b = 0; b < NB; ++b) {
#pragma unroll
      for (int i = 0; i < 8; ++i) fb[b][i] = 0.f;
      if (b_ok) {
        load4<TB>(Bp[b] + (int64_t)brow * g.K + k0 + lk, fb[b]);
        load4<TB>(Bp[b] + (int64_t)brow * g.K + k0 + lk + 4, fb[b] + 4);
      }
    }
  };
  fetch(k_begin);
  for (int k0 = k_begin; k0 < k_begin + k_len; k0 += SG_BK) {
#pragma unroll
    for (int i = 0; i < 8; ++i) As[lk + i][lr] = fa[i];
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
      for (int i = 0; i < 8; ++i) Bs[b][lk + i][lr] = fb[b][i];
    __syncthreads();
    if (k0 + SG_BK < k_begin + k_len) fetch(k0 + SG_BK);  // in flight during the compute below
    float part[NB][4][4];
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) part[b][i][j] = 0.f;
#pragma unroll
    for (int kk = 0; kk < SG_BK; ++kk) {
      float4 a = *reinterpret_cast<const float4*>(&As[kk][ty * 4]);
      float av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        float4 bq = *reinterpret_cast<const float4*>(&Bs[b][kk][tx * 4]);
        float bv[4] = {bq.x, bq.y, bq.z, bq.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) part[b][i][j] = fmaf(av[i], bv[j], part[b][i][j]);
      }
    }
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[b][i][j] += part[b][i][j];
    __syncthreads();
  }

  TC* C = reinterpret_cast<TC*>(g.C);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t m = m0 + ty * 4 + i;
    if (m >= m_end) continue;
    float scale = 1.f;
    if (EPI == EPI_SCALE && g.row_scale) scale = g.row_scale[m];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= g.N) continue;
      float v;
      if (EPI == EPI_SWIGLU) {
        const float a = acc[0][i][j];
        v = (a / (1.0f + expf(-a))) * acc[NB - 1][i][j];
      } else if (EPI == EPI_SCALE) {
        v = scale * acc[0][i][j];
      } else {
        v = acc[0][i][j];
      }
      C[m * g.N + n] = from_f32<TC>(v);
    }
  }
}

// ---------------------------------------------------------------------------
// Router logits for many experts (E > 16): r[t, e] = sum_j x[t, j] W_r[e, j]
// in fp32 FMA. 128 tokens x 128 experts per block, 256 threads, each thread
// 8 tokens x 8 experts, so a K step reads 16 operand values from shared memory
// for 64 FMAs. The sum is blocked like the generic kernel's: 32-term partials
// added to the accumulator, in a fixed order; grid.z splits K into
// RW_BK-multiple ranges whose partials the routing kernel adds in order.
// ---------------------------------------------------------------------------
constexpr int RW_BM = 128, RW_BN = 128, RW_BK = 32;

// K splits for the wide router: enough blocks to fill the SMs; K ranges stay
// whole multiples of RW_BK. Depends only on the shape.
inline int router_wide_split_k(int64_t T, int E, int K) {
  const int64_t blocks = ((E + RW_BN - 1) / RW_BN) * ((T + RW_BM - 1) / RW_BM);
  int split = 1;
  while (blocks * split < 296 && (K % (2 * split * RW_BK)) == 0 && K / (2 * split) >= 512)
    split *= 2;
  return split;
}

template <typename TA>
__global__ void __launch_bounds__(256, 1) router_wide_kernel(const TA* __restrict__ x,
                                                             const float* __restrict__ W_r,
                                                             int T, int K, int E, int splits,
                                                             float* __restrict__ logits) {
  pdl_wait();
  pdl_launch_dependents();
  __shared__ __align__(16) float As[RW_BK][RW_BM + 4];
  __shared__ __align__(16) float Bs[RW_BK][RW_BN + 4];
  const int k_len = K / splits;
  const int k_begin = (int)blockIdx.z * k_len;
  const int n0 = blockIdx.x * RW_BN;
  const int m0 = blockIdx.y * RW_BM;
  const int tid = threadIdx.x;
  const int lr = tid >> 1, lk = (tid & 1) * 16;  // staging: row lr, K elements lk .. lk+15
  const int ty = tid >> 4, tx = tid & 15;         // compute: rows 8ty.., columns 8tx..
  const bool a_ok = m0 + lr < T, b_ok = n0 + lr < E;
  const TA* arow = x + (int64_t)(m0 + lr) * K;
  const float* brow = W_r + (int64_t)(n0 + lr) * K;
  float fa[16], fb[16];
  auto fetch = [&](int k0) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if (a_ok) load4<TA>(arow + k0 + lk + 4 * q, fa + 4 * q);
      else fa[4 * q] = fa[4 * q + 1] = fa[4 * q + 2] = fa[4 * q + 3] = 0.f;
      if (b_ok) load4<float>(brow + k0 + lk + 4 * q, fb + 4 * q);
      else fb[4 * q] = fb[4 * q + 1] = fb[4 * q + 2] = fb[4 * q + 3] = 0.f;
    }
  };
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
  fetch(k_begin);
  for (int k0 = k_begin; k0 < k_begin + k_len; k0 += RW_BK) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      As[lk + i][lr] = fa[i];
      Bs[lk + i][lr] = fb[i];
    }
    __syncthreads();
    if (k0 + RW_BK < k_begin + k_len) fetch(k0 + RW_BK);  // in flight during the compute
    float part[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) part[i][j] = 0.f;
#pragma unroll 4
    for (int kk = 0; kk < RW_BK; ++kk) {
      const float4 a0 = *reinterpret_cast<const float4*>(&As[kk][ty * 8]);
      const float4 a1 = *reinterpret_cast<const float4*>(&As[kk][ty * 8 + 4]);
      const float4 b0 = *reinterpret_cast<const float4*>(&Bs[kk][tx * 8]);
      const float4 b1 = *reinterpret_cast<const float4*>(&Bs[kk][tx * 8 + 4]);
      const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) part[i][j] = fmaf(av[i], bv[j], part[i][j]);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[i][j] += part[i][j];
    __syncthreads();
  }
  float* C = logits + (int64_t)blockIdx.z * T * E;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int m = m0 + ty * 8 + i;
    if (m >= T) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int n = n0 + tx * 8 + j;
      if (n < E) C[(int64_t)m * E + n] = acc[i][j];
    }
  }
}

// ---------------------------------------------------------------------------
// Router logits for few experts (E <= NE, NE = 8 or 16): r[t, e] = sum_j x[t, j] W_r[e, j].
// This is bound by reading x, so there is no wasted output tile. A block
// owns NARROW_TB tokens and one K range (grid.y splits K; the routing kernel
// sums the split partials in a fixed order). Router rows are staged in shared
// memory 256 columns at a time and read by all 8 warps. Warp w owns tokens
// w*TOK .. w*TOK+TOK-1, and lane l takes columns 8l..8l+7 of each chunk.
// Every (token, expert) keeps one fp32 partial per lane: a chunk adds a dot
// of 8 terms to it (blocked summation), and the 32 lane partials are then
// summed by a fixed butterfly. The result is deterministic.
// ---------------------------------------------------------------------------
constexpr int NARROW_KC = 256;  // columns per staged chunk

template <typename TA>
__device__ __forceinline__ void load8(const TA* p, float* f);
template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* p, float* f) {
  Vec16<__nv_bfloat16>::unpack(ld_nc_v4(p), f);
}
template <>
__device__ __forceinline__ void load8<float>(const float* p, float* f) {
  Vec16<float>::unpack(ld_nc_v4(p), f);
  Vec16<float>::unpack(ld_nc_v4(p + 4), f + 4);
}

template <int NE> struct NarrowShape {
  static constexpr int TOK = NE <= 8 ? 8 : 4;  // tokens per warp
  static constexpr int TB = 8 * TOK;           // tokens per block
};

// K chunks for the narrow router: enough blocks for about two waves.
inline int narrow_split_k(int64_t T, int E, int d) {
  const int tb = E <= 8 ? NarrowShape<8>::TB : NarrowShape<16>::TB;
  const int64_t blocks = (T + tb - 1) / tb;
  const int chunks = d / NARROW_KC > 0 ? d / NARROW_KC : 1;
  int split = 1;
  while (blocks * split < 296 && split * 2 <= chunks) split *= 2;
  return split;
}

template <typename TA, int NE>
__global__ void __launch_bounds__(256) router_narrow_kernel(const TA* __restrict__ x,
                                                            const float* __restrict__ W_r, int T,
                                                            int d, int E, int splits,
                                                            float* __restrict__ logits) {
  pdl_wait();
  pdl_launch_dependents();
  constexpr int TOK = NarrowShape<NE>::TOK;
  constexpr int TB = NarrowShape<NE>::TB;
  __shared__ __align__(16) float ws[NE][NARROW_KC];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * TB + warp * TOK;
  // K range of this split: whole chunks, the last split takes the remainder
  const int chunks = (d + NARROW_KC - 1) / NARROW_KC;
  const int per = (chunks + splits - 1) / splits;
  const int c_begin = blockIdx.y * per;
  const int c_end = c_begin + per < chunks ? c_begin + per : chunks;
  float acc[TOK][NE];
#pragma unroll
  for (int t = 0; t < TOK; ++t)
#pragma unroll
    for (int e = 0; e < NE; ++e) acc[t][e] = 0.f;
  for (int c = c_begin; c < c_end; ++c) {
    const int k0 = c * NARROW_KC;
    const int kw = d - k0 < NARROW_KC ? d - k0 : NARROW_KC;  // a multiple of 8
    __syncthreads();  // previous chunk fully consumed
    for (int i = threadIdx.x; i < NE * (NARROW_KC / 4); i += blockDim.x) {
      const int e = i / (NARROW_KC / 4), q = (i % (NARROW_KC / 4)) * 4;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (e < E && q < kw) v = *reinterpret_cast<const float4*>(W_r + (size_t)e * d + k0 + q);
      *reinterpret_cast<float4*>(&ws[e][q]) = v;
    }
    const int j = lane * 8;
    float xv[TOK][8];
#pragma unroll
    for (int t = 0; t < TOK; ++t) {
      if (t0 + t < T && j < kw) load8<TA>(x + (size_t)(t0 + t) * d + k0 + j, xv[t]);
      else
#pragma unroll
        for (int i = 0; i < 8; ++i) xv[t][i] = 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int e = 0; e < NE; ++e) {
      const float4 w0 = *reinterpret_cast<const float4*>(&ws[e][j]);
      const float4 w1 = *reinterpret_cast<const float4*>(&ws[e][j + 4]);
      const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
      for (int t = 0; t < TOK; ++t) {
        float part = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) part = fmaf(xv[t][i], wv[i], part);
        acc[t][e] += part;
      }
    }
  }
#pragma unroll
  for (int t = 0; t < TOK; ++t)
#pragma unroll
    for (int e = 0; e < NE; ++e) {
      float v = acc[t][e];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      acc[t][e] = v;
    }
  // lane (t * NE + e) % 32 writes output (t, e)
  float* out = logits + (size_t)blockIdx.y * T * E;
#pragma unroll
  for (int t = 0; t < TOK; ++t)
#pragma unroll
    for (int e = 0; e < NE; ++e)
      if (lane == ((t * NE + e) & 31) && e < E && t0 + t < T)
        out[(size_t)(t0 + t) * E + e] = acc[t][e];
}

// ---------------------------------------------------------------------------
// Routing: ROUTE_CHUNK tokens per block, ROUTE_WARPS warps, each warp owning
// ROUTE_CHUNK / ROUTE_WARPS consecutive tokens, one token at a time:
//   softmax over all E logits (+ optional bias), per-expert probability sums
//   accumulated in fp64 in a fixed order; top-k by k rounds of a warp argmax
//   ordered by (logit descending, index ascending); gates as a softmax over
//   the k kept logits. Then stable ranks: for each assignment, how many
//   earlier tokens of the same chunk chose the same expert (a 32-bit token
//   mask per 32-token group and expert, prefix-summed over the groups).
// Outputs per block: hist[blk][e] and the block's probability sums (the
// warps' fp64 partials added in warp order).
// NV = ceil(E / 32) logits held per lane.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

constexpr int ROUTE_TOK_PER_WARP = ROUTE_CHUNK / ROUTE_WARPS;
constexpr int ROUTE_FAST_SPLITS = 16;  // K-split partials loaded together (few experts)
constexpr int ROUTE_RANK_GROUPS = ROUTE_CHUNK / 32;
static_assert(ROUTE_CHUNK % 32 == 0 && ROUTE_RANK_GROUPS <= ROUTE_WARPS, "route chunk shape");

// Dynamic shared memory of route_kernel for E experts.
__host__ __device__ constexpr size_t route_smem_bytes(int E) {
  return (size_t)ROUTE_WARPS * E * 8 + (size_t)2 * ROUTE_RANK_GROUPS * E * 4;
}

enum { GATE_RENORM = 0, GATE_RAW = 1, GATE_SIGMOID = 2 };

// ---------------------------------------------------------------------------
// Scan over experts (one block, thread e = expert e, E <= nthreads, nthreads a
// power of two <= 1024):
//   base[b][e]   = assignments to e in chunks before b (stable token-order rank base)
//   counts[e]    = routed assignments to e (before the capacity cut)
//   kept_e       = min(counts[e], C); segment of ceil(kept_e / ROW_TILE) tiles
//   tile_start   = exclusive scan of the segment sizes; tile_start[E] = total
//   pair_start   = exclusive scan of ceil(segment tiles / 2) (CTA-pair tiles)
//   probsum[e]   = sum of the probability partials, fp64, fixed order
//   aux          = E * sum_e (counts_e / (T k)) (probsum_e / T), fp64, fixed tree
// and clears the call's status word. s_scan holds 2 * nthreads ints, s_sum
// nthreads doubles. Every thread of the block must call it.
// ---------------------------------------------------------------------------
__device__ void scan_experts(int nthreads, const int32_t* __restrict__ hist, int nblk,
                             const double* __restrict__ psum_part, int nparts, int E, int64_t T,
                             int k, int64_t C, int32_t* __restrict__ counts,
                             int32_t* __restrict__ base, int32_t* __restrict__ tile_start,
                             int32_t* __restrict__ pair_start, double* __restrict__ probsum,
                             float* __restrict__ aux, int* __restrict__ call_err, int64_t rows_max,
                             int* s_scan, double* s_sum, int* s_cnt = nullptr,
                             double* s_psd = nullptr) {
  const int e = threadIdx.x;
  if (e == 0 && call_err != nullptr) *call_err = 0;  // the GEMMs of this call run after this
  if (s_cnt != nullptr) {
    // A warp per expert: each lane takes a contiguous range of chunks, a shuffle
    // scan turns the range sums into each range's start, and the lanes write the
    // chunks' bases; the probability partials are loaded 32 at a time and added
    // in part order, as one thread would.
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    const int per = (nblk + 31) / 32;
    for (int ee = warp; ee < E; ee += nw) {
      const int b0 = lane * per < nblk ? lane * per : nblk;
      const int b1 = b0 + per < nblk ? b0 + per : nblk;
      int local = 0;
      for (int b = b0; b < b1; ++b) local += hist[(size_t)b * E + ee];
      int incl = local;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += t;
      }
      int run = incl - local;
      for (int b = b0; b < b1; ++b) {
        base[(size_t)b * E + ee] = run;
        run += hist[(size_t)b * E + ee];
      }
      const int total = __shfl_sync(0xffffffffu, incl, 31);
      double ps = 0.0;
      for (int p0 = 0; p0 < nparts; p0 += 32) {
        const double v = p0 + lane < nparts ? psum_part[(size_t)(p0 + lane) * E + ee] : 0.0;
        const int n = nparts - p0 < 32 ? nparts - p0 : 32;
        for (int j = 0; j < n; ++j) ps += __shfl_sync(0xffffffffu, v, j);
      }
      if (lane == 0) {
        s_cnt[ee] = total;
        s_psd[ee] = ps;
      }
    }
    __syncthreads();
  }
  int tiles = 0;
  double term = 0.0;
  if (e < E) {
    int run = 0;
    double ps = 0.0;
    if (s_cnt != nullptr) {
      run = s_cnt[e];
      ps = s_psd[e];
    } else {
#pragma unroll 8
      for (int b = 0; b < nblk; ++b) {
        base[(size_t)b * E + e] = run;
        run += hist[(size_t)b * E + e];
      }
#pragma unroll 8
      for (int p = 0; p < nparts; ++p) ps += psum_part[(size_t)p * E + e];
    }
    counts[e] = run;
    const int kept = (C >= 0 && (int64_t)run > C) ? (int)C : run;
    tiles = (kept + ROW_TILE - 1) / ROW_TILE;
    probsum[e] = ps;
    term = (double)run * ps;
  }
  if (e < nthreads) {
    s_scan[e] = tiles;
    s_sum[e] = term;
  }
  __syncthreads();
  int cur = 0;
  for (int off = 1; off < nthreads; off <<= 1) {  // inclusive Hillis-Steele scan
    if (e < nthreads) {
      const int v = s_scan[cur * nthreads + e] + (e >= off ? s_scan[cur * nthreads + e - off] : 0);
      s_scan[(cur ^ 1) * nthreads + e] = v;
    }
    cur ^= 1;
    __syncthreads();
  }
  if (e < E) tile_start[e] = s_scan[cur * nthreads + e] - tiles;
  if (e == E - 1) {
    tile_start[E] = s_scan[cur * nthreads + e];
#if defined(MOE_DEBUG)
    if ((int64_t)s_scan[cur * nthreads + e] * ROW_TILE > rows_max) flag_bounds();
#else
    (void)rows_max;
#endif
  }
  // the same scan over pairs of tiles (a CTA pair computes two tiles of one expert)
  const int pairs = (tiles + 1) / 2;
  __syncthreads();
  if (e < nthreads) s_scan[e] = pairs;
  cur = 0;
  __syncthreads();
  for (int off = 1; off < nthreads; off <<= 1) {
    if (e < nthreads) {
      const int v = s_scan[cur * nthreads + e] + (e >= off ? s_scan[cur * nthreads + e - off] : 0);
      s_scan[(cur ^ 1) * nthreads + e] = v;
    }
    cur ^= 1;
    __syncthreads();
  }
  if (e < E) pair_start[e] = s_scan[cur * nthreads + e] - pairs;
  if (e == E - 1) pair_start[E] = s_scan[cur * nthreads + e];
  for (int half = nthreads / 2; half > 0; half >>= 1) {  // fixed-shape tree sum
    if (e < half) s_sum[e] += s_sum[e + half];
    __syncthreads();
  }
  if (e == 0) {
    const double denom = (double)T * (double)k * (double)T;
    aux[0] = (T > 0) ? (float)((double)E * s_sum[0] / denom) : 0.f;
  }
}

// Threads of the scan for E experts.
__host__ __device__ inline int scan_threads(int E) {
  int n = 32;
  while (n < E) n <<= 1;
  return n;
}
// Threads of the scan kernel. Up to 32 experts: a warp per expert (at least 8
// warps) walks the expert's chunks in parallel; above that a thread per expert
// walks them in sequence, as many experts at once.
constexpr int SCAN_WARP_PATH_MAX_E = 32;
__host__ __device__ inline int scan_kernel_threads(int E) {
  if (E <= SCAN_WARP_PATH_MAX_E) return 32 * E < 256 ? 256 : 32 * E;
  return scan_threads(E);
}

// Arguments of the scan when the routing kernel runs it itself (one chunk).
struct ScanArgs {
  bool fused;
  int64_t C, rows_max;
  int32_t* counts;
  int32_t* base;
  int32_t* tile_start;
  int32_t* pair_start;
  double* probsum;
  float* aux;
  int* call_err;
};

template <int NV>
__global__ void __launch_bounds__(256, 1) route_kernel(
    float* __restrict__ logits, int splits, const float* __restrict__ bias,
    const float* __restrict__ sel_bias, int gate_mode, int n_group, int topk_group, int T, int E,
    int k, int32_t* __restrict__ idx_out, float* __restrict__ gate_out,
    int32_t* __restrict__ lrank_out, int32_t* __restrict__ hist, double* __restrict__ psum_part,
    const ScanArgs sa) {
  pdl_wait();
  pdl_launch_dependents();
  extern __shared__ __align__(16) uint8_t route_smem_raw[];
  double* red = reinterpret_cast<double*>(route_smem_raw);  // [ROUTE_WARPS][E]
  uint32_t* bm = reinterpret_cast<uint32_t*>(red + (size_t)ROUTE_WARPS * E);  // [groups][E]
  int32_t* wbase = reinterpret_cast<int32_t*>(bm + (size_t)ROUTE_RANK_GROUPS * E);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int blk = blockIdx.x;
  for (int i = threadIdx.x; i < ROUTE_RANK_GROUPS * E; i += blockDim.x) bm[i] = 0u;

  // Warp w takes the chunk's tokens w, w + 8, w + 16, ... (interleaved, so that
  // a short batch still keeps every warp busy).
  auto tok = [&](int j) { return blk * ROUTE_CHUNK + j * ROUTE_WARPS + warp; };
  const bool grouped = n_group > 1 && topk_group < n_group;
  const int gsize = grouped ? E / n_group : E;
  double ps[NV];
  float bv[NV], sb[NV];
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    ps[i] = 0.0;
    const int e = lane + 32 * i;
    bv[i] = (bias != nullptr && e < E) ? bias[e] : 0.f;
    sb[i] = (sel_bias != nullptr && e < E) ? sel_bias[e] : 0.f;
  }

  // The next token's logits are loaded (and their K-split partials summed, in
  // a fixed order) while the current token is processed. For few experts all
  // of a logit's partials are loaded before any is added, so the loads are in
  // flight together instead of one round trip after another.
  const size_t split_stride = (size_t)T * E;
  float nxt[NV];
  auto load_logits = [&](int t) {
    const float* row = logits + (size_t)t * E;
    if (NV <= 2 && splits <= ROUTE_FAST_SPLITS) {
      float part[NV][ROUTE_FAST_SPLITS];
#pragma unroll
      for (int sp = 0; sp < ROUTE_FAST_SPLITS; ++sp)
#pragma unroll
        for (int i = 0; i < NV; ++i) {
          const int e = lane + 32 * i;
          part[i][sp] = (sp < splits && e < E) ? row[sp * split_stride + e] : 0.f;
        }
#pragma unroll
      for (int i = 0; i < NV; ++i) {
        float r = part[i][0];
#pragma unroll
        for (int sp = 1; sp < ROUTE_FAST_SPLITS; ++sp)
          if (sp < splits) r += part[i][sp];
        nxt[i] = r;
      }
      return;
    }
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int e = lane + 32 * i;
      float r = 0.f;
      if (e < E) {
        r = row[e];
        for (int sp = 1; sp < splits; ++sp) r += row[sp * split_stride + e];
      }
      nxt[i] = r;
    }
  };
  if (tok(0) < T) load_logits(tok(0));
  for (int j = 0; j < ROUTE_TOK_PER_WARP; ++j) {
    const int t = tok(j);
    if (t >= T) break;  // warp-uniform
    float raw[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) raw[i] = nxt[i];
    if (j + 1 < ROUTE_TOK_PER_WARP && tok(j + 1) < T) load_logits(tok(j + 1));
    float* row = logits + (size_t)t * E;
    float v[NV];
    uint32_t removed = 0u;
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int e = lane + 32 * i;
      if (e < E) {
        if (splits > 1) row[e] = raw[i];  // the summed logit, for readers of the workspace
        v[i] = raw[i] + bv[i];
        m = fmaxf(m, v[i]);
      } else {
        v[i] = -INFINITY;
        removed |= 1u << i;
      }
    }
    // probabilities of the balance statistic; affinities in sigmoid mode
    float prob[NV], aff[NV];
    if (gate_mode == GATE_SIGMOID) {
      float ssum = 0.f;
#pragma unroll
      for (int i = 0; i < NV; ++i) {
        aff[i] = (lane + 32 * i < E) ? 1.f / (1.f + expf(-v[i])) : 0.f;
        ssum += aff[i];
      }
      ssum = warp_sum(ssum);
#pragma unroll
      for (int i = 0; i < NV; ++i) prob[i] = aff[i] / ssum;
    } else {
      m = warp_max(m);
      float s = 0.f;
#pragma unroll
      for (int i = 0; i < NV; ++i) {
        prob[i] = (lane + 32 * i < E) ? expf(v[i] - m) : 0.f;
        aff[i] = 0.f;
        s += prob[i];
      }
      s = warp_sum(s);
#pragma unroll
      for (int i = 0; i < NV; ++i) prob[i] = prob[i] / s;
    }
#pragma unroll
    for (int i = 0; i < NV; ++i)
      if (lane + 32 * i < E) ps[i] += (double)prob[i];

    // selection scores: logit or affinity, plus the selection-only bias
    float sel[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) sel[i] = (gate_mode == GATE_SIGMOID ? aff[i] : v[i]) + sb[i];
    if (grouped) {
      // group g's best score ends up in lane g; the topk_group best lanes win
      float my_gb = -INFINITY;
      for (int g = 0; g < n_group; ++g) {
        float lm = -INFINITY;
#pragma unroll
        for (int i = 0; i < NV; ++i) {
          const int e = lane + 32 * i;
          if (e < E && e / gsize == g) lm = fmaxf(lm, sel[i]);
        }
        lm = warp_max(lm);
        if (lane == g) my_gb = lm;
      }
      bool chosen = false;
      for (int rnd = 0; rnd < topk_group; ++rnd) {
        float bvv = (lane < n_group && !chosen) ? my_gb : -INFINITY;
        int bg = (lane < n_group && !chosen) ? lane : 0x7fffffff;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          const float ov = __shfl_xor_sync(0xffffffffu, bvv, o);
          const int og = __shfl_xor_sync(0xffffffffu, bg, o);
          if (ov > bvv || (ov == bvv && og < bg)) { bvv = ov; bg = og; }
        }
        if (lane == bg) chosen = true;
      }
      const uint32_t gmask = __ballot_sync(0xffffffffu, chosen);
#pragma unroll
      for (int i = 0; i < NV; ++i) {
        const int e = lane + 32 * i;
        if (e < E && !((gmask >> (e / gsize)) & 1u)) removed |= 1u << i;
      }
    }

    int my_e = 0;
    float my_g = 0.f;  // the chosen expert's gate input: logit, probability or affinity
    for (int sl = 0; sl < k; ++sl) {
      float best_v = -INFINITY;
      int best_e = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < NV; ++i) {
        if (!((removed >> i) & 1u)) {
          const int e = lane + 32 * i;
          if (sel[i] > best_v || (sel[i] == best_v && e < best_e)) { best_v = sel[i]; best_e = e; }
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, best_v, o);
        const int oe = __shfl_xor_sync(0xffffffffu, best_e, o);
        if (ov > best_v || (ov == best_v && oe < best_e)) { best_v = ov; best_e = oe; }
      }
      const int bi = best_e >> 5;
      float gin = 0.f;
#pragma unroll
      for (int i = 0; i < NV; ++i)
        if (i == bi) gin = gate_mode == GATE_RENORM ? v[i] : (gate_mode == GATE_RAW ? prob[i] : aff[i]);
      gin = __shfl_sync(0xffffffffu, gin, best_e & 31);
      if (lane == sl) { my_e = best_e; my_g = gin; }
      if ((best_e & 31) == lane) removed |= 1u << bi;
    }
    float gate;
    if (gate_mode == GATE_RENORM) {
      const float vmax = warp_max(lane < k ? my_g : -INFINITY);
      const float z = (lane < k) ? expf(my_g - vmax) : 0.f;
      gate = z / warp_sum(z);
    } else if (gate_mode == GATE_RAW) {
      gate = my_g;
    } else {
      gate = my_g / warp_sum(lane < k ? my_g : 0.f);
    }
    if (lane < k) {
      idx_out[(size_t)t * k + lane] = my_e;
      gate_out[(size_t)t * k + lane] = gate;
    }
  }
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int e = lane + 32 * i;
    if (e < E) red[(size_t)warp * E + e] = ps[i];
  }
  __syncthreads();  // every token's choices are in idx_out, every partial in red

  const int t = blk * ROUTE_CHUNK + warp * 32 + lane;  // rank phase: warps 0..groups-1
  const bool ranker = warp < ROUTE_RANK_GROUPS && t < T;
  if (ranker) {
    for (int sl = 0; sl < k; ++sl) {
      const int e = idx_out[(size_t)t * k + sl];
      atomicOr(&bm[warp * E + e], 1u << lane);
    }
  }
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    double acc = 0.0;
#pragma unroll
    for (int w = 0; w < ROUTE_WARPS; ++w) acc += red[(size_t)w * E + e];  // fixed order
    psum_part[(size_t)blk * E + e] = acc;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = 0;
#pragma unroll
    for (int g = 0; g < ROUTE_RANK_GROUPS; ++g) {
      wbase[g * E + e] = run;
      run += __popc(bm[g * E + e]);
    }
    hist[(size_t)blk * E + e] = run;
  }
  __syncthreads();
  if (ranker) {
    const uint32_t lt = (1u << lane) - 1u;
    for (int sl = 0; sl < k; ++sl) {
      const int e = idx_out[(size_t)t * k + sl];
      lrank_out[(size_t)t * k + sl] = wbase[warp * E + e] + __popc(bm[warp * E + e] & lt);
    }
  }
  if (sa.fused) {
    // a batch of one chunk (E <= 256): the scan runs here, on this chunk's
    // histogram and probability sums, instead of in a kernel of its own
    __shared__ int f_scan[2 * 256];
    __shared__ double f_sum[256];
    __syncthreads();  // hist and psum_part are written (block-visible)
    scan_experts(scan_threads(E), hist, 1, psum_part, 1, E, T, k, sa.C, sa.counts, sa.base,
                 sa.tile_start, sa.pair_start, sa.probsum, sa.aux, sa.call_err, sa.rows_max,
                 f_scan, f_sum);
  }
}

// The scan as its own kernel: one block of scan_kernel_threads(E) threads.
__global__ void __launch_bounds__(1024) scan_kernel(
    const int32_t* __restrict__ hist, int nblk, const double* __restrict__ psum_part, int nparts,
    int E, int64_t T, int k, int64_t C, int32_t* __restrict__ counts, int32_t* __restrict__ base,
    int32_t* __restrict__ tile_start, int32_t* __restrict__ pair_start,
    double* __restrict__ probsum, float* __restrict__ aux, int* __restrict__ call_err,
    int64_t rows_max) {
  pdl_wait();
  pdl_launch_dependents();
  __shared__ int s_scan[2 * 1024];
  __shared__ double s_sum[1024];
  __shared__ int s_cnt[1024];
  __shared__ double s_psd[1024];
  const bool warp_path = E <= SCAN_WARP_PATH_MAX_E;
  scan_experts(blockDim.x, hist, nblk, psum_part, nparts, E, T, k, C, counts, base, tile_start,
               pair_start, probsum, aux, call_err, rows_max, s_scan, s_sum,
               warp_path ? s_cnt : nullptr, warp_path ? s_psd : nullptr);
}


}  // namespace moe
