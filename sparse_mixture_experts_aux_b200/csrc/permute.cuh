// Permute (scatter of token rows into expert-grouped segments, with the
// capacity cut) and combine (gate-weighted un-permute plus the shared expert).
//
// Sources: Zero to Frontier 13.1 "Why MoE", "In PyTorch" (gather each
// expert's tokens into one batch, add the weighted result back; a sort by
// expert replaces the loop's bookkeeping); kevinluzbetak "Mixture-Of-Experts"
// (production layers sort tokens by expert; capacity example: overflow
// assignments skip the expert, the token keeps its other expert's term);
// AI Engineering Illustrated "Mixture of Experts", "The safety valve is a
// capacity limit".
#pragma once
#include "common.cuh"
#include <cuda_fp16.h>

namespace moe {

// Column chunk of one warp in the scatter and combine kernels: 32 lanes x
// PERMUTE_VPL 16-byte vectors. grid.y walks the chunks of a row, so a small
// batch still spreads over many SMs.
constexpr int PERMUTE_VPL = 4;
constexpr int PERMUTE_CHUNK_VECS = 32 * PERMUTE_VPL;

// One warp per (token, column chunk). Lane s (< k) resolves assignment s: its
// rank in token order within the expert is base[chunk][e] + lrank; it is kept
// when the rank is below the capacity C, and lands at row
// tile_start[e]*ROW_TILE + rank (blocks with blockIdx.y == 0 record it). The
// chunk of the token's row is then copied to every kept position with 16-byte
// loads and stores (coalesced across the warp).
// bf16 x 8 -> fp16 x 8, saturating at +-65504 (the FP8-weight GEMMs run
// f16 x f16; every bf16 value in [2^-14, 65504] converts exactly).
__device__ __forceinline__ uint4 bf16x8_to_f16x8(const uint4& u) {
  float f[8];
  Vec16<__nv_bfloat16>::unpack(u, f);
  uint4 r;
  uint32_t* o = reinterpret_cast<uint32_t*>(&r);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float a = fminf(fmaxf(f[2 * i], -65504.f), 65504.f);
    const float b = fminf(fmaxf(f[2 * i + 1], -65504.f), 65504.f);
    const __half2 h = __floats2half2_rn(a, b);
    o[i] = *reinterpret_cast<const uint32_t*>(&h);
  }
  return r;
}

// TO_F16: write the rows as fp16 (bf16 input only), for the FP8-weight GEMMs.
template <typename TX, bool TO_F16 = false>
__global__ void __launch_bounds__(256) scatter_kernel(
    const TX* __restrict__ x, int d, int T, int k, int E, int64_t C,
    const int32_t* __restrict__ idx, const float* __restrict__ gate,
    const int32_t* __restrict__ lrank, const int32_t* __restrict__ base,
    const int32_t* __restrict__ tile_start, int32_t* __restrict__ slot_pos,
    float* __restrict__ row_gate, TX* __restrict__ xp, int64_t rows_max,
    const float* __restrict__ scale_in = nullptr, float* __restrict__ scale_out = nullptr) {
  pdl_wait();
  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + warp;
  if (t >= T) return;  // warp-uniform
  int mypos = -1;
  if (lane < k) {
    const size_t a = (size_t)t * k + lane;
    const int e = idx[a];
    const int rank = base[(size_t)(t / ROUTE_CHUNK) * E + e] + lrank[a];
    if (C < 0 || (int64_t)rank < C) mypos = tile_start[e] * ROW_TILE + rank;
#if defined(MOE_DEBUG)
    // the row must lie inside its expert's segment and the permuted buffers
    if (mypos >= 0 && ((int64_t)mypos >= rows_max || mypos >= tile_start[e + 1] * ROW_TILE ||
                       e < 0 || e >= E)) {
      flag_bounds();
      mypos = -1;
    }
#endif
    if (blockIdx.y == 0) {
      if (mypos >= 0) {
        row_gate[mypos] = gate[a];
        if (scale_out != nullptr) scale_out[mypos] = scale_in[t];  // E4M3 rows' scales
      }
      slot_pos[a] = mypos;
    }
  }
  const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * d);
  const int nvec = (int)((size_t)d * sizeof(TX) / 16);
  const int c_begin = blockIdx.y * PERMUTE_CHUNK_VECS;
  const int c_end = c_begin + PERMUTE_CHUNK_VECS < nvec ? c_begin + PERMUTE_CHUNK_VECS : nvec;
  for (int s = 0; s < k; ++s) {
    const int p = __shfl_sync(0xffffffffu, mypos, s);
    if (p < 0) continue;
    uint4* dst = reinterpret_cast<uint4*>(xp + (size_t)p * d);
    for (int c = c_begin + lane; c < c_end; c += 32) {
      const uint4 v = ld_nc_v4(src + c);
      st_v4(dst + c, TO_F16 ? bf16x8_to_f16x8(v) : v);
    }
  }
}

// One warp per (token, column chunk): y[t] = sum_s Yrows[slot_pos[t][s]]
// (dropped slots skipped) + Ys[t] (shared expert, if any), summed in fp32 in
// slot order with a single rounding to the output type. Yrows already carry
// the gate factor.
template <typename TY>
__global__ void __launch_bounds__(256) combine_kernel(
    const TY* __restrict__ yrows, const TY* __restrict__ ys, const int32_t* __restrict__ slot_pos,
    int T, int k, int d, TY* __restrict__ y, int64_t rows_max) {
  pdl_wait();
  pdl_launch_dependents();
  constexpr int VN = Vec16<TY>::N;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + warp;
  if (t >= T) return;  // warp-uniform
  int mypos = (lane < k) ? slot_pos[(size_t)t * k + lane] : -1;
#if defined(MOE_DEBUG)
  if ((int64_t)mypos >= rows_max) {  // a permuted row outside the buffers
    flag_bounds();
    mypos = -1;
  }
#else
  (void)rows_max;
#endif
  const int nvec = (int)((size_t)d * sizeof(TY) / 16);
  const int c_begin = blockIdx.y * PERMUTE_CHUNK_VECS;
  const int c_end = c_begin + PERMUTE_CHUNK_VECS < nvec ? c_begin + PERMUTE_CHUNK_VECS : nvec;
  for (int c0 = c_begin; c0 < c_end; c0 += 32) {
    const int c = c0 + lane;
    const bool active = c < c_end;
    float acc[VN];
#pragma unroll
    for (int i = 0; i < VN; ++i) acc[i] = 0.f;
    // four slots' loads in flight at once (separate registers), then summed in
    // slot order, so the result is the same as one slot at a time
    for (int s0 = 0; s0 < k; s0 += 4) {
      uint4 v[4];
      bool has[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int s = s0 + j;
        const int p = __shfl_sync(0xffffffffu, mypos, s < k ? s : 0);
        has[j] = s < k && p >= 0 && active;
        if (has[j]) v[j] = ld_v4(reinterpret_cast<const uint4*>(yrows + (size_t)p * d) + c);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (!has[j]) continue;
        float f[VN];
        Vec16<TY>::unpack(v[j], f);
#pragma unroll
        for (int i = 0; i < VN; ++i) acc[i] += f[i];
      }
    }
    if (!active) continue;
    if (ys != nullptr) {
      float f[VN];
      Vec16<TY>::unpack(ld_v4(reinterpret_cast<const uint4*>(ys + (size_t)t * d) + c), f);
#pragma unroll
      for (int i = 0; i < VN; ++i) acc[i] += f[i];
    }
    st_v4(reinterpret_cast<uint4*>(y + (size_t)t * d) + c, Vec16<TY>::pack(acc));
  }
}

}  // namespace moe
