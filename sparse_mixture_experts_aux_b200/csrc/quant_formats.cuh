// Quantised expert-weight formats: on-chip decoders and the quantisers.
//
// FP8: E4M3 codes with one fp32 scale per weight row. MXFP4: E2M1 codes packed
// two per byte (the even element in the low nibble), one power-of-two E8M0
// scale per 32 weights along K, and a per-row fp32 factor 2^(the row's largest
// block exponent). The weights stay in HBM as codes, so a weight-streaming pass
// reads half (FP8) or about a quarter (MXFP4: 4.25 bits per weight) of the
// bytes of bf16 weights.
//
// Both decode to fp16 exactly: every E4M3 value and every E2M1 value is an fp16
// value, one hardware conversion per pair. An MXFP4 value is then multiplied in
// fp16 by 2^(X_block - X_row), a power of two, which is exact while
// X_block >= X_row - 23; the row factor 2^X_row (FP8: the row scale) multiplies
// the fp32 accumulator in the GEMM's epilogue. The GEMMs on these weights run
// tcgen05 kind::f16 with fp16 operands: the permuted activations arrive as fp16
// (the scatter kernel converts them; exact for 2^-14 <= |x| <= 65504,
// saturating above).
// Sources: AI Engineering Illustrated "Mixture of Experts", "Trade-offs to
// weigh" (small-batch MoE inference is limited by reading weights; quantising
// the expert weights attacks that directly); jacopoparretti "Mixture of
// experts, token by token", "Memory" (DeepSeek-V3 ships FP8 weights).
#pragma once
#include "tc_gemm.cuh"
#include <cuda_fp4.h>
#include <cuda_fp8.h>
#include <limits.h>

namespace moe {
namespace tcf8 {

enum { WQ_FP8 = 0, WQ_MXFP4 = 1 };

// Four E4M3 codes (code i in byte i of `w`) -> four fp16 values, as two f16x2
// words (codes 0,1 and codes 2,3), with the hardware conversion: one
// instruction per pair, exact for every finite code (E4M3 values, subnormals
// included, are fp16 values). Per instruction this is a quarter of the work of
// building bf16 values with integer operations, which is why the FP8-weight
// GEMMs run f16 x f16: the converters would otherwise bound the kernel.
// Codes 0x7F / 0xFF (E4M3 NaN) are never written by the quantiser.
__device__ __forceinline__ void e4m3x4_to_f16x4(uint32_t w, uint32_t& lo, uint32_t& hi) {
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, l;\n\tcvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(w));
}

// Eight E2M1 codes (two per byte, the even element in the low nibble) -> eight
// fp16 values as four f16x2 words, with the hardware conversion: one
// instruction per pair, exact (every E2M1 value is an fp16 value).
__device__ __forceinline__ void e2m1x8_to_f16x8(uint32_t w, uint32_t* o) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\tcvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\tcvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(o[0]), "=r"(o[1]), "=r"(o[2]), "=r"(o[3])
      : "r"(w));
}

// The fp16 multiplier 2^(X - 127) / row_factor of one MXFP4 block: a power of
// two when the row factor is one (2^X_row), exact in fp16 down to 2^-24. For
// exponent codes 1..254, 2^(X - 127) is a normal fp32 built from its bits, and
// one multiply gives the correctly rounded product, the value ldexpf returns;
// codes 0 and 255 take ldexpf itself.
__device__ __forceinline__ uint32_t mx_block_multiplier(uint32_t e8m0, float inv_row_factor) {
  const float m = (e8m0 - 1u < 254u) ? __uint_as_float(e8m0 << 23) * inv_row_factor
                                     : ldexpf(inv_row_factor, (int)e8m0 - 127);
  const __half2 h = __float2half2_rn(m);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Sixteen MXFP4 codes (8 bytes) of one block -> sixteen fp16 values
// code * multiplier, as eight f16x2 words.
__device__ __forceinline__ void mxfp4x16_to_f16x16(uint2 c, uint32_t mult, uint32_t* o) {
  e2m1x8_to_f16x8(c.x, o);
  e2m1x8_to_f16x8(c.y, o + 4);
  const __half2 m = *reinterpret_cast<const __half2*>(&mult);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    __half2 v = *reinterpret_cast<const __half2*>(&o[i]);
    v = __hmul2(v, m);
    o[i] = *reinterpret_cast<const uint32_t*>(&v);
  }
}

// Instruction descriptor, kind::f16 with A and B fp16 (format 0), D fp32.
__host__ __device__ constexpr uint32_t make_idesc_f16(int M, int N) {
  return (1u << 4) | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}


// ---------------------------------------------------------------------------
// Per-row E4M3 quantisation of expert weights (run once, outside the forward
// pass): scale = absmax / 448 (1 for an all-zero row), code = E4M3(w / scale)
// with round-to-nearest-even and saturation to +-448.
// ---------------------------------------------------------------------------
template <typename TW>
__global__ void __launch_bounds__(256) quantize_rows_fp8_kernel(
    const TW* __restrict__ w, int64_t rows, int cols, uint8_t* __restrict__ codes,
    float* __restrict__ scales, const int32_t* __restrict__ tile_start = nullptr,
    const int32_t* __restrict__ counts = nullptr, int E = 0, int64_t C = -1) {
  pdl_wait();
  pdl_launch_dependents();
  // Rows of the permuted buffers (tile_start given): only the rows an expert
  // actually holds (min(count, C) at the head of its 128-row segments) are
  // quantised; the padding rows behind them are left alone.
  if (tile_start != nullptr) rows = min(rows, (int64_t)tile_start[E] * ROW_TILE);
  constexpr int VN = Vec16<TW>::N;  // elements per 16-byte vector
  const int nvec = cols / VN;       // cols is a multiple of 16
  __shared__ float red[8];
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    if (tile_start != nullptr) {
      int lo = 0, hi = E - 1;  // the expert whose segment holds row r
      const int tr = (int)(r / ROW_TILE);
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (tile_start[mid] <= tr) lo = mid; else hi = mid - 1;
      }
      const int64_t kept = C < 0 ? counts[lo] : min((int64_t)counts[lo], C);
      if (r - (int64_t)tile_start[lo] * ROW_TILE >= kept) continue;  // block-uniform
    }
    const uint4* wr = reinterpret_cast<const uint4*>(w + r * cols);
    float m = 0.f;
    for (int c = threadIdx.x; c < nvec; c += blockDim.x) {
      float f[VN];
      Vec16<TW>::unpack(ld_nc_v4(wr + c), f);
#pragma unroll
      for (int i = 0; i < VN; ++i) m = fmaxf(m, fabsf(f[i]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    float absmax = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) absmax = fmaxf(absmax, red[i]);
    const float scale = absmax > 0.f ? absmax / 448.0f : 1.0f;
    uint8_t* cr = codes + r * cols;
    for (int c = threadIdx.x; c < nvec; c += blockDim.x) {
      float f[VN];
      Vec16<TW>::unpack(ld_nc_v4(wr + c), f);
      uint32_t packed[VN / 4];
#pragma unroll
      for (int j = 0; j < VN / 4; ++j) {
        uint32_t v = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i)
          v |= static_cast<uint32_t>(
                   __nv_cvt_float_to_fp8(f[4 * j + i] / scale, __NV_SATFINITE, __NV_E4M3))
               << (8 * i);
        packed[j] = v;
      }
      if (VN == 8)
        *reinterpret_cast<uint2*>(cr + c * VN) = make_uint2(packed[0], packed[VN / 4 - 1]);
      else
        *reinterpret_cast<uint32_t*>(cr + c * VN) = packed[0];
    }
    if (threadIdx.x == 0) scales[r] = scale;
    __syncthreads();
  }
}

// out[r][c] = value(codes[r][c]) * scales[r] in fp32, decoding each code with
// the routine the GEMM converters use. One thread per 16 codes.
__global__ void __launch_bounds__(256) dequantize_rows_fp8_kernel(const uint8_t* __restrict__ codes,
                                                                  const float* __restrict__ scales,
                                                                  int64_t rows, int cols,
                                                                  float* __restrict__ out) {
  const int64_t vec_per_row = cols / 16;
  const int64_t n = rows * vec_per_row;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / vec_per_row;
    const float s = scales[r];
    const uint4 v = ld_nc_v4(codes + i * 16);
    const uint32_t in[4] = {v.x, v.y, v.z, v.w};
    float4* o = reinterpret_cast<float4*>(out + i * 16);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t lo, hi;
      e4m3x4_to_f16x4(in[j], lo, hi);
      const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&lo));
      const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&hi));
      o[j] = make_float4(a.x * s, a.y * s, b.x * s, b.y * s);
    }
  }
}

// ---------------------------------------------------------------------------
// Per-block MXFP4 quantisation of weight rows (run once, outside the forward
// pass). For each block of 32 consecutive weights of a row: X = floor(log2
// absmax) - 2 (0 for an all-zero block), the codes are the E2M1 values nearest
// to w / 2^X (ties to even, saturating at +-6), two per byte with the even
// element in the low nibble, and the block byte is X + 127 (E8M0). The row
// factor is 2^(the largest X among the row's non-zero blocks), 1 if none.
// One thread per block (cols / 32 per row); a block of 256 threads per row.
// ---------------------------------------------------------------------------
template <typename TW>
__global__ void __launch_bounds__(256) quantize_rows_mxfp4_kernel(
    const TW* __restrict__ w, int64_t rows, int cols, uint8_t* __restrict__ codes,
    uint8_t* __restrict__ bscales, float* __restrict__ row_factor) {
  constexpr int VN = Vec16<TW>::N;  // elements per 16-byte vector
  const int nblk = cols / 32;
  __shared__ int red[8];
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    int xmax = INT_MIN;
    for (int b = threadIdx.x; b < nblk; b += blockDim.x) {
      float f[32];
      const uint4* src = reinterpret_cast<const uint4*>(w + r * cols + b * 32);
#pragma unroll
      for (int q = 0; q < 32 / VN; ++q) Vec16<TW>::unpack(ld_nc_v4(src + q), f + q * VN);
      float amax = 0.f;
#pragma unroll
      for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(f[i]));
      int X = 0;
      if (amax > 0.f) {
        int ex;
        (void)frexpf(amax, &ex);  // amax = m 2^ex, m in [0.5, 1): floor(log2 amax) = ex - 1
        X = ex - 3;
        xmax = max(xmax, X);
      }
      uint32_t packed[4] = {0u, 0u, 0u, 0u};
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const uint32_t byte = __nv_cvt_float2_to_fp4x2(
            make_float2(ldexpf(f[2 * j], -X), ldexpf(f[2 * j + 1], -X)), __NV_E2M1,
            cudaRoundNearest);
        packed[j >> 2] |= (byte & 0xFFu) << (8 * (j & 3));
      }
      *reinterpret_cast<uint4*>(codes + r * (cols / 2) + b * 16) =
          make_uint4(packed[0], packed[1], packed[2], packed[3]);
      bscales[r * nblk + b] = static_cast<uint8_t>(X + 127);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) xmax = max(xmax, __shfl_xor_sync(0xffffffffu, xmax, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = xmax;
    __syncthreads();
    if (threadIdx.x == 0) {
      int m = INT_MIN;
#pragma unroll
      for (int i = 0; i < 8; ++i) m = max(m, red[i]);
      row_factor[r] = m == INT_MIN ? 1.0f : ldexpf(1.0f, m);
    }
    __syncthreads();
  }
}

// out[r][c] = the weight an MXFP4 layer computes with, code * 2^X of its block,
// built by the routine the GEMM converters use (fp16 code * 2^(X - X_row), then
// the row factor 2^X_row in fp32). One thread per 16 codes.
__global__ void __launch_bounds__(256) dequantize_rows_mxfp4_kernel(
    const uint8_t* __restrict__ codes, const uint8_t* __restrict__ bscales,
    const float* __restrict__ row_factor, int64_t rows, int cols, float* __restrict__ out) {
  const int64_t vec_per_row = cols / 16;
  const int64_t n = rows * vec_per_row;
  const int nblk = cols / 32;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / vec_per_row;
    const int j = (int)(i - r * vec_per_row);
    const float rf = row_factor[r];
    const uint2 c = __ldg(reinterpret_cast<const uint2*>(codes + r * (cols / 2) + j * 8));
    uint32_t o[8];
    mxfp4x16_to_f16x16(c, mx_block_multiplier(bscales[r * nblk + j / 2], 1.0f / rf), o);
    float4* dst = reinterpret_cast<float4*>(out + r * cols + j * 16);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&o[2 * q]));
      const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&o[2 * q + 1]));
      dst[q] = make_float4(a.x * rf, a.y * rf, b.x * rf, b.y * rf);
    }
  }
}

}  // namespace tcf8
}  // namespace moe
