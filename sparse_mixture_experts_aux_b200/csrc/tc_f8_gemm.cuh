// Grouped expert GEMMs with FP8 (E4M3) expert weights, dequantised on chip.
//
// The weights stay in HBM as E4M3 codes with one fp32 scale per output row,
// so a weight-streaming (decode) pass reads half the bytes of bf16 weights.
// The activations stay bf16, and the tensor cores run kind::f16 exactly as in
// the bf16 kernel. Three shared-memory rings:
//   A  bf16 activation boxes (AR rows x 64), one per 64-deep K step; TMA in,
//      released by the MMA's commit
//   Q  FP8 weight tiles, 256 rows x 128 codes (two K steps, full 128-byte
//      lines, 128-byte swizzle); TMA in, released by the converter warps as
//      soon as they have turned both halves into bf16, so the weight stream
//      never waits for the tensor cores
//   B  bf16 weight tiles (256 x 64, the 128-byte-swizzled K-major layout the
//      MMA reads); written by 8 converter warps, released by the MMA's commit
// The MMA (one thread) reads A and B, accumulates fp32 in TMEM; the epilogue
// multiplies by the per-row weight scale, then applies SwiGLU or the gate
// scale as the bf16 kernel does.
// Sources: AI Engineering Illustrated "Mixture of Experts", "Trade-offs to
// weigh" (small-batch MoE inference is limited by reading weights; quantising
// the expert weights attacks that directly); jacopoparretti "Mixture of
// experts, token by token", "Memory" (DeepSeek-V3 ships FP8 weights).
//
// Synchronisation (all waits bounded, as in the bf16 kernel):
//   afull[a] producer expect_tx + TMA bytes;   aempty[a] 1 MMA commit
//   qfull[q] producer expect_tx + TMA bytes;   qempty[q] 8 converter-warp arrivals
//   bfull[b] 8 converter-warp arrivals;        bempty[b] 1 MMA commit
//   tfull/tempty/done as in the bf16 kernel.
#pragma once
#include "tc_gemm.cuh"
#include <cuda_fp8.h>

namespace moe {
namespace tcf8 {

using tc::BK;
using tc::BM;
using tc::BN;
using tc::UMMA_K;
using tc::TcMaps;

constexpr int CONV_WARPS = 8;
// warp 0 producer, 1 MMA, 2-5 epilogue, 6-13 converters
constexpr int NUM_THREADS = (6 + CONV_WARPS) * 32;
constexpr uint32_t TMEM_COLS = 512;
constexpr int BAR_BYTES = 256;
constexpr int CONV_WARP0 = 6;

template <int AR>
struct F8Shape {
  static_assert(AR == 128 || AR == 64 || AR == 32, "activation box rows");
  static constexpr int A_BYTES = AR * BK * 2;        // bf16 activation box
  static constexpr int QK = 2 * BK;                  // codes per weight row in a Q stage
  static constexpr int Q_BYTES = BN * QK;            // FP8 weight tile: 256 rows x 128 B
  static constexpr int B16_BYTES = BN * BK * 2;      // converted bf16 weight tile
  // a Q stage feeds two K steps, so the activation ring holds two boxes per Q stage
  static constexpr int NQ = AR == 128 ? 2 : 3;
  static constexpr int NA = 2 * NQ;
  static constexpr int NB = AR == 32 ? 3 : 2;
  static constexpr int RING_BYTES = NA * A_BYTES + NQ * Q_BYTES + NB * B16_BYTES;
  static constexpr int SMEM_BYTES = 1024 + RING_BYTES + BAR_BYTES + 4 * (tc::MAX_E + 1);
  static_assert(SMEM_BYTES <= 232448, "shared memory per block");
  // the M = 128 MMA reads 16 KB from an activation slot; the Q ring follows the
  // A ring, so the rows beyond AR stay inside this CTA's shared memory
  static_assert(NA * A_BYTES + NQ * Q_BYTES >= (NA - 1) * A_BYTES + BM * BK * 2,
                "activation reads stay inside shared memory");
  static_assert(A_BYTES % 1024 == 0 && Q_BYTES % 1024 == 0, "1024-byte aligned slots");
};

struct F8Group {
  tc::TcGroup g;           // rows, tiles, output, gate scale (row_scale) as in the bf16 kernel
  const float* scale0;     // per output row of the weight: gate (SwiGLU) or down scales
  const float* scale1;     // up scales (SwiGLU)
  int64_t scale_stride;    // floats between experts
};

struct F8Params {
  F8Group grp;
  unsigned long long timeout_ns;
  unsigned long long drain_timeout_ns;
};

// Four E4M3 codes (code i in byte i of `w`) -> four bf16 values, as two bf16x2
// words (codes 0,1 and codes 2,3). Exact for every finite code, with integer
// operations and one bf16x2 FMA per pair instead of format conversions:
// the code's sign goes to bf16 bit 15 and its 7 magnitude bits to bits 10..4.
// Read as bf16, that is the E4M3 value times 2^-120: the 4-bit exponent field
// sits in the low bits of bf16's 8-bit field (bias 127 instead of 7) and the
// 3 mantissa bits lead bf16's 7; exponent field 0 (the E4M3 subnormals) lands
// on bf16 subnormals with the same factor. Multiplying by 2^120 (an FMA with a
// -0 addend, which keeps the sign of zero) restores the value without rounding.
// Codes 0x7F / 0xFF (E4M3 NaN) are never written by the quantiser; they would
// read as +-480.
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, 0, %2;" : "=r"(r) : "r"(a), "r"(sel));
  return r;
}
__device__ __forceinline__ uint32_t bf16x2_scale(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(0x80008000u));
  return r;
}
__device__ __forceinline__ void e4m3x4_to_bf16x4(uint32_t w, uint32_t& lo, uint32_t& hi) {
  constexpr uint32_t MASK = 0x87F087F0u;       // bf16 sign and bits 10..4, both halves
  constexpr uint32_t POW2_120 = 0x7B807B80u;   // bf16x2 (2^120, 2^120)
  // bytes sign-extended to 16-bit halves (prmt selector nibble 8|i: sign of byte i)
  const uint32_t t01 = prmt(w, 0x9180u), t23 = prmt(w, 0xB3A2u);
  lo = bf16x2_scale((t01 << 4) & MASK, POW2_120);
  hi = bf16x2_scale((t23 << 4) & MASK, POW2_120);
}

__device__ __forceinline__ void fence_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Tile walk: one group of routed experts, the same order as the bf16 kernel.
__device__ __forceinline__ tc::TileInfo decode_tile_f8(long long tile, const tc::TcGroup& g,
                                                      const int32_t* s_ts) {
  tc::TileInfo ti;
  ti.g = 0;
  const long long q = tile / g.n_tiles;
  int lo = 0, hi = g.E - 1;  // last expert whose first tile is at or before q
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s_ts[mid] <= q) lo = mid; else hi = mid - 1;
  }
  const int me = s_ts[lo + 1] - s_ts[lo];
  const long long in_e = tile - (long long)g.n_tiles * s_ts[lo];
  ti.e = lo;
  ti.nb = (int)(in_e / me);
  ti.row0 = (s_ts[lo] + (int)(in_e % me)) * BM;
  return ti;
}


template <int EPI, int AR>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    tc_f8_grouped_gemm_kernel(const __grid_constant__ TcMaps maps, const F8Params p) {
  using Sh = F8Shape<AR>;
  constexpr int NA = Sh::NA, NQ = Sh::NQ, NB = Sh::NB;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = tc::smem_addr(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* a_base = smem;                                   // ring A: NA activation boxes
  uint8_t* q_base = a_base + NA * Sh::A_BYTES;              // ring Q: NQ x 32 KB FP8 tiles
  uint8_t* b_base = q_base + NQ * Sh::Q_BYTES;              // ring B: NB x 32 KB bf16 tiles
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Sh::RING_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * (NA + NQ + NB) + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int32_t* s_ts = reinterpret_cast<int32_t*>(smem + Sh::RING_BYTES + BAR_BYTES);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t a_0 = tc::smem_addr(a_base);
  const uint32_t q_0 = tc::smem_addr(q_base);
  const uint32_t b_0 = tc::smem_addr(b_base);
  const uint32_t bar0 = tc::smem_addr(bars);
  auto afull = [&](int i) { return bar0 + 8u * i; };
  auto aempty = [&](int i) { return bar0 + 8u * (NA + i); };
  auto qfull = [&](int i) { return bar0 + 8u * (2 * NA + i); };
  auto qempty = [&](int i) { return bar0 + 8u * (2 * NA + NQ + i); };
  auto bfull = [&](int i) { return bar0 + 8u * (2 * NA + 2 * NQ + i); };
  auto bempty = [&](int i) { return bar0 + 8u * (2 * NA + 2 * NQ + NB + i); };
  constexpr int T0 = 2 * (NA + NQ + NB);
  auto tfull = [&](int a) { return bar0 + 8u * (T0 + a); };
  auto tempty = [&](int a) { return bar0 + 8u * (T0 + 2 + a); };
  const uint32_t done_bar = bar0 + 8u * (T0 + 4);

  const tc::TcGroup& G = p.grp.g;
  for (int i = threadIdx.x; i <= G.E; i += NUM_THREADS) s_ts[i] = G.tile_start[i];
  if (threadIdx.x == 0) {
    for (int i = 0; i < NA; ++i) {
      tc::mbar_init(afull(i), 1);
      tc::mbar_init(aempty(i), 1);
    }
    for (int i = 0; i < NQ; ++i) {
      tc::mbar_init(qfull(i), 1);
      tc::mbar_init(qempty(i), CONV_WARPS);
    }
    for (int i = 0; i < NB; ++i) {
      tc::mbar_init(bfull(i), CONV_WARPS);
      tc::mbar_init(bempty(i), 1);
    }
    for (int a = 0; a < 2; ++a) {
      tc::mbar_init(tfull(a), 1);
      tc::mbar_init(tempty(a), 4);
    }
    tc::mbar_init(done_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    tc::tmem_alloc(tc::smem_addr(tmem_slot), TMEM_COLS);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const long long total = (long long)G.n_tiles * s_ts[G.E];
  const int kbs = G.k_blocks;
  const unsigned long long tmo = p.timeout_ns, drain_tmo = p.drain_timeout_ns;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    // In issue order: the Q tile of K steps kb and kb + 1, then the two
    // activation boxes of those steps. A TMA unit serves its copies roughly in
    // order, so a box issued far behind a deep queue of weight tiles would
    // arrive late; issued right behind its own tile, it lands with it.
    if (lane == 0) {
      tc::prefetch_map(&maps.a[0]);
      tc::prefetch_map(&maps.b0[0]);
      if (EPI == tc::EPI_SWIGLU_TC) tc::prefetch_map(&maps.b1[0]);
      int as = 0, qs = 0;
      uint32_t aph = 0, qph = 0, a_issued = 0, a_par = 0, q_issued = 0, q_par = 0;
      bool ok = true;
      for (long long tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
        const tc::TileInfo ti = decode_tile_f8(tile, G, s_ts);
        for (int kb = 0; ok && kb < kbs; ++kb) {
          if ((kb & 1) == 0) {
            if (!tc::wait_bounded(qempty(qs), qph ^ 1u, abort_flag, tmo)) { ok = false; break; }
            const uint32_t dq = q_0 + qs * Sh::Q_BYTES;
            tc::mbar_expect_tx(qfull(qs), Sh::Q_BYTES);
            if (EPI == tc::EPI_SWIGLU_TC) {
              tc::tma_load_3d(dq, &maps.b0[0], qfull(qs), kb * (BK / 4), ti.nb * (BN / 2), ti.e);
              tc::tma_load_3d(dq + Sh::Q_BYTES / 2, &maps.b1[0], qfull(qs), kb * (BK / 4),
                              ti.nb * (BN / 2), ti.e);
            } else {
              tc::tma_load_3d(dq, &maps.b0[0], qfull(qs), kb * (BK / 4), ti.nb * BN, ti.e);
            }
            q_issued |= 1u << qs;
            q_par = (q_par & ~(1u << qs)) | (qph << qs);
            if (++qs == NQ) { qs = 0; qph ^= 1u; }
          }
          if (!tc::wait_bounded(aempty(as), aph ^ 1u, abort_flag, tmo)) { ok = false; break; }
          tc::mbar_expect_tx(afull(as), Sh::A_BYTES);
          tc::tma_load_2d(a_0 + as * Sh::A_BYTES, &maps.a[0], afull(as), kb * BK, ti.row0);
          a_issued |= 1u << as;
          a_par = (a_par & ~(1u << as)) | (aph << as);
          if (++as == NA) { as = 0; aph ^= 1u; }
        }
      }
      if (!ok) {  // let every copy already issued land before the CTA exits
        for (int i = 0; i < NQ; ++i)
          if ((q_issued >> i) & 1u) tc::wait_drain(qfull(i), (q_par >> i) & 1u, drain_tmo);
        for (int i = 0; i < NA; ++i)
          if ((a_issued >> i) & 1u) tc::wait_drain(afull(i), (a_par >> i) & 1u, drain_tmo);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC = tc::make_idesc(BM, BN);
      int as = 0, bs = 0;
      uint32_t aph = 0, bph = 0, acc = 0, acc_phase = 0;
      bool ok = true;
      for (long long tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
        if (!tc::wait_bounded(tempty(acc), acc_phase ^ 1u, abort_flag, tmo)) { ok = false; break; }
        tc::tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < kbs; ++kb) {
          if (!tc::wait_bounded(afull(as), aph, abort_flag, tmo) ||
              !tc::wait_bounded(bfull(bs), bph, abort_flag, tmo)) {
            ok = false;
            break;
          }
          tc::tc_fence_after();
          const uint64_t ad = tc::sw128_kmajor_desc(a_0 + as * Sh::A_BYTES);
          const uint64_t bd = tc::sw128_kmajor_desc(b_0 + bs * Sh::B16_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / UMMA_K; ++kk)
            tc::tc_mma(d_tmem, ad + 2u * kk, bd + 2u * kk, IDESC, (kb | kk) != 0 ? 1u : 0u);
          tc::tc_commit(aempty(as));  // this activation box has been read
          tc::tc_commit(bempty(bs));  // and these converted weights
          if (++as == NA) { as = 0; aph ^= 1u; }
          if (++bs == NB) { bs = 0; bph ^= 1u; }
        }
        if (!ok) break;
        tc::tc_commit(tfull(acc));
        acc ^= 1u;
        if (acc == 0u) acc_phase ^= 1u;
      }
      tc::tc_commit(done_bar);
      tc::wait_drain(done_bar, 0u, drain_tmo);
    }
  } else if (warp >= CONV_WARP0 && warp < CONV_WARP0 + CONV_WARPS) {
    // ---------------------------------------------------------------- converters
    // For the K step kb, 256 threads turn half (kb & 1) of the Q tile (chunks
    // 4h..4h+3 of each 128-byte row, stored at chunk ^ (row & 7)) into the bf16
    // tile: 16 codes -> two 16-byte chunks at (2c, 2c+1) ^ (row & 7). A thread
    // owns rows r, r+64, r+128, r+192 with r & 7 = its lane & 7, so the 8 lanes
    // of every shared-memory phase hit 8 different 16-byte bank groups, both
    // when reading and when writing.
    const int ct = threadIdx.x - CONV_WARP0 * 32;
    const int r_lo = ct & 7, c4 = (ct >> 3) & 3, r_hi = ct >> 5;
    const int row0 = r_hi * 8 + r_lo;  // 0..63
    const int pos0 = ((2 * c4) ^ r_lo) << 4, pos1 = ((2 * c4 + 1) ^ r_lo) << 4;
    const uint32_t q_row = row0 * Sh::QK;
    const uint32_t b_row = r_hi * 1024 + r_lo * 128;
    int qs = 0, bs = 0;
    uint32_t qph = 0, bph = 0;
    for (long long tile = blockIdx.x; tile < total; tile += gridDim.x) {
      bool ok = true;
      for (int kb = 0; kb < kbs; ++kb) {
        const int h = kb & 1;
        // lane 0 waits (bounded); the others then observe the completed phase
        // themselves (it cannot move on before this warp arrives), which gives
        // each lane its own acquire for the TMA-written tile
        int w = 1;
        if (lane == 0)
          w = ((h != 0 || tc::wait_bounded(qfull(qs), qph, abort_flag, tmo)) &&
               tc::wait_bounded(bempty(bs), bph ^ 1u, abort_flag, tmo))
                  ? 1
                  : 0;
        if (!__shfl_sync(0xffffffffu, w, 0)) { ok = false; break; }
        (void)tc::mbar_try_wait(qfull(qs), qph);
        (void)tc::mbar_try_wait(bempty(bs), bph ^ 1u);
        const uint8_t* q = q_base + qs * Sh::Q_BYTES + q_row + ((((4 * h + c4) ^ r_lo)) << 4);
        uint8_t* b16 = b_base + bs * Sh::B16_BYTES + b_row;
        uint4 v[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = *reinterpret_cast<const uint4*>(q + i * 64 * Sh::QK);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          uint32_t o[8];
          e4m3x4_to_bf16x4(v[i].x, o[0], o[1]);
          e4m3x4_to_bf16x4(v[i].y, o[2], o[3]);
          e4m3x4_to_bf16x4(v[i].z, o[4], o[5]);
          e4m3x4_to_bf16x4(v[i].w, o[6], o[7]);
          uint8_t* rowp = b16 + i * 8 * 1024;  // rows + 64 i
          *reinterpret_cast<uint4*>(rowp + pos0) = make_uint4(o[0], o[1], o[2], o[3]);
          *reinterpret_cast<uint4*>(rowp + pos1) = make_uint4(o[4], o[5], o[6], o[7]);
        }
        fence_async_shared();  // generic-proxy writes -> visible to the tensor cores
        __syncwarp();
        const bool q_done = h == 1 || kb == kbs - 1;
        if (lane == 0) {
          tc::mbar_arrive(bfull(bs));
          if (q_done) tc::mbar_arrive(qempty(qs));
        }
        if (q_done && ++qs == NQ) { qs = 0; qph ^= 1u; }
        if (++bs == NB) { bs = 0; bph ^= 1u; }
      }
      if (!ok) break;
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int quad = warp & 3;
    const int r_in_tile = quad * 32 + lane;
    uint32_t acc = 0, acc_phase = 0;
    for (long long tile = blockIdx.x; tile < total; tile += gridDim.x) {
      const tc::TileInfo ti = decode_tile_f8(tile, G, s_ts);
      int ok = 1;
      if (lane == 0) ok = tc::wait_bounded(tfull(acc), acc_phase, abort_flag, tmo) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc::tc_fence_after();
      const int row = ti.row0 + r_in_tile;
      const uint32_t tb = tmem_base + acc * BN + (static_cast<uint32_t>(quad * 32) << 16);
      __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(G.out) + (size_t)row * G.N;
      const float* sc0 = p.grp.scale0 + (int64_t)ti.e * p.grp.scale_stride;
      const float* sc1 = p.grp.scale1 + (int64_t)ti.e * p.grp.scale_stride;
      if (quad * 32 < AR) {
        if (EPI == tc::EPI_SWIGLU_TC) {
#pragma unroll 1
          for (int c = 0; c < (BN / 2) / 32; ++c) {
            float gv[32], uv[32];
            __syncwarp();
            tc::tmem_ld32(tb + c * 32, gv);
            tc::tmem_ld32(tb + BN / 2 + c * 32, uv);
            const int col0 = ti.nb * (BN / 2) + c * 32;
            if (col0 < G.N) {
#pragma unroll
              for (int qq = 0; qq < 4; ++qq) {
                float h[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                  const int col = col0 + qq * 8 + i;
                  h[i] = silu_f32(gv[qq * 8 + i] * sc0[col]) * (uv[qq * 8 + i] * sc1[col]);
                }
                st_v4(out + col0 + qq * 8, Vec16<__nv_bfloat16>::pack(h));
              }
            }
          }
        } else {
          const float rs = G.row_scale != nullptr ? G.row_scale[row] : 1.f;
#pragma unroll 1
          for (int c = 0; c < BN / 32; ++c) {
            float v[32];
            __syncwarp();
            tc::tmem_ld32(tb + c * 32, v);
            const int col0 = ti.nb * BN + c * 32;
            if (col0 < G.N) {
#pragma unroll
              for (int qq = 0; qq < 4; ++qq) {
                float h[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) h[i] = rs * (v[qq * 8 + i] * sc0[col0 + qq * 8 + i]);
                st_v4(out + col0 + qq * 8, Vec16<__nv_bfloat16>::pack(h));
              }
            }
          }
        }
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(tempty(acc));
      acc ^= 1u;
      if (acc == 0u) acc_phase ^= 1u;
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tc::tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// Per-row E4M3 quantisation of expert weights (run once, outside the forward
// pass): scale = absmax / 448 (1 for an all-zero row), code = E4M3(w / scale)
// with round-to-nearest-even and saturation to +-448.
// ---------------------------------------------------------------------------
template <typename TW>
__global__ void __launch_bounds__(256) quantize_rows_fp8_kernel(const TW* __restrict__ w,
                                                                int64_t rows, int cols,
                                                                uint8_t* __restrict__ codes,
                                                                float* __restrict__ scales) {
  __shared__ float red[8];
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    const TW* wr = w + r * cols;
    float m = 0.f;
    for (int c = threadIdx.x; c < cols; c += blockDim.x) m = fmaxf(m, fabsf(to_f32(wr[c])));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    float absmax = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) absmax = fmaxf(absmax, red[i]);
    const float scale = absmax > 0.f ? absmax / 448.0f : 1.0f;
    for (int c = threadIdx.x; c < cols; c += blockDim.x)
      codes[r * cols + c] = __nv_cvt_float_to_fp8(to_f32(wr[c]) / scale, __NV_SATFINITE, __NV_E4M3);
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
      e4m3x4_to_bf16x4(in[j], lo, hi);
      o[j] = make_float4(__uint_as_float(lo << 16) * s, __uint_as_float(lo & 0xFFFF0000u) * s,
                         __uint_as_float(hi << 16) * s, __uint_as_float(hi & 0xFFFF0000u) * s);
    }
  }
}

}  // namespace tcf8
}  // namespace moe
