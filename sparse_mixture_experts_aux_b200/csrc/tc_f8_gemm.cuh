// Grouped expert GEMMs with quantised expert weights, dequantised on chip:
// FP8 (E4M3 codes, one fp32 scale per output row) or MXFP4 (E2M1 codes packed
// two per byte, one power-of-two E8M0 scale per 32 weights along K, and a
// per-row fp32 factor 2^(the row's largest block exponent)).
//
// The weights stay in HBM as codes, so a weight-streaming (decode) pass reads
// half (FP8) or about a quarter (MXFP4: 4.25 bits per weight) of the bytes of
// bf16 weights. MXFP4 codes decode to fp16 exactly with one instruction per
// pair; each is then multiplied in fp16 by 2^(X_block - X_row), a power of two,
// which is exact while X_block >= X_row - 23, and the row factor 2^X_row
// multiplies the fp32 accumulator in the epilogue like the FP8 row scale.
// The MMAs run kind::f16 with fp16 operands: E4M3 codes convert to fp16 exactly
// with one instruction per pair, the permuted activations arrive as fp16 (the
// scatter kernel converts them; exact for 2^-14 <= |x| <= 65504, saturating
// above), and this kernel stores H as fp16. Three shared-memory rings:
//   Q  weight code tiles, 256 rows x 128 bytes (FP8: 128 codes, two 64-deep K
//      chunks; MXFP4: 256 codes, four chunks), full 128-byte lines, 128-byte
//      swizzle; TMA in, released by the converter warps once decoded, so the
//      weight stream never waits for the MMAs
//   A  stages of CH fp16 activation boxes (TMA), released by the MMA commit;
//      deeper than S, so the boxes (L2 hits) are fetched well ahead
//   S  stages of CH decoded fp16 weight tiles (256 x 64 each, the
//      128-byte-swizzled K-major layout the MMA reads, written by 8 converter
//      warps); released by the MMA commit
// The MMA thread waits once and commits once per stage. Every barrier
// operation of one thread is a serial step of roughly a hundred cycles, so
// per 64-deep chunk it matters how many each role issues: with two chunks per
// stage the MMA thread spends 1 wait + 8 MMAs + 1 commit per 128-deep step.
// The epilogue multiplies by the per-row weight scale, then applies SwiGLU or
// the gate scale as the bf16 kernel does.
// Sources: AI Engineering Illustrated "Mixture of Experts", "Trade-offs to
// weigh" (small-batch MoE inference is limited by reading weights; quantising
// the expert weights attacks that directly); jacopoparretti "Mixture of
// experts, token by token", "Memory" (DeepSeek-V3 ships FP8 weights).
//
// Synchronisation (all waits bounded, as in the bf16 kernel):
//   qfull[q]  Q producer expect_tx + TMA bytes;   qempty[q] 8 converter-warp arrivals
//   afull[a]  A producer expect_tx + TMA bytes (waited by the first converter
//             warp);                                 aempty[a] 1 MMA commit
//   full[s]   8 converter-warp arrivals (the first one after afull[a]): activations
//             landed and weights decoded;          empty[s]  1 MMA commit
//   tfull/tempty/done as in the bf16 kernel.
#pragma once
#include "tc_gemm.cuh"
#include <cuda_fp4.h>
#include <cuda_fp8.h>
#include <limits.h>

namespace moe {
namespace tcf8 {

using tc::BK;
using tc::BM;
using tc::BN;
using tc::UMMA_K;
using tc::TcMaps;

constexpr int CONV_WARPS = 8;
// warp 0 activation producer, 1 MMA, 2-5 epilogue, 6-13 converters, 14 weight producer
constexpr int NUM_THREADS = (7 + CONV_WARPS) * 32;
constexpr int QPROD_WARP = 6 + CONV_WARPS;
constexpr uint32_t TMEM_COLS = 512;
constexpr int BAR_BYTES = 256;
constexpr int CONV_WARP0 = 6;

enum { WQ_FP8 = 0, WQ_MXFP4 = 1 };

// Ring shape for an activation box of AR rows and weight format WQ. For small
// boxes (weight-streaming shapes) a stage is two 64-deep chunks: each stage
// hand-off between converters and the MMA thread costs a roughly fixed
// latency, so fewer, larger stages stream faster (measured: one chunk per stage
// with a four-deep code ring took about 2000 cycles per chunk, two chunks per
// stage about 1400). For 128-row boxes a stage is one chunk.
template <int AR, int WQ = WQ_FP8>
struct F8Shape {
  static_assert(AR == 128 || AR == 64 || AR == 32, "activation box rows");
  static constexpr int CH = AR == 128 ? 1 : 2;       // 64-deep K chunks per stage
  static constexpr int A_SUB = AR * BK * 2;          // fp16 activation box of one chunk
  static constexpr int B_SUB = BN * BK * 2;          // decoded fp16 weights of one chunk
  static constexpr int A_BYTES = CH * A_SUB;         // a stage of ring A
  static constexpr int S_BYTES = CH * B_SUB;         // a stage of ring S (weights)
  static constexpr int Q_ROW = 128;                  // bytes per weight row in a Q stage
  static constexpr int QK = WQ == WQ_MXFP4 ? 256 : 128;  // codes per weight row in a Q stage
  static constexpr int QCH = QK / BK;                // 64-deep chunks per Q stage
  static constexpr int Q_BYTES = BN * Q_ROW;         // 256 rows x 128 B
  static constexpr int NS = AR == 128 ? 3 : 2;
  static constexpr int NA = AR == 64 ? 2 : 4;        // activations run ahead of the weights
  static constexpr int NQ = 2;
  static constexpr int RING_BYTES = NS * S_BYTES + NA * A_BYTES + NQ * Q_BYTES;
  static constexpr int SMEM_BYTES = 1024 + RING_BYTES + BAR_BYTES;
  static_assert(SMEM_BYTES <= 232448, "shared memory per block");
  // the M = 128 MMA reads 16 KB from an A chunk; ring Q follows ring A, so the
  // rows beyond AR stay inside this CTA's shared memory
  static_assert(NA * A_BYTES - A_SUB + NQ * Q_BYTES >= BM * BK * 2, "activation reads in bounds");
  static_assert(A_SUB % 1024 == 0 && S_BYTES % 1024 == 0 && Q_BYTES % 1024 == 0,
                "1024-byte aligned slots");
};

struct F8Group {
  tc::TcGroup g;           // rows, tiles, output, gate scale (row_scale) as in the bf16 kernel
  const float* scale0;     // per output row of the weight: gate (SwiGLU) or down scales
  const float* scale1;     // up scales (SwiGLU)
  int64_t scale_stride;    // floats between experts
  // MXFP4 only: E8M0 block exponents (biased by 127), [rows][K / 32] per expert
  const uint8_t* bscale0;  // gate (SwiGLU) or down
  const uint8_t* bscale1;  // up (SwiGLU)
  int64_t bscale_stride;   // bytes between experts
  int kblk;                // bytes per weight row (K / 32)
};

struct F8Params {
  F8Group grp;
  unsigned long long timeout_ns;
  unsigned long long drain_timeout_ns;
  int* call_err;  // the call's own status word (NULL: none)
};

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
// two when the row factor is one (2^X_row), exact in fp16 down to 2^-24.
__device__ __forceinline__ uint32_t mx_block_multiplier(uint32_t e8m0, float inv_row_factor) {
  const float m = ldexpf(inv_row_factor, (int)e8m0 - 127);
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

// fp32 pair -> f16x2, saturating at +-65504 (H of the FP8-weight path).
__device__ __forceinline__ uint32_t f16x2_sat(float a, float b) {
  const __half2 h = __floats2half2_rn(fminf(fmaxf(a, -65504.f), 65504.f),
                                      fminf(fmaxf(b, -65504.f), 65504.f));
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Instruction descriptor, kind::f16 with A and B fp16 (format 0), D fp32.
__host__ __device__ constexpr uint32_t make_idesc_f16(int M, int N) {
  return (1u << 4) | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
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


template <int EPI, int AR, int WQ = WQ_FP8>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    tc_f8_grouped_gemm_kernel(const __grid_constant__ TcMaps maps, const F8Params p) {
  using Sh = F8Shape<AR, WQ>;
  constexpr int NS = Sh::NS, NA = Sh::NA, NQ = Sh::NQ, CH = Sh::CH;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = tc::smem_addr(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* s_base = smem;                                   // ring S: NS decoded weight stages
  uint8_t* a_base = s_base + NS * Sh::S_BYTES;              // ring A: NA activation stages
  uint8_t* q_base = a_base + NA * Sh::A_BYTES;              // ring Q: NQ x 32 KB FP8 tiles
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Sh::RING_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * NS + 2 * NA + 2 * NQ + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  // segment starts: read from global memory (L1-cached) by the few threads that
  // walk tiles, which leaves all of shared memory to the rings
  const int32_t* s_ts = p.grp.g.tile_start;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t s_0 = tc::smem_addr(s_base);
  const uint32_t a_0 = tc::smem_addr(a_base);
  const uint32_t q_0 = tc::smem_addr(q_base);
  const uint32_t bar0 = tc::smem_addr(bars);
  auto full = [&](int i) { return bar0 + 8u * i; };
  auto empty = [&](int i) { return bar0 + 8u * (NS + i); };
  auto afull = [&](int i) { return bar0 + 8u * (2 * NS + i); };
  auto aempty = [&](int i) { return bar0 + 8u * (2 * NS + NA + i); };
  auto qfull = [&](int i) { return bar0 + 8u * (2 * NS + 2 * NA + i); };
  auto qempty = [&](int i) { return bar0 + 8u * (2 * NS + 2 * NA + NQ + i); };
  constexpr int T0 = 2 * NS + 2 * NA + 2 * NQ;
  auto tfull = [&](int a) { return bar0 + 8u * (T0 + a); };
  auto tempty = [&](int a) { return bar0 + 8u * (T0 + 2 + a); };
  const uint32_t done_bar = bar0 + 8u * (T0 + 4);

  const tc::TcGroup& G = p.grp.g;
  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      tc::mbar_init(full(i), CONV_WARPS);
      tc::mbar_init(empty(i), 1);
    }
    for (int i = 0; i < NA; ++i) {
      tc::mbar_init(afull(i), 1);
      tc::mbar_init(aempty(i), 1);
    }
    for (int i = 0; i < NQ; ++i) {
      tc::mbar_init(qfull(i), 1);
      tc::mbar_init(qempty(i), CONV_WARPS);
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
  pdl_wait();  // the routing results and rows this GEMM reads are complete
  pdl_launch_dependents();
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const long long total = (long long)G.n_tiles * s_ts[G.E];
  const int nck = G.k_blocks;                 // 64-deep K chunks per tile
  const int nst = (nck + CH - 1) / CH;        // S stages per tile
  const int nqs = (nck + Sh::QCH - 1) / Sh::QCH;  // Q stages per tile
  const unsigned long long tmo = p.timeout_ns, drain_tmo = p.drain_timeout_ns;

  if (warp == 0) {
    // ------------------------------------------------------ activation producer
    if (lane == 0) {
      tc::prefetch_map(&maps.a[0]);
      int as = 0;
      uint32_t aph = 0, issued = 0, par = 0;
      bool ok = true;
      for (long long tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
        const tc::TileInfo ti = decode_tile_f8(tile, G, s_ts);
        if (tc::tile_out_of_bounds(ti.e, ti.nb, ti.row0, BM, G)) {
          flag_bounds();
          continue;
        }
        for (int st = 0; st < nst; ++st) {
          if (!tc::wait_fast(aempty(as), aph ^ 1u, abort_flag, tmo)) { ok = false; break; }
          const int nv = min(CH, nck - st * CH);
          tc::mbar_expect_tx(afull(as), nv * Sh::A_SUB);
          for (int c = 0; c < nv; ++c)
            tc::tma_load_2d(a_0 + as * Sh::A_BYTES + c * Sh::A_SUB, &maps.a[0], afull(as),
                            (st * CH + c) * BK, ti.row0);
          issued |= 1u << as;
          par = (par & ~(1u << as)) | (aph << as);
          if (++as == NA) { as = 0; aph ^= 1u; }
        }
      }
      if (!ok)  // let every copy already issued land before the CTA exits
        for (int i = 0; i < NA; ++i)
          if ((issued >> i) & 1u) tc::wait_drain(afull(i), (par >> i) & 1u, abort_flag, drain_tmo);
    }
  } else if (warp == QPROD_WARP) {
    // ---------------------------------------------------------- weight producer
    if (lane == 0) {
      tc::prefetch_map(&maps.b0[0]);
      if (EPI == tc::EPI_SWIGLU_TC) tc::prefetch_map(&maps.b1[0]);
      int qs = 0;
      uint32_t qph = 0, issued = 0, par = 0;
      bool ok = true;
      for (long long tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
        const tc::TileInfo ti = decode_tile_f8(tile, G, s_ts);
        if (tc::tile_out_of_bounds(ti.e, ti.nb, ti.row0, BM, G)) continue;
        for (int qi = 0; qi < nqs; ++qi) {
          if (!tc::wait_fast(qempty(qs), qph ^ 1u, abort_flag, tmo)) { ok = false; break; }
          const uint32_t dq = q_0 + qs * Sh::Q_BYTES;
          const int x = qi * (Sh::Q_ROW / 4);  // the codes are described as 32-bit words
          tc::mbar_expect_tx(qfull(qs), Sh::Q_BYTES);
          if (EPI == tc::EPI_SWIGLU_TC) {
            tc::tma_load_3d(dq, &maps.b0[0], qfull(qs), x, ti.nb * (BN / 2), ti.e);
            tc::tma_load_3d(dq + Sh::Q_BYTES / 2, &maps.b1[0], qfull(qs), x, ti.nb * (BN / 2),
                            ti.e);
          } else {
            tc::tma_load_3d(dq, &maps.b0[0], qfull(qs), x, ti.nb * BN, ti.e);
          }
          issued |= 1u << qs;
          par = (par & ~(1u << qs)) | (qph << qs);
          if (++qs == NQ) { qs = 0; qph ^= 1u; }
        }
      }
      if (!ok)
        for (int i = 0; i < NQ; ++i)
          if ((issued >> i) & 1u) tc::wait_drain(qfull(i), (par >> i) & 1u, abort_flag, drain_tmo);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC = make_idesc_f16(BM, BN);
      int ss = 0, as = 0;
      uint32_t sph = 0, aph = 0, acc = 0, acc_phase = 0;
      bool ok = true;
      for (long long tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
#if defined(MOE_DEBUG)
        const tc::TileInfo ti = decode_tile_f8(tile, G, s_ts);
        if (tc::tile_out_of_bounds(ti.e, ti.nb, ti.row0, BM, G)) continue;
#endif
        if (!tc::wait_bounded(tempty(acc), acc_phase ^ 1u, abort_flag, tmo)) { ok = false; break; }
        tc::tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int st = 0; st < nst; ++st) {
          if (!tc::wait_fast(full(ss), sph, abort_flag, tmo)) { ok = false; break; }
          tc::tc_fence_after();
          const int nv = min(CH, nck - st * CH);
          for (int c = 0; c < nv; ++c) {
            const uint64_t ad = tc::sw128_kmajor_desc(a_0 + as * Sh::A_BYTES + c * Sh::A_SUB);
            const uint64_t bd = tc::sw128_kmajor_desc(s_0 + ss * Sh::S_BYTES + c * Sh::B_SUB);
            const int chunk = st * CH + c;
#pragma unroll
            for (int kk = 0; kk < BK / UMMA_K; ++kk)
              tc::tc_mma(d_tmem, ad + 2u * kk, bd + 2u * kk, IDESC, (chunk | kk) != 0 ? 1u : 0u);
          }
          tc::tc_commit(aempty(as));  // this stage's activations have been read
          tc::tc_commit(empty(ss));   // and its decoded weights
          if (++ss == NS) { ss = 0; sph ^= 1u; }
          if (++as == NA) { as = 0; aph ^= 1u; }
        }
        if (!ok) break;
        tc::tc_commit(tfull(acc));
        acc ^= 1u;
        if (acc == 0u) acc_phase ^= 1u;
      }
      tc::tc_commit(done_bar);
      tc::wait_drain(done_bar, 0u, abort_flag, drain_tmo);
    }
  } else if (warp >= CONV_WARP0 && warp < CONV_WARP0 + CONV_WARPS) {
    // ---------------------------------------------------------------- converters
    // For chunk g, 256 threads turn part h = g % QCH of the Q tile into the
    // fp16 tile (the 128-byte rows are stored with 16-byte chunk j at
    // j ^ (row & 7)). FP8: 16 codes (16-byte chunk 4h + c4) -> two 16-byte
    // chunks at (2c, 2c+1) ^ (row & 7). MXFP4: 16 codes (the 8-byte half
    // c4 & 1 of 16-byte chunk 2h + c4/2, one 32-weight block shared by two
    // threads) -> the same two chunks. A thread owns rows r, r+64, r+128, r+192
    // with r & 7 = its lane & 7, so the 8 lanes of every shared-memory phase
    // hit 8 different 16-byte bank groups, both when reading and when writing.
    const int ct = threadIdx.x - CONV_WARP0 * 32;
    const int r_lo = ct & 7, c4 = (ct >> 3) & 3, r_hi = ct >> 5;
    const int row0 = r_hi * 8 + r_lo;  // 0..63
    const int pos0 = ((2 * c4) ^ r_lo) << 4, pos1 = ((2 * c4 + 1) ^ r_lo) << 4;
    const uint32_t q_row = row0 * Sh::Q_ROW;
    const uint32_t b_row = r_hi * 1024 + r_lo * 128;
    const bool first = warp == CONV_WARP0;
    int ss = 0, qs = 0, as = 0;
    uint32_t sph = 0, qph = 0, aph = 0;
    bool ok = true;
    // MXFP4: per owned row, its block exponents (this Q stage's eight, and the
    // next stage's, loaded one stage ahead) and 1 / its row factor
    const uint8_t* bsrow[4] = {nullptr, nullptr, nullptr, nullptr};
    float inv_rf[4] = {0.f, 0.f, 0.f, 0.f};
    uint2 bs_cur[4], bs_nxt[4];
    auto load_bs = [&](int qi) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        bs_nxt[i] = bsrow[i] != nullptr
                        ? __ldg(reinterpret_cast<const uint2*>(bsrow[i] + (size_t)qi * 8))
                        : make_uint2(0u, 0u);
    };
    for (long long tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
#if defined(MOE_DEBUG)
      {
        const tc::TileInfo td = decode_tile_f8(tile, G, s_ts);
        if (tc::tile_out_of_bounds(td.e, td.nb, td.row0, BM, G)) continue;
      }
#endif
      if constexpr (WQ == WQ_MXFP4) {
        const tc::TileInfo ti = decode_tile_f8(tile, G, s_ts);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int rr = row0 + 64 * i;  // row of the 256-row weight tile
          const bool up = EPI == tc::EPI_SWIGLU_TC && rr >= BN / 2;
          const int grow = EPI == tc::EPI_SWIGLU_TC ? ti.nb * (BN / 2) + (rr & (BN / 2 - 1))
                                                    : ti.nb * BN + rr;
          const bool valid = grow < G.N;  // rows past N are zero-filled by TMA
          const uint8_t* bs = up ? p.grp.bscale1 : p.grp.bscale0;
          const float* rf = up ? p.grp.scale1 : p.grp.scale0;
          bsrow[i] = valid ? bs + (int64_t)ti.e * p.grp.bscale_stride + (int64_t)grow * p.grp.kblk
                           : nullptr;
          inv_rf[i] = valid ? 1.0f / __ldg(rf + (int64_t)ti.e * p.grp.scale_stride + grow) : 0.f;
        }
        load_bs(0);
      }
      for (int st = 0; st < nst; ++st) {
        // lane 0 waits (bounded) for the stage's slot to be free; __syncwarp
        // then orders the other lanes' writes after it
        int w = 1;
        if (lane == 0) w = tc::wait_fast(empty(ss), sph ^ 1u, abort_flag, tmo) ? 1 : 0;
        if (!__shfl_sync(0xffffffffu, w, 0)) { ok = false; break; }
        const int nv = min(CH, nck - st * CH);
        uint8_t* const bst = s_base + ss * Sh::S_BYTES + b_row;
        // all of this stage's codes are loaded before any is decoded
        uint4 v[CH][4];    // FP8: 16 codes per owned row
        uint2 v4[CH][4];   // MXFP4: 16 codes per owned row
        uint32_t mult[CH][4];
        for (int c = 0; c < nv; ++c) {
          const int g = st * CH + c, h = g % Sh::QCH;
          if (h == 0) {
            // lane 0 waits for the Q tile; the others then observe the completed
            // phase themselves (it cannot move on before this warp releases it),
            // which gives each lane its own acquire for the TMA-written bytes
            w = 1;
            if (lane == 0) w = tc::wait_fast(qfull(qs), qph, abort_flag, tmo) ? 1 : 0;
            if (!__shfl_sync(0xffffffffu, w, 0)) { ok = false; break; }
            (void)tc::mbar_try_wait(qfull(qs), qph);
            if constexpr (WQ == WQ_MXFP4) {
#pragma unroll
              for (int i = 0; i < 4; ++i) bs_cur[i] = bs_nxt[i];
              if (g / Sh::QCH + 1 < nqs) load_bs(g / Sh::QCH + 1);
            }
          }
          const uint8_t* qt = q_base + qs * Sh::Q_BYTES + q_row;
          if constexpr (WQ == WQ_MXFP4) {
            const uint8_t* q = qt + (((2 * h + (c4 >> 1)) ^ r_lo) << 4) + (c4 & 1) * 8;
            const int blk = 2 * h + (c4 >> 1);  // block of this Q stage's row
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              v4[c][i] = *reinterpret_cast<const uint2*>(q + i * 64 * Sh::Q_ROW);
              const uint32_t wbs = blk < 4 ? bs_cur[i].x : bs_cur[i].y;
              mult[c][i] = mx_block_multiplier((wbs >> (8 * (blk & 3))) & 0xFFu, inv_rf[i]);
            }
          } else {
            const uint8_t* q = qt + (((4 * h + c4) ^ r_lo) << 4);
#pragma unroll
            for (int i = 0; i < 4; ++i) v[c][i] = *reinterpret_cast<const uint4*>(q + i * 64 * Sh::Q_ROW);
          }
          if (h == Sh::QCH - 1 || g == nck - 1) {  // this Q tile is fully read: hand it back
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(qempty(qs));
            if (++qs == NQ) { qs = 0; qph ^= 1u; }
          }
        }
        if (!ok) break;
#pragma unroll
        for (int c = 0; c < CH; ++c) {
          if (c >= nv) break;
          uint8_t* b16 = bst + c * Sh::B_SUB;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint32_t o[8];
            if constexpr (WQ == WQ_MXFP4) {
              mxfp4x16_to_f16x16(v4[c][i], mult[c][i], o);
            } else {
              e4m3x4_to_f16x4(v[c][i].x, o[0], o[1]);
              e4m3x4_to_f16x4(v[c][i].y, o[2], o[3]);
              e4m3x4_to_f16x4(v[c][i].z, o[4], o[5]);
              e4m3x4_to_f16x4(v[c][i].w, o[6], o[7]);
            }
            uint8_t* rowp = b16 + i * 8 * 1024;  // rows + 64 i
            *reinterpret_cast<uint4*>(rowp + pos0) = make_uint4(o[0], o[1], o[2], o[3]);
            *reinterpret_cast<uint4*>(rowp + pos1) = make_uint4(o[4], o[5], o[6], o[7]);
          }
        }
        fence_async_shared();  // generic-proxy writes -> visible to the tensor cores
        __syncwarp();
        if (lane == 0) {
          // the first converter warp also vouches for the activation boxes
          if (first && !tc::wait_bounded(afull(as), aph, abort_flag, tmo)) ok = false;
          tc::mbar_arrive(full(ss));
        }
        if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) { ok = false; break; }
        if (++ss == NS) { ss = 0; sph ^= 1u; }
        if (++as == NA) { as = 0; aph ^= 1u; }
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int quad = warp & 3;
    const int r_in_tile = quad * 32 + lane;
    uint32_t acc = 0, acc_phase = 0;
    for (long long tile = blockIdx.x; tile < total; tile += gridDim.x) {
      const tc::TileInfo ti = decode_tile_f8(tile, G, s_ts);
      if (tc::tile_out_of_bounds(ti.e, ti.nb, ti.row0, BM, G)) continue;
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
                // H feeds the f16 x f16 down GEMM: stored as fp16
                st_v4(out + col0 + qq * 8, make_uint4(f16x2_sat(h[0], h[1]), f16x2_sat(h[2], h[3]),
                                                      f16x2_sat(h[4], h[5]), f16x2_sat(h[6], h[7])));
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
  tc::record_call_status(abort_flag, p.call_err);
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
