// Grouped expert GEMMs with quantised expert weights (FP8 or MXFP4): operands
// swapped, decoded weights in TMEM.
//
// The weights are the MMA's A operand (M = 128 weight rows) and the token rows
// are B (N = 32, 64 or 128, the activation box, chosen by the batch size). At
// the weight-streaming (decode) shape every expert holds a handful of token
// rows, and a 32-row box makes one MMA step an eighth of a 128 x 256 step; at
// prefill a 128-row box gives each 64-deep chunk 512 tensor cycles against
// about 300 cycles of decoding, and the token tile is the innermost index of
// the tile walk, so concurrent tiles share a weight tile through L2. Each
// converter thread owns one weight row: it reads the
// row's codes from the shared-memory code ring, decodes them to fp16 in
// registers (FP8: hardware e4m3x2 conversion; MXFP4: e2m1x2 conversion times
// the block's 2^(X - X_row)), and stores them straight into TMEM with
// tcgen05.st, where the MMA reads A (tcgen05.mma with A in tensor memory).
// Decoded weights therefore never touch shared memory, which holds only codes
// (six stages, 192 KB at N = 32; four at N = 128) and activation boxes, and
// TMEM holds up to six (N = 128: four) decoded 64-deep chunks ahead of the MMA.
//
// Tile: one 128-row tile of an expert's segment of routed rows, of which the
// activation box loads the first N (at N = 32 or 64 the batch holds at most N
// rows, so a segment is one tile and its rows fit the box), against two
// 128-row weight matrices: gate/up = W_g and W_u rows [128 nb, 128 nb + 128),
// down = W_d rows [256 nb, 256 nb + 256) as two halves. D holds, per matrix,
// 128 weight rows (TMEM lanes) x N tokens (columns), double buffered at N <= 64
// so one tile's epilogue overlaps the next tile's MMAs (single at N = 128).
// Epilogue: lane j = weight row, column c = token: gate/up writes
// H[c][j] = SiLU(g s_g) (u s_u) as fp16; down writes Yrows[c][j] =
// gate_c (d s_d) as bf16, s_* the per-row weight scale (FP8) or row factor
// (MXFP4).
//
// Warp roles (512 threads): 0 activation producer, 1 TMEM owner and MMA issuer
// of matrix 0, 2..5 epilogue (TMEM lane quadrant w % 4), 6..13 converters
// (matrix (w - 6) / 4, lane quadrant w % 4), 14 weight-code producer, 15 MMA
// issuer of matrix 1.
// Synchronisation, all waits bounded:
//   qfull[q]  code producer expect_tx + TMA bytes;     qempty[q] 8 converter warps
//   bfull[b]  activation producer expect_tx + bytes;   bempty[b] 2 MMA commits
//   afull[a]  8 converter warps (after tcgen05.st, wait::st and the tcgen05
//             fence);                                   aempty[a] 2 MMA commits
// The ring of decoded chunks in TMEM is short (six slots at N = 32), so its
// round trip (decode, store, publish, MMA issue, MMA completion, release) sets
// the pace: every chunk is published on its own as soon as it is stored, and
// the token box is checked by the MMA threads, not by a converter warp (the
// slowest of the eight converter warps gates every chunk).
//   tfull[2]  2 MMA commits;                            tempty[2] 4 epilogue warps
// Sources: AI Engineering Illustrated "Mixture of Experts", "Trade-offs to
// weigh" (small-batch MoE is bound by reading expert weights; quantising them
// attacks that directly); jacopoparretti "Mixture of experts, token by token",
// "Memory".
#pragma once
#include "quant_formats.cuh"

namespace moe {
namespace wqs {

using tc::BK;
using tc::BM;
using tc::UMMA_K;
using tc::TcMaps;

constexpr int CONV_WARPS = 8;
constexpr int CONV_WARP0 = 6;
constexpr int QPROD_WARP = CONV_WARP0 + CONV_WARPS;
constexpr int MMA2_WARP = QPROD_WARP + 1;  // issues matrix 1's MMAs (warp 1 issues matrix 0's)
constexpr int NUM_THREADS = (MMA2_WARP + 1) * 32;
constexpr int MMA_ISSUERS = 2;
constexpr int EPI_WARPS = 4;
constexpr uint32_t TMEM_COLS = 512;
constexpr int BAR_BYTES = 512;
constexpr int Q_ROW = 128;                  // bytes per weight row in a code stage
constexpr int Q_BYTES = 2 * BM * Q_ROW;     // two 128-row matrices: 32 KB
constexpr int A_COLS = 2 * (BK / 2);        // TMEM columns of one decoded chunk (2 matrices)

// Shape for token boxes of NB rows (32, 64 or 128) and weight format WQ. With
// 128-row boxes two accumulators would fill TMEM, so D is single-buffered there
// (the epilogue then does not overlap the next tile's MMAs) and four decoded
// chunks fit beside it.
template <int NB, int WQ>
struct WqShape {
  static_assert(NB == 32 || NB == 64 || NB == 128, "token box rows");
  static constexpr int QCH = WQ == tcf8::WQ_MXFP4 ? 4 : 2;  // 64-deep chunks per code stage
  static constexpr int B_BYTES = NB * BK * 2;               // fp16 token box of one chunk
  static constexpr int NBS = NB == 128 ? 6 : 8;             // token boxes in flight
  static constexpr int NACC = NB == 128 ? 1 : 2;            // accumulator buffers
  static constexpr int D_COLS = NACC * 2 * NB;              // buffers x 2 matrices x NB
  static constexpr int NA = (TMEM_COLS - D_COLS) / A_COLS;  // decoded chunks in TMEM
  static constexpr int NQ = (232448 - 1024 - BAR_BYTES - NBS * B_BYTES) / Q_BYTES;
  static constexpr int SMEM_BYTES = 1024 + NQ * Q_BYTES + NBS * B_BYTES + BAR_BYTES;
  static_assert(NA >= 2 && NQ >= 2, "rings");
  static_assert(SMEM_BYTES <= 232448, "shared memory per block");
  static_assert(2 * NQ + 2 * NBS + 2 * NA + 6 <= BAR_BYTES / 8 - 2, "barrier area");
};

struct WqGroup {
  const int32_t* tile_start;  // [E + 1] segment starts (128-row tiles) of the routed rows
  int E;
  int rows;                   // rows of the permuted buffers (bounds checks of MOE_DEBUG)
  int n_tiles;                // weight-row tiles per expert (128 rows per matrix, 2 matrices)
  int k_blocks;               // K / 64
  int N;                      // weight rows of the matrix (output columns)
  void* out;                  // gate/up: fp16 H [rows, N]; down: bf16 Yrows [rows, N]
  const float* row_gate;      // down: gate of each permuted row
  const float* scale0;        // per weight row: W_g (gate/up) or W_d scales / row factors
  const float* scale1;        // W_u (gate/up)
  int64_t scale_stride;       // floats between experts
  const uint8_t* bscale0;     // MXFP4 block exponents, [rows][K / 32] per expert
  const uint8_t* bscale1;
  int64_t bscale_stride;      // bytes between experts
  int kblk;                   // K / 32
};

struct WqParams {
  WqGroup grp;
  unsigned long long timeout_ns;
  unsigned long long drain_timeout_ns;
  int* call_err;
};

// 32 consecutive 32-bit TMEM columns of this warp's 32 lanes <- 32 registers.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),
      "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),
      "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T: A in tensor memory (one row per lane, K along
// the columns, two fp16 per column), B a K-major shared-memory tile.
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accum)
      : "memory");
}

// Tile walk: experts in order, each expert's weight-row tiles in order.
__device__ __forceinline__ tc::TileInfo decode_tile_wq(long long tile, const WqGroup& g,
                                                      const int32_t* ts) {
  tc::TileInfo ti;
  ti.g = 0;
  const long long q = tile / g.n_tiles;
  int lo = 0, hi = g.E - 1;  // last expert whose first tile is at or before q
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (ts[mid] <= q) lo = mid; else hi = mid - 1;
  }
  const int me = ts[lo + 1] - ts[lo];
  const long long in_e = tile - (long long)g.n_tiles * ts[lo];
  ti.e = lo;
  ti.nb = (int)(in_e / me);
  ti.row0 = (ts[lo] + (int)(in_e % me)) * BM;
  return ti;
}

// Builds with MOE_DEBUG: a tile outside the buffers (see tc::tile_out_of_bounds).
__device__ __forceinline__ bool wq_tile_bad(const tc::TileInfo& ti, const WqGroup& g, int nb_rows) {
#if defined(MOE_DEBUG)
  return ti.nb < 0 || ti.nb >= g.n_tiles || ti.e < 0 || ti.e >= g.E || ti.row0 < 0 ||
         ti.row0 + nb_rows > g.rows;
#else
  (void)ti; (void)g; (void)nb_rows;
  return false;
#endif
}

template <int EPI, int NB, int WQ>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    tc_wq_swap_kernel(const __grid_constant__ TcMaps maps, const WqParams p) {
  using Sh = WqShape<NB, WQ>;
  constexpr int NQ = Sh::NQ, NBS = Sh::NBS, NA = Sh::NA, QCH = Sh::QCH;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = tc::smem_addr(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* q_base = smem;                               // NQ code stages
  uint8_t* b_base = q_base + NQ * Q_BYTES;              // NBS token boxes
  uint64_t* bars = reinterpret_cast<uint64_t*>(b_base + NBS * Sh::B_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * NQ + 2 * NBS + 2 * NA + 6);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t q_0 = tc::smem_addr(q_base);
  const uint32_t b_0 = tc::smem_addr(b_base);
  const uint32_t bar0 = tc::smem_addr(bars);
  auto qfull = [&](int i) { return bar0 + 8u * i; };
  auto qempty = [&](int i) { return bar0 + 8u * (NQ + i); };
  auto bfull = [&](int i) { return bar0 + 8u * (2 * NQ + i); };
  auto bempty = [&](int i) { return bar0 + 8u * (2 * NQ + NBS + i); };
  auto afull = [&](int i) { return bar0 + 8u * (2 * NQ + 2 * NBS + i); };
  auto aempty = [&](int i) { return bar0 + 8u * (2 * NQ + 2 * NBS + NA + i); };
  constexpr int T0 = 2 * NQ + 2 * NBS + 2 * NA;
  auto tfull = [&](int a) { return bar0 + 8u * (T0 + a); };
  auto tempty = [&](int a) { return bar0 + 8u * (T0 + 2 + a); };
  const uint32_t done_bar = bar0 + 8u * (T0 + 4);  // one per MMA issuer

  const WqGroup& G = p.grp;
  if (threadIdx.x == 0) {
    for (int i = 0; i < NQ; ++i) {
      tc::mbar_init(qfull(i), 1);
      tc::mbar_init(qempty(i), CONV_WARPS);
    }
    for (int i = 0; i < NBS; ++i) {
      tc::mbar_init(bfull(i), 1);
      tc::mbar_init(bempty(i), MMA_ISSUERS);
    }
    for (int i = 0; i < NA; ++i) {
      tc::mbar_init(afull(i), CONV_WARPS);
      tc::mbar_init(aempty(i), MMA_ISSUERS);
    }
    for (int a = 0; a < 2; ++a) {
      tc::mbar_init(tfull(a), MMA_ISSUERS);
      tc::mbar_init(tempty(a), EPI_WARPS);
    }
    for (int i = 0; i < MMA_ISSUERS; ++i) tc::mbar_init(done_bar + 8u * i, 1);
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
  // TMEM columns: D[buffer][matrix] at (2 buffer + matrix) NB; decoded chunk
  // slot s at D_COLS + s A_COLS, matrix m's 32 columns at + 32 m
  auto d_col = [&](int buf, int m) { return (uint32_t)((2 * buf + m) * NB); };
  auto a_col = [&](int s, int m) { return (uint32_t)(Sh::D_COLS + s * A_COLS + m * (BK / 2)); };

  const int32_t* ts = G.tile_start;
  const long long total = (long long)G.n_tiles * ts[G.E];
  const int nck = G.k_blocks;
  const int nqs = (nck + QCH - 1) / QCH;
  const unsigned long long tmo = p.timeout_ns, drain_tmo = p.drain_timeout_ns;

  if (warp == 0) {
    // ------------------------------------------------------ token-box producer
    if (lane == 0) {
      tc::prefetch_map(&maps.a[0]);
      int bs = 0;
      uint32_t bph = 0, issued = 0, par = 0;
      bool ok = true;
      for (long long tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
        const tc::TileInfo ti = decode_tile_wq(tile, G, ts);
        if (wq_tile_bad(ti, G, NB)) {
          flag_bounds();
          continue;
        }
        for (int g = 0; g < nck; ++g) {
          if (!tc::wait_bounded(bempty(bs), bph ^ 1u, abort_flag, tmo)) { ok = false; break; }
          tc::mbar_expect_tx(bfull(bs), Sh::B_BYTES);
          tc::tma_load_2d(b_0 + bs * Sh::B_BYTES, &maps.a[0], bfull(bs), g * BK, ti.row0);
          issued |= 1u << bs;
          par = (par & ~(1u << bs)) | (bph << bs);
          if (++bs == NBS) { bs = 0; bph ^= 1u; }
        }
      }
      if (!ok)  // let every copy already issued land before the CTA exits
        for (int i = 0; i < NBS; ++i)
          if ((issued >> i) & 1u) tc::wait_drain(bfull(i), (par >> i) & 1u, abort_flag, drain_tmo);
    }
  } else if (warp == QPROD_WARP) {
    // ---------------------------------------------------------- code producer
    if (lane == 0) {
      tc::prefetch_map(&maps.b0[0]);
      if (EPI == tc::EPI_SWIGLU_TC) tc::prefetch_map(&maps.b1[0]);
      int qs = 0;
      uint32_t qph = 0, issued = 0, par = 0;
      bool ok = true;
      for (long long tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
        const tc::TileInfo ti = decode_tile_wq(tile, G, ts);
        if (wq_tile_bad(ti, G, NB)) continue;
        for (int qi = 0; qi < nqs; ++qi) {
          if (!tc::wait_bounded(qempty(qs), qph ^ 1u, abort_flag, tmo)) { ok = false; break; }
          const uint32_t dq = q_0 + qs * Q_BYTES;
          const int x = qi * (Q_ROW / 4);  // the codes are described as 32-bit words
          tc::mbar_expect_tx(qfull(qs), Q_BYTES);
          if (EPI == tc::EPI_SWIGLU_TC) {
            tc::tma_load_3d(dq, &maps.b0[0], qfull(qs), x, ti.nb * BM, ti.e);
            tc::tma_load_3d(dq + Q_BYTES / 2, &maps.b1[0], qfull(qs), x, ti.nb * BM, ti.e);
          } else {
            tc::tma_load_3d(dq, &maps.b0[0], qfull(qs), x, ti.nb * 2 * BM, ti.e);
            tc::tma_load_3d(dq + Q_BYTES / 2, &maps.b0[0], qfull(qs), x, ti.nb * 2 * BM + BM, ti.e);
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
  } else if (warp == 1 || warp == MMA2_WARP) {
    // --------------------------------------------------------------- MMA issuers
    // Two threads issue the tile's MMAs, one per weight matrix (its own D), so
    // that the small MMAs of the swapped shape are issued twice as fast; both
    // commit to the shared barriers (counts of two).
    if (lane == 0) {
      const int mi = warp == 1 ? 0 : 1;
      constexpr uint32_t IDESC = tcf8::make_idesc_f16(BM, NB);
      int as = 0, bs = 0;
      uint32_t aph = 0, bph = 0, acc = 0, acc_phase = 0;
      bool ok = true;
      for (long long tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
        {
          const tc::TileInfo ti = decode_tile_wq(tile, G, ts);
          if (wq_tile_bad(ti, G, NB)) continue;
        }
        if (!tc::wait_bounded(tempty(acc), acc_phase ^ 1u, abort_flag, tmo)) { ok = false; break; }
        tc::tc_fence_after();
        for (int g = 0; g < nck; ++g) {
          if (!tc::wait_fast(afull(as), aph, abort_flag, tmo)) { ok = false; break; }
          if (!tc::wait_fast(bfull(bs), bph, abort_flag, tmo)) { ok = false; break; }
          tc::tc_fence_after();
          const uint64_t bd = tc::sw128_kmajor_desc(b_0 + bs * Sh::B_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / UMMA_K; ++kk) {
            // +32 bytes per K step in the B descriptor; +8 TMEM columns in A
            tc_mma_ts(tmem_base + d_col(acc, mi), tmem_base + a_col(as, mi) + 8u * kk, bd + 2u * kk,
                      IDESC, (g | kk) != 0 ? 1u : 0u);
          }
          tc::tc_commit(aempty(as));  // the decoded chunk has been read
          tc::tc_commit(bempty(bs));  // and the token box
          if (++as == NA) { as = 0; aph ^= 1u; }
          if (++bs == NBS) { bs = 0; bph ^= 1u; }
        }
        if (!ok) break;
        tc::tc_commit(tfull(acc));
        if (++acc == (uint32_t)Sh::NACC) { acc = 0; acc_phase ^= 1u; }
      }
      tc::tc_commit(done_bar + 8u * mi);
      tc::wait_drain(done_bar + 8u * mi, 0u, abort_flag, drain_tmo);
    }
  } else if (warp >= CONV_WARP0 && warp < CONV_WARP0 + CONV_WARPS) {
    // ---------------------------------------------------------------- converters
    // Thread (matrix m, quadrant q, lane l) owns weight row r = 32 q + l of
    // matrix m: row m * 128 + r of the code stage, TMEM lane r. Per 64-deep chunk
    // h of a code stage it reads the row's codes (FP8: 64 bytes, 16-byte chunks
    // 4h..4h+3; MXFP4: 32 bytes, chunks 2h, 2h+1; chunk j of a row is stored at
    // j ^ (row & 7), so the 8 lanes of every shared-memory phase read 8 distinct
    // 16-byte bank groups), decodes 64 fp16 values and stores them to the chunk's
    // TMEM slot, 32 columns.
    const int m = (warp - CONV_WARP0) >> 2;
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const int qrow = m * BM + r;
    const uint32_t q_row_off = qrow * Q_ROW;
    const int rsw = qrow & 7;
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    int qs = 0, as = 0;
    uint32_t qph = 0, aph = 0;
    bool ok = true;
    // MXFP4: this row's block exponents (this code stage's eight and the next
    // stage's, loaded one stage ahead) and 1 / its row factor
    const uint8_t* bsrow = nullptr;
    float inv_rf = 0.f;
    uint2 bs_cur = make_uint2(0u, 0u), bs_nxt = make_uint2(0u, 0u);
    for (long long tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
      const tc::TileInfo ti = decode_tile_wq(tile, G, ts);
      if (wq_tile_bad(ti, G, NB)) continue;
      if constexpr (WQ == tcf8::WQ_MXFP4) {
        const int grow = EPI == tc::EPI_SWIGLU_TC ? ti.nb * BM + r : ti.nb * 2 * BM + m * BM + r;
        const bool valid = grow < G.N;  // rows past N are zero-filled by TMA
        const uint8_t* bs = (EPI == tc::EPI_SWIGLU_TC && m == 1) ? G.bscale1 : G.bscale0;
        const float* rf = (EPI == tc::EPI_SWIGLU_TC && m == 1) ? G.scale1 : G.scale0;
        bsrow = valid ? bs + (int64_t)ti.e * G.bscale_stride + (int64_t)grow * G.kblk : nullptr;
        inv_rf = valid ? 1.0f / __ldg(rf + (int64_t)ti.e * G.scale_stride + grow) : 0.f;
        bs_nxt = bsrow != nullptr ? __ldg(reinterpret_cast<const uint2*>(bsrow)) : make_uint2(0u, 0u);
      }
      for (int g = 0; g < nck; ++g) {
        const int h = g % QCH;
        int w = 1;
        if (lane == 0) w = tc::wait_fast(aempty(as), aph ^ 1u, abort_flag, tmo) ? 1 : 0;
        if (!__shfl_sync(0xffffffffu, w, 0)) { ok = false; break; }
        tc::tc_fence_after();
        if (h == 0) {
          // lane 0 waits for the code stage; the others then observe the completed
          // phase themselves (it cannot move on before this warp releases it)
          if (lane == 0) w = tc::wait_fast(qfull(qs), qph, abort_flag, tmo) ? 1 : 0;
          if (!__shfl_sync(0xffffffffu, w, 0)) { ok = false; break; }
          (void)tc::mbar_try_wait(qfull(qs), qph);
          if constexpr (WQ == tcf8::WQ_MXFP4) {
            bs_cur = bs_nxt;
            const int qn = g / QCH + 1;
            if (qn < nqs && bsrow != nullptr)
              bs_nxt = __ldg(reinterpret_cast<const uint2*>(bsrow + (size_t)qn * 8));
          }
        }
        uint32_t o[32];
        const uint8_t* qr = q_base + qs * Q_BYTES + q_row_off;
        if constexpr (WQ == tcf8::WQ_MXFP4) {
          uint2 cc[4];
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const uint4 v = *reinterpret_cast<const uint4*>(qr + (((2 * h + j) ^ rsw) << 4));
            cc[2 * j] = make_uint2(v.x, v.y);
            cc[2 * j + 1] = make_uint2(v.z, v.w);
          }
#pragma unroll
          for (int j = 0; j < 2; ++j) {  // blocks 2h + j of this code stage
            const int blk = 2 * h + j;
            const uint32_t wbs = blk < 4 ? bs_cur.x : bs_cur.y;
            const uint32_t mult =
                tcf8::mx_block_multiplier((wbs >> (8 * (blk & 3))) & 0xFFu, inv_rf);
            tcf8::mxfp4x16_to_f16x16(cc[2 * j], mult, o + 16 * j);
            tcf8::mxfp4x16_to_f16x16(cc[2 * j + 1], mult, o + 16 * j + 8);
          }
        } else {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint4 v = *reinterpret_cast<const uint4*>(qr + (((4 * h + j) ^ rsw) << 4));
            tcf8::e4m3x4_to_f16x4(v.x, o[8 * j], o[8 * j + 1]);
            tcf8::e4m3x4_to_f16x4(v.y, o[8 * j + 2], o[8 * j + 3]);
            tcf8::e4m3x4_to_f16x4(v.z, o[8 * j + 4], o[8 * j + 5]);
            tcf8::e4m3x4_to_f16x4(v.w, o[8 * j + 6], o[8 * j + 7]);
          }
        }
        if (h == QCH - 1 || g == nck - 1) {  // this code stage is fully read
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(qempty(qs));
          if (++qs == NQ) { qs = 0; qph ^= 1u; }
        }
        tmem_st32(tmem_base + lane_base + a_col(as, m), o);
        tmem_st_wait();
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(afull(as));
        if (++as == NA) { as = 0; aph ^= 1u; }
      }
    }
    tmem_st_wait();  // an aborted chunk may have stores in flight: TMEM is freed below
  } else {
    // ---------------------------------------------------------------- epilogue
    const int q = warp & 3;
    const int r = q * 32 + lane;  // weight row within each 128-row matrix
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    uint32_t acc = 0, acc_phase = 0;
    for (long long tile = blockIdx.x; tile < total; tile += gridDim.x) {
      const tc::TileInfo ti = decode_tile_wq(tile, G, ts);
      if (wq_tile_bad(ti, G, NB)) continue;
      int ok = 1;
      if (lane == 0) ok = tc::wait_bounded(tfull(acc), acc_phase, abort_flag, tmo) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc::tc_fence_after();
#pragma unroll 1
      for (int c0 = 0; c0 < NB; c0 += 32) {
        float d0[32], d1[32];
        __syncwarp();
        tc::tmem_ld32(tmem_base + lane_base + d_col(acc, 0) + c0, d0);
        tc::tmem_ld32(tmem_base + lane_base + d_col(acc, 1) + c0, d1);
        if (EPI == tc::EPI_SWIGLU_TC) {
          const int col = ti.nb * BM + r;
          if (col < G.N) {
            const float s0 = G.scale0[(int64_t)ti.e * G.scale_stride + col];
            const float s1 = G.scale1[(int64_t)ti.e * G.scale_stride + col];
            __half* out = reinterpret_cast<__half*>(G.out) + col;
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              const float hv = silu_f32(d0[c] * s0) * (d1[c] * s1);
              out[(size_t)(ti.row0 + c0 + c) * G.N] =
                  __float2half_rn(fminf(fmaxf(hv, -65504.f), 65504.f));
            }
          }
        } else {
#pragma unroll
          for (int mm = 0; mm < 2; ++mm) {
            const int col = ti.nb * 2 * BM + mm * BM + r;
            if (col < G.N) {
              const float s = G.scale0[(int64_t)ti.e * G.scale_stride + col];
              __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(G.out) + col;
              const float* dv = mm == 0 ? d0 : d1;
#pragma unroll
              for (int c = 0; c < 32; ++c) {
                const int row = ti.row0 + c0 + c;
                out[(size_t)row * G.N] = __float2bfloat16_rn(G.row_gate[row] * (dv[c] * s));
              }
            }
          }
        }
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(tempty(acc));
      if (++acc == (uint32_t)Sh::NACC) { acc = 0; acc_phase ^= 1u; }
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

}  // namespace wqs
}  // namespace moe
