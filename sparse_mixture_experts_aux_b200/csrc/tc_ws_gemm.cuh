// Grouped expert GEMMs with bf16 weights and the operands swapped, for layers
// whose experts get a few hundred routed rows each.
//
// Each expert's routed rows sit in a segment padded to 128-row tiles. The
// token-major kernel (tc_gemm.cuh) multiplies whole 128-row tiles, so at about
// 256 rows per expert (the DeepSeek-V3 shape: 8192 tokens x 8 of 256 experts)
// the padding of each segment's last tile is a fifth to a quarter of its MMAs.
// Here the weights are the MMA's A operand (M = 128 weight rows, straight from
// the shared-memory stage) and the tile's token rows are B, with N = the
// tile's valid rows rounded up to 16, so a tile computes at most 15 padding
// rows. Tile walk as in the token-major kernel: group 0 (routed experts) then
// group 1 (the shared expert over all tokens), n-tile-major with the token
// tiles fastest, so the tiles that run at the same time share a weight tile
// through L2.
//
// Tile: one 128-row token tile of an expert's segment against two 128-row
// weight matrices: gate/up = W_g and W_u rows [128 nb, 128 nb + 128), down =
// W_d rows [256 nb, 256 nb + 256) as two halves. D per matrix: 128 weight rows
// (TMEM lanes) x up to 128 tokens (columns), double buffered (2 buffers x 2
// matrices x 128 columns = the 512 TMEM columns), so one tile's epilogue
// overlaps the next tile's MMAs.
// Warp roles (256 threads): 0 and 7 TMA producers (alternate K steps of one
// walk), 1 TMEM owner and MMA issuer of matrix 0, 6 MMA issuer of matrix 1,
// 2..5 epilogue (TMEM lane quadrant w % 4): lane j = weight row, column c =
// token; gate/up writes H[c][j] = SiLU(g) u, down writes Yrows[c][j] =
// gate_c d, as bf16, for the tile's valid rows only.
// Synchronisation, all waits bounded:
//   full[s]   producer expect_tx + TMA bytes;   empty[s]  2 MMA commits
//   tfull[2]  2 MMA commits;                    tempty[2] 4 epilogue warps
// Sources: Zero to Frontier 13.1 "The MoE layer" (grouped expert GEMMs over
// the sorted rows); jacopoparretti "Mixture of experts, token by token"
// (DeepSeek-V3: 256 routed experts, 8 per token, one shared expert).
#pragma once
#include "tc_gemm.cuh"

namespace moe {
namespace tcws {

using tc::BK;
using tc::BM;
using tc::UMMA_K;
using tc::TcGroup;
using tc::TcMaps;
using tc::TcParams;
using tc::TileInfo;

constexpr int NB = 128;                           // token rows per tile
constexpr int STAGES = 4;
constexpr int W_BYTES = BM * BK * 2;              // one weight box, 128 rows x 64 bf16
constexpr int X_BYTES = NB * BK * 2;              // the token box
constexpr int STAGE_BYTES = 2 * W_BYTES + X_BYTES;
constexpr int BAR_BYTES = 256;
constexpr int NUM_THREADS = 256;
constexpr int MMA2_WARP = 6;
constexpr int PROD2_WARP = 7;
constexpr int EPI_WARPS = 4;
constexpr uint32_t TMEM_COLS = 512;
constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + BAR_BYTES + 4 * (tc::MAX_E + 1);
static_assert(SMEM_BYTES <= 232448, "shared memory per block");
static_assert(W_BYTES % 1024 == 0 && X_BYTES % 1024 == 0, "1024-byte aligned boxes");

// Valid token rows of a tile, 1..128: routed groups take the expert's kept
// rows (its count, capped at the capacity), dense groups the group's rows.
__device__ __forceinline__ int tile_rows(const TileInfo& ti, const TcGroup& g,
                                         const int32_t* s_ts) {
  int v;
  if (ti.g == 0 && g.tile_start != nullptr) {
    int kept = g.counts[ti.e];
    if (g.cap >= 0 && kept > g.cap) kept = static_cast<int>(g.cap);
    v = kept - (ti.row0 - s_ts[ti.e] * BM);
  } else {
    v = g.rows - ti.row0;
  }
  return v < 1 ? 1 : (v > NB ? NB : v);
}

template <int EPI>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    tc_ws_grouped_gemm_kernel(const __grid_constant__ TcMaps maps, const TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = tc::smem_addr(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  // bars: full[STAGES], empty[STAGES], tfull[2], tempty[2], done[2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 6);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int32_t* s_ts = reinterpret_cast<int32_t*>(smem + STAGES * STAGE_BYTES + BAR_BYTES);
  static_assert((2 * STAGES + 6) * 8 + 8 <= BAR_BYTES, "barrier area");

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t stage0 = tc::smem_addr(smem);
  const uint32_t bar0 = tc::smem_addr(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + 2 + a); };
  auto done_bar = [&](int i) { return bar0 + 8u * (2 * STAGES + 4 + i); };

  const TcGroup& G0 = p.g[0];
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      tc::mbar_init(full_bar(s), 1);
      tc::mbar_init(empty_bar(s), 2);  // one commit per MMA issuer
    }
    for (int a = 0; a < 2; ++a) {
      tc::mbar_init(tfull_bar(a), 2);
      tc::mbar_init(tempty_bar(a), EPI_WARPS);
    }
    tc::mbar_init(done_bar(0), 1);
    tc::mbar_init(done_bar(1), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    tc::tmem_alloc(tc::smem_addr(tmem_slot), TMEM_COLS);
    tc::tmem_relinquish();
  }
  pdl_wait();  // the routing results and rows this GEMM reads are complete
  pdl_launch_dependents();
  if (G0.tile_start != nullptr)
    for (int i = threadIdx.x; i <= G0.E; i += NUM_THREADS) s_ts[i] = G0.tile_start[i];
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const long long tiles0 =
      (long long)G0.n_tiles *
      (G0.tile_start != nullptr ? (long long)s_ts[G0.E] : (long long)((G0.rows + BM - 1) / BM));
  const long long tiles1 =
      p.num_groups > 1 ? (long long)p.g[1].n_tiles * ((p.g[1].rows + BM - 1) / BM) : 0;
  const long long total = tiles0 + tiles1;
  const unsigned long long tmo = p.timeout_ns;
  const unsigned long long drain_tmo = p.drain_timeout_ns;

  if (warp == 0 || warp == PROD2_WARP) {
    // ------------------------------------------------------------ producers
    // Two threads take alternate K steps of the same walk (the step's stage is
    // its running index modulo STAGES).
    if (lane == 0) {
      const long long me = warp == 0 ? 0 : 1;
      for (int g = 0; g < p.num_groups; ++g) {
        tc::prefetch_map(&maps.a[g]);
        tc::prefetch_map(&maps.b0[g]);
        if (EPI == tc::EPI_SWIGLU_TC) tc::prefetch_map(&maps.b1[g]);
      }
      uint32_t issued = 0, last_par = 0;
      long long gs = 0;
      bool ok = true;
      for (long long tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
        const TileInfo ti = tc::decode_tile(tile, tiles0, p, s_ts);
        if (tc::tile_out_of_bounds(ti.e, ti.nb, ti.row0, BM, p.g[ti.g])) {
          if (me == 0) flag_bounds();
          continue;
        }
        const int kbs = p.g[ti.g].k_blocks;
        for (int kb = 0; kb < kbs; ++kb, ++gs) {
          if ((gs & 1) != me) continue;
          const int stage = (int)(gs % STAGES);
          const uint32_t phase = (uint32_t)((gs / STAGES) & 1);
          if (!tc::wait_fast(empty_bar(stage), phase ^ 1u, abort_flag, tmo)) { ok = false; break; }
          const uint32_t sw = stage0 + stage * STAGE_BYTES;
          const uint32_t fb = full_bar(stage);
          tc::mbar_expect_tx(fb, STAGE_BYTES);
          if (EPI == tc::EPI_SWIGLU_TC) {
            tc::tma_load_3d(sw, &maps.b0[ti.g], fb, kb * BK, ti.nb * BM, ti.e);
            tc::tma_load_3d(sw + W_BYTES, &maps.b1[ti.g], fb, kb * BK, ti.nb * BM, ti.e);
          } else {
            tc::tma_load_3d(sw, &maps.b0[ti.g], fb, kb * BK, ti.nb * 2 * BM, ti.e);
            tc::tma_load_3d(sw + W_BYTES, &maps.b0[ti.g], fb, kb * BK, ti.nb * 2 * BM + BM, ti.e);
          }
          tc::tma_load_2d(sw + 2 * W_BYTES, &maps.a[ti.g], fb, kb * BK, ti.row0);
          issued |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
        }
      }
      if (!ok)  // let every copy this thread issued land before the CTA exits
        for (int s = 0; s < STAGES; ++s)
          if ((issued >> s) & 1u) tc::wait_drain(full_bar(s), (last_par >> s) & 1u, abort_flag, drain_tmo);
    }
  } else if (warp == 1 || warp == MMA2_WARP) {
    // ------------------------------------------------------------ MMA issuers
    // One thread per weight matrix (its own D); both commit to the shared
    // barriers (counts of two).
    if (lane == 0) {
      const int mi = warp == 1 ? 0 : 1;
      int stage = 0;
      uint32_t phase = 0, acc = 0, acc_phase = 0;
      bool ok = true;
      for (long long tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
        const TileInfo ti = tc::decode_tile(tile, tiles0, p, s_ts);
        if (tc::tile_out_of_bounds(ti.e, ti.nb, ti.row0, BM, p.g[ti.g])) continue;
        const int n_mma = (tile_rows(ti, p.g[ti.g], s_ts) + 15) & ~15;
        const uint32_t idesc = tc::make_idesc(BM, n_mma);
        const int kbs = p.g[ti.g].k_blocks;
        if (!tc::wait_bounded(tempty_bar(acc), acc_phase ^ 1u, abort_flag, tmo)) { ok = false; break; }
        tc::tc_fence_after();
        const uint32_t d_tmem = tmem_base + (2u * acc + mi) * NB;
        for (int kb = 0; kb < kbs; ++kb) {
          if (!tc::wait_fast(full_bar(stage), phase, abort_flag, tmo)) { ok = false; break; }
          tc::tc_fence_after();
          const uint32_t sw = stage0 + stage * STAGE_BYTES;
          const uint64_t ad = tc::sw128_kmajor_desc(sw + mi * W_BYTES);
          const uint64_t bd = tc::sw128_kmajor_desc(sw + 2 * W_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / UMMA_K; ++kk)  // +32 bytes per K step in both descriptors
            tc::tc_mma(d_tmem, ad + 2u * kk, bd + 2u * kk, idesc, (kb | kk) != 0 ? 1u : 0u);
          tc::tc_commit(empty_bar(stage));  // frees the stage once these MMAs have read it
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc::tc_commit(tfull_bar(acc));
        acc ^= 1u;
        if (acc == 0u) acc_phase ^= 1u;
      }
      tc::tc_commit(done_bar(mi));  // every MMA issued above has completed once this fires
      tc::wait_drain(done_bar(mi), 0u, abort_flag, drain_tmo);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int r = q * 32 + lane;  // weight row within each 128-row matrix
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    uint32_t acc = 0, acc_phase = 0;
    for (long long tile = blockIdx.x; tile < total; tile += gridDim.x) {
      const TileInfo ti = tc::decode_tile(tile, tiles0, p, s_ts);
      const TcGroup& g = p.g[ti.g];
      if (tc::tile_out_of_bounds(ti.e, ti.nb, ti.row0, BM, g)) continue;
      const int v = tile_rows(ti, g, s_ts);
      int ok = 1;
      if (lane == 0) ok = tc::wait_bounded(tfull_bar(acc), acc_phase, abort_flag, tmo) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc::tc_fence_after();
      __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(g.out);
#pragma unroll 1
      for (int c0 = 0; c0 < v; c0 += 32) {
        float d0[32], d1[32];
        __syncwarp();  // tcgen05.ld is warp-collective: reconverge after the stores
        tc::tmem_ld32(tmem_base + lane_base + (2u * acc) * NB + c0, d0);
        tc::tmem_ld32(tmem_base + lane_base + (2u * acc + 1u) * NB + c0, d1);
        if (EPI == tc::EPI_SWIGLU_TC) {
          const int col = ti.nb * BM + r;
          if (col < g.N) {
#pragma unroll
            for (int c = 0; c < 32; ++c)
              if (c0 + c < v)
                out[(size_t)(ti.row0 + c0 + c) * g.N + col] =
                    __float2bfloat16_rn(silu_f32(d0[c]) * d1[c]);
          }
        } else {
          // the 32 tokens' gate scales: one coalesced load, lane c holds token c's,
          // broadcast by shuffle (a load per element would wait once per store)
          const float rs = (g.row_scale != nullptr && c0 + lane < v)
                               ? g.row_scale[ti.row0 + c0 + lane] : 1.f;
          const int col0 = ti.nb * 2 * BM + r, col1 = col0 + BM;
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const float sc = __shfl_sync(0xffffffffu, rs, c);  // warp-uniform point
            if (c0 + c < v) {
              __nv_bfloat16* o = out + (size_t)(ti.row0 + c0 + c) * g.N;
              if (col0 < g.N) o[col0] = __float2bfloat16_rn(sc * d0[c]);
              if (col1 < g.N) o[col1] = __float2bfloat16_rn(sc * d1[c]);
            }
          }
        }
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(tempty_bar(acc));
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

}  // namespace tcws
}  // namespace moe
