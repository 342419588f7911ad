// Grouped expert GEMMs on CTA pairs (tcgen05 cta_group::2), sm_100a.
//
// A cluster of two CTAs on two SMs computes one 256x256 fp32 tile: each CTA
// TMA-loads its own 128 rows of A and its own 128-row half of B into its own
// shared memory (no multicast loads anywhere), the leader CTA issues
// tcgen05.mma.cta_group::2 over both CTAs' operands, and each CTA's TMEM ends
// up holding its 128 rows x 256 columns. Per SM this moves 32 KB per 64-deep
// K step for 2 x 128x256x64 MACs, two thirds of the 1-CTA tile's 48 KB.
//
// For the SwiGLU epilogue the leader's B half is 128 rows of W_g and the
// peer's is the matching 128 rows of W_u, so accumulator columns 0..127 are
// the gate and 128..255 the up projection, exactly as in the 1-CTA kernel.
//
// Synchronisation (all waits bounded):
//   full[s]   leader only: one arrive.expect_tx by the leader's producer for
//             both CTAs' bytes; both CTAs' copies complete_tx on it
//             (cp.async.bulk.tensor.cta_group::2 may signal the peer's barrier)
//   empty[s]  both CTAs: the leader's tcgen05.commit multicast to both
//   tfull[a]  both CTAs: the leader's commit multicast to both
//   tempty[a] leader only: 8 epilogue warps of each CTA arrive (remote for the peer)
// Rows are grouped per expert in 128-row segments; a pair tile covers two
// consecutive 128-row tiles of one expert, and when an expert has an odd tile
// count the peer half of its last pair is computed but not stored.
// The SWAP form (down GEMM) exchanges the roles: A is 256 weight rows across
// the pair and B the pair tile's token rows, with N set per tile to its valid
// rows rounded up to 16, so the odd expert's last tile is not padded.
#pragma once
#include "tc_gemm.cuh"

namespace moe {
namespace tc2 {

using tc::BK;
using tc::UMMA_K;
using tc::TcMaps;

constexpr int HALF_M = 128;                // rows per CTA
constexpr int BN = 256;                    // accumulator columns
constexpr int STAGES = 6;
constexpr int A_BYTES = HALF_M * BK * 2;   // 16 KB
constexpr int B_BYTES = 128 * BK * 2;      // 16 KB (this CTA's half of B)
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
// warp 0 producer, 1 MMA, 2-5 and 6-9 epilogue (two warps per TMEM lane
// quadrant, each taking every other 32-column chunk)
constexpr int NUM_THREADS = 320;
constexpr int EPI_WARPS = 8;
constexpr uint32_t TMEM_COLS = 512;
constexpr int BAR_BYTES = 256;
constexpr int SMEM_BYTES =
    1024 + STAGES * STAGE_BYTES + BAR_BYTES + 2 * 4 * (tc::MAX_E + 1);
constexpr unsigned long long ABORT_SETTLE_NS = 200000;  // let stray copies land on abort

static_assert(HALF_M == ROW_TILE, "pair halves must match the segment padding");

struct Tc2Group {
  const int32_t* tile_start;  // routed: [E+1] segment starts in 128-row tiles; NULL = dense
  const int32_t* pair_start;  // routed: [E+1] exclusive scan of ceil(tiles_e / 2)
  int E;
  int rows;                   // dense groups: valid rows; routed groups: rows of the permuted
                              // buffers (the bounds checks of MOE_DEBUG builds)
  int n_tiles;                // output tiles per expert along N
  int k_blocks;               // K / BK
  int N;                      // output columns
  void* out;                  // bf16 [rows, N]
  const float* row_scale;     // scale epilogue: factor per row; NULL = 1
  // SWAP kernels: assignments per expert and the capacity (-1: none), which
  // give each token tile's valid rows
  const int32_t* counts;
  int64_t cap;
};

struct Tc2Params {
  Tc2Group g[2];
  int num_groups;
  unsigned long long timeout_ns;
  unsigned long long drain_timeout_ns;
  int* call_err;  // the call's own status word (NULL: none)
};

// ----------------------------------------------------------------------------
// Cluster / cta_group::2 PTX wrappers.
// ----------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Address of the same shared-memory variable in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
// Per-thread (non-.aligned) cluster barrier: safe where a warp's lanes arrive
// from different code paths.
__device__ __forceinline__ void cluster_sync() {
  asm volatile(
      "barrier.cluster.arrive.release;\n\t"
      "barrier.cluster.wait.acquire;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}
__device__ __forceinline__ void st_cluster_u32(uint32_t cluster_addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(cluster_addr), "r"(v) : "memory");
}
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map,
                                                 uint32_t bar_cluster, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d_pair(uint32_t dst, const CUtensorMap* map,
                                                 uint32_t bar_cluster, int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_mma_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum)
      : "memory");
}
// Arrive once on the barrier at offset `bar` in every CTA of `mask` when all
// tcgen05 operations issued so far by this thread have completed.
__device__ __forceinline__ void tc_commit_pair_mc(uint32_t bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(bar),
      "h"(mask)
      : "memory");
}
__device__ __forceinline__ void tc_commit_pair(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}

// Bounded wait that also tells the peer CTA to stop when it gives up.
__device__ __noinline__ bool wait_pair(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                       uint32_t peer_abort_cluster,
                                       unsigned long long timeout_ns) {
  if (tc::mbar_try_wait(bar, parity)) return true;
  const uint64_t limit = wait_cycles(timeout_ns);
  const long long t0 = clock64();
  for (uint32_t it = 1;; ++it) {
    if (tc::mbar_try_wait(bar, parity)) return true;
    if ((it & 15u) == 1u) {
      if (*abort_flag) return false;
      if (static_cast<uint64_t>(clock64() - t0) > limit) {
        atomicOr(&g_dev_error, DEVERR_TIMEOUT);
        *abort_flag = 1;
        st_cluster_u32(peer_abort_cluster, 1u);
        return false;
      }
    }
  }
}

// The same with the first test inline: a phase that has already completed
// costs one try_wait instead of a call (the issuing threads of the main loop
// wait once per K step).
__device__ __forceinline__ bool wait_pair_fast(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                               uint32_t peer_abort, unsigned long long timeout_ns) {
  return tc::mbar_try_wait(bar, parity) || wait_pair(bar, parity, abort_flag, peer_abort, timeout_ns);
}

struct PairTile {
  int g, e, row0, nb;
  bool half_valid[2];
};

// Tile order: group 0 then group 1; within a routed group expert by expert,
// within an expert n-tile-major with the pair index fastest.
__device__ __forceinline__ PairTile decode_pair(long long tile, long long tiles0,
                                                const Tc2Params& p, const int32_t* s_ts,
                                                const int32_t* s_ps) {
  PairTile t;
  const Tc2Group* g;
  long long local = tile;
  if (tile < tiles0) {
    t.g = 0;
    g = &p.g[0];
  } else {
    t.g = 1;
    g = &p.g[1];
    local = tile - tiles0;
  }
  if (t.g == 0 && g->tile_start != nullptr) {
    const long long q = local / g->n_tiles;
    int lo = 0, hi = g->E - 1;  // last expert whose first pair is at or before q
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_ps[mid] <= q) lo = mid; else hi = mid - 1;
    }
    const int pe = s_ps[lo + 1] - s_ps[lo];
    const int me = s_ts[lo + 1] - s_ts[lo];
    const long long in_e = local - (long long)g->n_tiles * s_ps[lo];
    const int pm = (int)(in_e % pe);
    t.e = lo;
    t.nb = (int)(in_e / pe);
    t.row0 = (s_ts[lo] + 2 * pm) * HALF_M;
    t.half_valid[0] = true;
    t.half_valid[1] = (2 * pm + 1) < me;
  } else {
    const int mt = (g->rows + HALF_M - 1) / HALF_M;
    const int pt = (mt + 1) / 2;
    t.e = 0;
    t.nb = (int)(local / pt);
    t.row0 = (int)(local % pt) * 2 * HALF_M;
    t.half_valid[0] = true;
    t.half_valid[1] = true;  // dense rows are masked by row < rows
  }
  return t;
}

// Builds with MOE_DEBUG: a pair tile whose expert, N block or rows fall outside
// the buffers (routed: both CTAs' rows when the second half is valid, else the
// first CTA's; dense: the first row). Release builds: false.
__device__ __forceinline__ bool pair_out_of_bounds(const PairTile& t, const Tc2Group& g) {
#if defined(MOE_DEBUG)
  if (t.nb < 0 || t.nb >= g.n_tiles || t.row0 < 0) return true;
  if (g.tile_start != nullptr)
    return t.e < 0 || t.e >= g.E || t.row0 + HALF_M * (t.half_valid[1] ? 2 : 1) > g.rows;
  return t.row0 >= g.rows;
#else
  (void)t; (void)g;
  return false;
#endif
}

// SWAP kernels: valid token rows of a pair tile's 256-row token tile, 1..256
// (routed groups: the expert's kept rows past the tile's start; dense: the
// group's rows).
__device__ __forceinline__ int pair_rows(const PairTile& t, const Tc2Group& g,
                                         const int32_t* s_ts) {
  int v;
  if (t.g == 0 && g.tile_start != nullptr) {
    int kept = g.counts[t.e];
    if (g.cap >= 0 && kept > g.cap) kept = static_cast<int>(g.cap);
    v = kept - (t.row0 - s_ts[t.e] * HALF_M);
  } else {
    v = g.rows - t.row0;
  }
  return v < 1 ? 1 : (v > 2 * HALF_M ? 2 * HALF_M : v);
}

// SWAP (down GEMM only): the operands swapped, as in tc_ws_gemm.cuh. A = 256
// rows of W_d across the pair (128 per CTA: maps.a is the weight map), B = the
// tile's 256-row token tile (maps.b0, the rows' map): each CTA loads its half,
// N / 2 rows from row0 + (N / 2) rank, N = the tile's valid rows rounded up to
// 16, so the segment padding of an expert's last tile is not multiplied. Each
// CTA's TMEM holds its 128 weight rows x N tokens; the epilogue stores
// transposed (lane = output column).
template <int EPI, bool SWAP = false>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    tc2_grouped_gemm_kernel(const __grid_constant__ TcMaps maps, const Tc2Params p) {
  static_assert(!SWAP || EPI == tc::EPI_SCALE_TC, "swapped operands: the down GEMM");
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = tc::smem_addr(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int32_t* s_ts = reinterpret_cast<int32_t*>(smem + STAGES * STAGE_BYTES + BAR_BYTES);
  int32_t* s_ps = s_ts + (tc::MAX_E + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const uint32_t stage0 = tc::smem_addr(smem);
  const uint32_t bar0 = tc::smem_addr(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + 2 + a); };
  const uint32_t done_bar = bar0 + 8u * (2 * STAGES + 4);
  const uint32_t peer_abort = mapa_shared(tc::smem_addr(const_cast<int*>(abort_flag)), rank ^ 1u);

  const Tc2Group& G0 = p.g[0];
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      tc::mbar_init(full_bar(s), 1);
      tc::mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      tc::mbar_init(tfull_bar(a), 1);
      tc::mbar_init(tempty_bar(a), 2 * EPI_WARPS);  // the epilogue warps of both CTAs
    }
    tc::mbar_init(done_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    tmem_alloc_pair(tc::smem_addr(tmem_slot), TMEM_COLS);
    tmem_relinquish_pair();
  }
  pdl_wait();  // the routing results and rows this GEMM reads are complete
  pdl_launch_dependents();
  if (G0.tile_start != nullptr) {
    for (int i = threadIdx.x; i <= G0.E; i += NUM_THREADS) {
      s_ts[i] = G0.tile_start[i];
      s_ps[i] = G0.pair_start[i];
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before either signals the other's
  tc::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const long long pairs0 =
      G0.tile_start != nullptr ? (long long)s_ps[G0.E]
                               : (long long)(((G0.rows + HALF_M - 1) / HALF_M + 1) / 2);
  const long long tiles0 = (long long)G0.n_tiles * pairs0;
  const long long tiles1 =
      p.num_groups > 1
          ? (long long)p.g[1].n_tiles * ((((p.g[1].rows + HALF_M - 1) / HALF_M) + 1) / 2)
          : 0;
  const long long total = tiles0 + tiles1;
  const long long cluster_id = blockIdx.x >> 1;
  const long long num_clusters = gridDim.x >> 1;
  const unsigned long long tmo = p.timeout_ns;
  const unsigned long long drain_tmo = p.drain_timeout_ns;
  bool aborted = false;

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    if (lane == 0) {
      for (int g = 0; g < p.num_groups; ++g) {
        tc::prefetch_map(&maps.a[g]);
        tc::prefetch_map(&maps.b0[g]);
        if (EPI == tc::EPI_SWIGLU_TC) tc::prefetch_map(&maps.b1[g]);
      }
      int stage = 0;
      uint32_t phase = 0, issued = 0, last_par = 0;
      bool ok = true;
      for (long long tile = cluster_id; ok && tile < total; tile += num_clusters) {
        const PairTile ti = decode_pair(tile, tiles0, p, s_ts, s_ps);
        if (pair_out_of_bounds(ti, p.g[ti.g])) {
          flag_bounds();
          continue;
        }
        const int kbs = p.g[ti.g].k_blocks;
        const int arow = ti.row0 + HALF_M * (int)rank;
        // SWAP: this CTA's half of the token tile starts N / 2 rows in for the peer
        const int brow = SWAP ? ti.row0 + ((pair_rows(ti, p.g[ti.g], s_ts) + 15) & ~15) / 2 *
                                              (int)rank
                              : 0;
        for (int kb = 0; kb < kbs; ++kb) {
          if (!wait_pair_fast(empty_bar(stage), phase ^ 1u, abort_flag, peer_abort, tmo)) {
            ok = false;
            break;
          }
          const uint32_t sa = stage0 + stage * STAGE_BYTES;
          const uint32_t sb = sa + A_BYTES;
          const uint32_t fb_leader = mapa_shared(full_bar(stage), 0u);
          if (leader) tc::mbar_expect_tx(full_bar(stage), 2 * STAGE_BYTES);
          if constexpr (SWAP) {
            tma_load_3d_pair(sa, &maps.a[ti.g], fb_leader, kb * BK, ti.nb * BN + 128 * (int)rank,
                             ti.e);
            tma_load_2d_pair(sb, &maps.b0[ti.g], fb_leader, kb * BK, brow);
          } else if (EPI == tc::EPI_SWIGLU_TC) {
            tma_load_2d_pair(sa, &maps.a[ti.g], fb_leader, kb * BK, arow);
            tma_load_3d_pair(sb, leader ? &maps.b0[ti.g] : &maps.b1[ti.g], fb_leader, kb * BK,
                             ti.nb * (BN / 2), ti.e);
          } else {
            tma_load_2d_pair(sa, &maps.a[ti.g], fb_leader, kb * BK, arow);
            tma_load_3d_pair(sb, &maps.b0[ti.g], fb_leader, kb * BK,
                             ti.nb * BN + 128 * (int)rank, ti.e);
          }
          issued |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        aborted = true;
        if (leader)  // phases the leader armed complete once both CTAs' bytes land
          for (int s = 0; s < STAGES; ++s)
            if ((issued >> s) & 1u)
              tc::wait_drain(full_bar(s), (last_par >> s) & 1u, abort_flag, drain_tmo);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader)
    if (lane == 0 && leader) {
      constexpr uint32_t IDESC = tc::make_idesc(2 * HALF_M, BN);
      int stage = 0;
      uint32_t phase = 0, acc = 0, acc_phase = 0;
      bool ok = true;
      for (long long tile = cluster_id; ok && tile < total; tile += num_clusters) {
        const PairTile ti = decode_pair(tile, tiles0, p, s_ts, s_ps);
        if (pair_out_of_bounds(ti, p.g[ti.g])) continue;
        const int kbs = p.g[ti.g].k_blocks;
        const uint32_t idesc =
            SWAP ? tc::make_idesc(2 * HALF_M, (pair_rows(ti, p.g[ti.g], s_ts) + 15) & ~15) : IDESC;
        if (!wait_pair(tempty_bar(acc), acc_phase ^ 1u, abort_flag, peer_abort, tmo)) {
          ok = false;
          break;
        }
        tc::tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < kbs; ++kb) {
          if (!wait_pair_fast(full_bar(stage), phase, abort_flag, peer_abort, tmo)) {
            ok = false;
            break;
          }
          tc::tc_fence_after();
          const uint32_t sa = stage0 + stage * STAGE_BYTES;
          const uint64_t ad = tc::sw128_kmajor_desc(sa);
          const uint64_t bd = tc::sw128_kmajor_desc(sa + A_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / UMMA_K; ++kk)
            tc_mma_pair(d_tmem, ad + 2u * kk, bd + 2u * kk, idesc, (kb | kk) != 0 ? 1u : 0u);
          tc_commit_pair_mc(empty_bar(stage), 0x3);  // frees the stage in both CTAs
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit_pair_mc(tfull_bar(acc), 0x3);
        acc ^= 1u;
        if (acc == 0u) acc_phase ^= 1u;
      }
      if (!ok) aborted = true;
      tc_commit_pair(done_bar);
      tc::wait_drain(done_bar, 0u, abort_flag, drain_tmo);
    }
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int quad = warp & 3;
    const int half = warp >= 6 ? 1 : 0;
    const int r_in_half = quad * 32 + lane;
    uint32_t acc = 0, acc_phase = 0;
    for (long long tile = cluster_id; tile < total; tile += num_clusters) {
      const PairTile ti = decode_pair(tile, tiles0, p, s_ts, s_ps);
      const Tc2Group& g = p.g[ti.g];
      if (pair_out_of_bounds(ti, g)) continue;
      int ok = 1;
      if (lane == 0)
        ok = wait_pair(tfull_bar(acc), acc_phase, abort_flag, peer_abort, tmo) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) {
        aborted = true;
        break;
      }
      tc::tc_fence_after();
      if constexpr (SWAP) {
        // lane = this CTA's weight row (output column), columns = the tile's tokens
        const int v = pair_rows(ti, g, s_ts);
        const int col = ti.nb * BN + 128 * (int)rank + r_in_half;
        const uint32_t tb = tmem_base + acc * BN + (static_cast<uint32_t>(quad * 32) << 16);
        __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(g.out);
#pragma unroll 1
        for (int c = half; c * 32 < v; c += 2) {
          float d[32];
          __syncwarp();
          tc::tmem_ld32(tb + c * 32, d);
          const int c0 = c * 32;
          // the 32 tokens' gate scales: one load, broadcast at a warp-uniform point
          const float rs = (g.row_scale != nullptr && c0 + lane < v)
                               ? g.row_scale[ti.row0 + c0 + lane] : 1.f;
#pragma unroll
          for (int cc = 0; cc < 32; ++cc) {
            const float sc = __shfl_sync(0xffffffffu, rs, cc);
            if (c0 + cc < v && col < g.N)
              out[(size_t)(ti.row0 + c0 + cc) * g.N + col] = __float2bfloat16_rn(sc * d[cc]);
          }
        }
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(mapa_shared(tempty_bar(acc), 0u));
        acc ^= 1u;
        if (acc == 0u) acc_phase ^= 1u;
        continue;
      }
      const int row = ti.row0 + HALF_M * (int)rank + r_in_half;
      const bool row_ok =
          ti.half_valid[rank] && ((g.tile_start != nullptr) || row < g.rows);
      const uint32_t tb = tmem_base + acc * BN + (static_cast<uint32_t>(quad * 32) << 16);
      __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(g.out) + (size_t)row * g.N;
      if (EPI == tc::EPI_SWIGLU_TC) {
#pragma unroll 1
        for (int c = half; c < (BN / 2) / 32; c += 2) {
          float gv[32], uv[32];
          __syncwarp();
          tc::tmem_ld32(tb + c * 32, gv);
          tc::tmem_ld32(tb + BN / 2 + c * 32, uv);
          const int col0 = ti.nb * (BN / 2) + c * 32;
          if (row_ok && col0 < g.N) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              float h[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) h[i] = silu_f32(gv[q * 8 + i]) * uv[q * 8 + i];
              st_v4(out + col0 + q * 8, Vec16<__nv_bfloat16>::pack(h));
            }
          }
        }
      } else {
        const float sc = (row_ok && g.row_scale != nullptr) ? g.row_scale[row] : 1.f;
#pragma unroll 1
        for (int c = half; c < BN / 32; c += 2) {
          float v[32];
          __syncwarp();
          tc::tmem_ld32(tb + c * 32, v);
          const int col0 = ti.nb * BN + c * 32;
          if (row_ok && col0 < g.N) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              float h[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) h[i] = sc * v[q * 8 + i];
              st_v4(out + col0 + q * 8, Vec16<__nv_bfloat16>::pack(h));
            }
          }
        }
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(tempty_bar(acc), 0u));
      acc ^= 1u;
      if (acc == 0u) acc_phase ^= 1u;
    }
  }

  // On an abort, copies issued by one CTA may still be landing in its shared
  // memory and on the leader's barriers: give them time before either CTA
  // releases its shared memory.
  if (aborted || *abort_flag) {
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < ABORT_SETTLE_NS) {
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  cluster_sync();  // the leader's MMAs into this CTA's TMEM have completed
  tc::tc_fence_after();
  tc::record_call_status(abort_flag, p.call_err);
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

}  // namespace tc2
}  // namespace moe
