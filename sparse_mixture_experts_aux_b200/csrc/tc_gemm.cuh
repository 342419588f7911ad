// Grouped expert GEMMs on the 5th-generation tensor cores (sm_100a):
// TMA (cp.async.bulk.tensor, 128-byte swizzle) -> shared-memory ring ->
// single-thread tcgen05.mma (bf16 x bf16, or E4M3 x E4M3, -> fp32 in TMEM) -> tcgen05.ld
// epilogue. Persistent: one CTA per SM walks a static tile list that it
// derives on the device from the per-expert segment starts, so no host
// synchronisation sits between routing and the expert products.
//
// Two epilogues:
//   SwiGLU (gate/up projection): each 256-column accumulator tile holds 128
//     gate columns (x W_g) followed by the matching 128 up columns (x W_u);
//     the epilogue writes H = SiLU(gate) * up as bf16 (fp32 with E4M3
//     operands, for the per-row quantiser of H that follows).
//   Scale (down projection): Yrows = g_row * (H W_d) as bf16, g_row the gate
//     of the assignment that owns the row (1 for the shared expert).
// Sources: Zero to Frontier 13.1 "Why MoE", "The MoE layer" (SwiGLU experts,
// FFN_i(x) = (SiLU(x W_g) * x W_u) W_d) and "In PyTorch" (a grouped matrix
// multiply replaces the loop over experts).
//
// Warp roles (352 threads): warps 0 and 6 = TMA producers (alternate K steps),
// warp 1 = TMEM owner and MMA issuer, warps 2..5 and 7..10 = epilogue (warp w
// reads TMEM lanes 32*(w%4)..+31; the two warps of a quadrant split its column
// chunks).
// With Q8 (E4M3 operands, tcgen05 kind::f8f6f4) the same pipeline runs on code
// tiles, 128 codes per K step, and the epilogue applies the operands' row scales.
// TMEM holds two 128x256 fp32 accumulators (512 columns), so the epilogue of
// one tile overlaps the main loop of the next.
// Every mbarrier wait is bounded: on expiry the kernel records
// DEVERR_TIMEOUT, tells the other roles to stop, waits (bounded) for its own
// copies and MMAs in flight, frees TMEM and returns.
#pragma once
#include "common.cuh"
#include <cuda.h>

namespace moe {
namespace tc {

constexpr int BM = 128;            // rows per tile (= ROW_TILE)
constexpr int BN = 256;            // accumulator columns per tile (UMMA N)
constexpr int BK = 64;             // K per stage: one 128-byte swizzle row of bf16
constexpr int UMMA_K = 16;         // K of one tcgen05.mma kind::f16
constexpr int B_BYTES = BN * BK * 2;
// warp 0 producer, 1 MMA, 2-5 epilogue (first half of the columns), 6 second
// producer, 7-10 epilogue (second half)
constexpr int NUM_THREADS = 352;
constexpr int PROD2_WARP = 6;
constexpr int EPI_WARPS = 8;
constexpr uint32_t TMEM_COLS = 512;
constexpr int MAX_E = 1024;
constexpr int BAR_BYTES = 256;

static_assert(BM == ROW_TILE, "GEMM row tile must match the segment padding");

// Shape of the 1-CTA kernel for an activation box of AR rows. AR = 128 is the
// general case. When every expert holds at most 32 (64) rows, which holds for
// any batch of at most that many tokens, the box shrinks to AR rows, so a
// stage is smaller and the ring deeper: more weight bytes in flight for the
// weight-streaming (decode) shapes. The M = 128 MMA still reads 128 rows from
// the A slot. The rows past AR are stale bytes inside the same stage buffer;
// their results land only in the padding rows of the expert's 128-row segment,
// and the epilogue warps that own them skip their stores.
template <int AR>
struct TcShape {
  static_assert(AR == 128 || AR == 64 || AR == 32, "activation box rows");
  static constexpr int A_BYTES = AR * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = AR == 128 ? 4 : (AR == 64 ? 5 : 6);
  static constexpr int SMEM_BYTES =
      1024 + STAGES * STAGE_BYTES + BAR_BYTES + 4 * (MAX_E + 1);
  static_assert(SMEM_BYTES <= 232448, "shared memory per block");
  static_assert(A_BYTES % 1024 == 0, "B slot must stay 1024-byte aligned");
};

enum { EPI_SWIGLU_TC = 0, EPI_SCALE_TC = 1 };

struct TcGroup {
  const int32_t* tile_start;  // routed rows: [E + 1] segment starts in BM-row tiles; NULL = dense
  int E;
  int rows;                   // dense groups: valid rows; routed groups: rows of the permuted
                              // buffers (the bounds checks of MOE_DEBUG builds)
  int n_tiles;                // output tiles per expert along N
  int k_blocks;               // K / BK
  int N;                      // output columns
  void* out;                  // bf16 [rows, N]
  const float* row_scale;     // scale epilogue: factor per row; NULL = 1
  // E4M3 operands (Q8 kernels only): A row scales, B row scales of the
  // output columns (gate/up: b_scale0 gate, b_scale1 up), floats per expert
  const float* a_scale;
  const float* b_scale0;
  const float* b_scale1;
  int64_t b_scale_stride;
  // Routed groups of the swapped-operand kernel (tc_ws_gemm.cuh): assignments
  // per expert and the capacity (-1: none), which give each tile's valid rows
  const int32_t* counts;
  int64_t cap;
};

struct TcParams {
  TcGroup g[2];
  int num_groups;
  unsigned long long timeout_ns;        // limit of each pipeline wait
  unsigned long long drain_timeout_ns;  // limit of the teardown waits for work in flight
  int* call_err;                        // the call's own status word (NULL: none)
};

struct TcMaps {
  CUtensorMap a[2];   // activations [rows, K], box {BK, BM}
  CUtensorMap b0[2];  // weights [E][N][K]: box {BK, BN} (scale) or {BK, BN/2} (gate)
  CUtensorMap b1[2];  // SwiGLU up weights, box {BK, BN/2}
};

// ----------------------------------------------------------------------------
// PTX wrappers (PTX ISA: mbarrier, cp.async.bulk.tensor, tcgen05).
// ----------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0u;
}

// Wait until the phase with `parity` of barrier `bar` has completed. Gives up
// (returns false) when another role has aborted, or after timeout_ns, in which
// case it records the timeout and raises the abort flag itself.
__device__ __noinline__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          unsigned long long timeout_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t limit = wait_cycles(timeout_ns);
  const long long t0 = clock64();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    // try_wait itself suspends for a while, so check on the first re-poll too
    if ((it & 15u) == 1u) {
      if (*abort_flag) return false;
      if (static_cast<uint64_t>(clock64() - t0) > limit) {
        atomicOr(&g_dev_error, DEVERR_TIMEOUT);
        *abort_flag = 1;
        return false;
      }
    }
  }
}

// The same with the first test inline: a phase that has already completed
// costs one try_wait instead of a call (the bounded loop stays out of line).
__device__ __forceinline__ bool wait_fast(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          unsigned long long timeout_ns) {
  return mbar_try_wait(bar, parity) || wait_bounded(bar, parity, abort_flag, timeout_ns);
}

// Same, not stopping on the abort flag (it raises it when it gives up): used
// only in teardown, to let copies and MMAs already in flight land before
// shared memory and TMEM are released.
__device__ __noinline__ bool wait_drain(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                        unsigned long long timeout_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t limit = wait_cycles(timeout_ns);
  const long long t0 = clock64();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 15u) == 1u && static_cast<uint64_t>(clock64() - t0) > limit) {
      atomicOr(&g_dev_error, DEVERR_TIMEOUT);
      *abort_flag = 1;
      return false;
    }
  }
}

// After the CTA's roles have finished: a CTA that gave up anywhere records it
// in the call's own status word as well.
__device__ __forceinline__ void record_call_status(volatile int* abort_flag, int* call_err) {
  if (threadIdx.x == 0 && call_err != nullptr && *abort_flag) atomicOr(call_err, DEVERR_TIMEOUT);
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void prefetch_map(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Arrive once on `bar` when every tcgen05 operation this thread issued so far has completed.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}
// D[tmem] (+)= A[smem] * B[smem]^T, both K-major; accumulate when `accum` != 0.
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum)
      : "memory");
}

// The same with E4M3 operands (kind::f8f6f4): 32 codes of K per instruction,
// so a 128-byte shared-memory row is 128 codes and the descriptors advance
// exactly as for bf16 (+32 bytes per instruction).
__device__ __forceinline__ void tc_mma_e4m3(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum)
      : "memory");
}

// Load 32 consecutive fp32 columns of this warp's 32 TMEM lanes (one row per
// thread) and wait for them in the same asm block, so that no use of the
// registers can be scheduled before the wait.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* f) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) f[i] = __uint_as_float(r[i]);
}

// Shared-memory matrix descriptor (tcgen05 format) for a K-major bf16 tile
// written by TMA with 128-byte swizzle: rows of 128 bytes, 8-row groups 1024
// bytes apart (stride byte offset), leading byte offset unused (1), version 1
// (bits 46-47), layout SWIZZLE_128B (2 in bits 61-63). The tile base must be
// 1024-byte aligned; a K step of 16 elements inside the swizzle row advances
// the start address by 32 bytes.
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t saddr) {
  return static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4) | (static_cast<uint64_t>(1) << 16) |
         (static_cast<uint64_t>(1024 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) |
         (static_cast<uint64_t>(2) << 61);
}

// Instruction descriptor, kind::f16: D fp32 (bits 4-5 = 1), A and B bf16
// (bits 7-9 = 1, bits 10-12 = 1), both K-major (bits 15, 16 = 0),
// N >> 3 in bits 17-22, M >> 4 in bits 24-28.
__host__ __device__ constexpr uint32_t make_idesc(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}
// kind::f8f6f4 with A and B E4M3 (format 0), D fp32, both K-major.
__host__ __device__ constexpr uint32_t make_idesc_e4m3(int M, int N) {
  return (1u << 4) | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

struct TileInfo {
  int g, e, row0, nb;
};

// Tile order: group 0 then group 1. Within a routed group, expert by expert;
// within an expert, n-tile-major with the m-tiles fastest, so CTAs running at
// the same time share weight tiles through L2.
__device__ __forceinline__ TileInfo decode_tile(long long tile, long long tiles0,
                                                const TcParams& p, const int32_t* s_ts) {
  TileInfo ti;
  const TcGroup* g;
  long long local = tile;
  if (tile < tiles0) {
    ti.g = 0;
    g = &p.g[0];
  } else {
    ti.g = 1;
    g = &p.g[1];
    local = tile - tiles0;
  }
  if (ti.g == 0 && g->tile_start != nullptr) {
    const long long q = local / g->n_tiles;
    int lo = 0, hi = g->E - 1;  // last expert whose first tile is at or before q
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_ts[mid] <= q) lo = mid; else hi = mid - 1;
    }
    const int me = s_ts[lo + 1] - s_ts[lo];
    const long long in_e = local - (long long)g->n_tiles * s_ts[lo];
    ti.e = lo;
    ti.nb = (int)(in_e / me);
    ti.row0 = (s_ts[lo] + (int)(in_e % me)) * BM;
  } else {
    const int mt = (g->rows + BM - 1) / BM;
    ti.e = 0;
    ti.nb = (int)(local / mt);
    ti.row0 = (int)(local % mt) * BM;
  }
  return ti;
}

// Builds with MOE_DEBUG: true when a tile's expert, N block or rows fall outside
// what its tensor maps and stores cover (routed groups: the whole 128-row tile
// inside the group's `rows` permuted rows; dense groups: its first row inside).
// Every role of a kernel skips such a tile, so the pipeline stays in step, and
// one producer records it in the device error word. Release builds: false.
__device__ __forceinline__ bool tile_out_of_bounds(int e, int nb, int row0, int span,
                                                   const TcGroup& g) {
#if defined(MOE_DEBUG)
  if (nb < 0 || nb >= g.n_tiles || row0 < 0) return true;
  if (g.tile_start != nullptr) return e < 0 || e >= g.E || row0 + span > g.rows;
  return row0 >= g.rows;
#else
  (void)e; (void)nb; (void)row0; (void)span; (void)g;
  return false;
#endif
}

// Q8: A and B are E4M3 codes (tensor maps over 16-bit elements, 2 codes each,
// so a K step is the same 128-byte line as in bf16: 128 codes), and the
// epilogue multiplies each accumulator by the A row's and the B column's
// scales before its own arithmetic.
template <int EPI, int AR, bool Q8 = false>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    tc_grouped_gemm_kernel(const __grid_constant__ TcMaps maps, const TcParams p) {
  constexpr int KX = BK;  // TMA x-coordinate units (16-bit elements) per K step
  constexpr int STAGES = TcShape<AR>::STAGES;
  constexpr int A_BYTES = TcShape<AR>::A_BYTES;
  constexpr int STAGE_BYTES = TcShape<AR>::STAGE_BYTES;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_addr(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  // bars: full[STAGES], empty[STAGES], tfull[2], tempty[2], done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int32_t* s_ts = reinterpret_cast<int32_t*>(smem + STAGES * STAGE_BYTES + BAR_BYTES);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t stage0 = smem_addr(smem);
  const uint32_t bar0 = smem_addr(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + 2 + a); };
  const uint32_t done_bar = bar0 + 8u * (2 * STAGES + 4);

  const TcGroup& G0 = p.g[0];
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), EPI_WARPS);  // one arrival per epilogue warp
    }
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  pdl_wait();  // the routing results and rows this GEMM reads are complete
  pdl_launch_dependents();
  if (G0.tile_start != nullptr)
    for (int i = threadIdx.x; i <= G0.E; i += NUM_THREADS) s_ts[i] = G0.tile_start[i];
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
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
    // Two producer threads take alternate K steps of the same walk (the step's
    // stage is its running index modulo STAGES), so each thread's serial chain
    // of wait, expect_tx and copies covers only every other stage.
    if (lane == 0) {
      const uint32_t me = warp == 0 ? 0u : 1u;
      for (int g = 0; g < p.num_groups; ++g) {
        prefetch_map(&maps.a[g]);
        prefetch_map(&maps.b0[g]);
        if (EPI == EPI_SWIGLU_TC) prefetch_map(&maps.b1[g]);
      }
      uint32_t issued = 0, last_par = 0;
      long long gs = 0;  // running K-step index over this CTA's tiles
      bool ok = true;
      for (long long tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
        const TileInfo ti = decode_tile(tile, tiles0, p, s_ts);
        if (tile_out_of_bounds(ti.e, ti.nb, ti.row0, BM, p.g[ti.g])) {
          if (me == 0) flag_bounds();
          continue;
        }
        const int kbs = p.g[ti.g].k_blocks;
        for (int kb = 0; kb < kbs; ++kb, ++gs) {
          if ((uint32_t)(gs & 1) != me) continue;
          const int stage = (int)(gs % STAGES);
          const uint32_t phase = (uint32_t)((gs / STAGES) & 1);
          if (!wait_fast(empty_bar(stage), phase ^ 1u, abort_flag, tmo)) { ok = false; break; }
          const uint32_t sa = stage0 + stage * STAGE_BYTES;
          const uint32_t sb = sa + A_BYTES;
          const uint32_t fb = full_bar(stage);
          mbar_expect_tx(fb, STAGE_BYTES);
          tma_load_2d(sa, &maps.a[ti.g], fb, kb * KX, ti.row0);
          if (EPI == EPI_SWIGLU_TC) {
            tma_load_3d(sb, &maps.b0[ti.g], fb, kb * KX, ti.nb * (BN / 2), ti.e);
            tma_load_3d(sb + B_BYTES / 2, &maps.b1[ti.g], fb, kb * KX, ti.nb * (BN / 2), ti.e);
          } else {
            tma_load_3d(sb, &maps.b0[ti.g], fb, kb * KX, ti.nb * BN, ti.e);
          }
          issued |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
        }
      }
      if (!ok) {  // let every copy this thread issued land before the CTA exits
        for (int s = 0; s < STAGES; ++s)
          if ((issued >> s) & 1u)
            wait_drain(full_bar(s), (last_par >> s) & 1u, abort_flag, drain_tmo);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC = Q8 ? make_idesc_e4m3(BM, BN) : make_idesc(BM, BN);
      int stage = 0;
      uint32_t phase = 0, acc = 0, acc_phase = 0;
      bool ok = true;
      for (long long tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
        const TileInfo ti = decode_tile(tile, tiles0, p, s_ts);
        if (tile_out_of_bounds(ti.e, ti.nb, ti.row0, BM, p.g[ti.g])) continue;
        const int kbs = p.g[ti.g].k_blocks;
        if (!wait_bounded(tempty_bar(acc), acc_phase ^ 1u, abort_flag, tmo)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < kbs; ++kb) {
          if (!wait_fast(full_bar(stage), phase, abort_flag, tmo)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = stage0 + stage * STAGE_BYTES;
          const uint64_t ad = sw128_kmajor_desc(sa);
          const uint64_t bd = sw128_kmajor_desc(sa + A_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / UMMA_K; ++kk) {
            // +32 bytes per K step = +2 in the descriptor's address field
            if (Q8)
              tc_mma_e4m3(d_tmem, ad + 2u * kk, bd + 2u * kk, IDESC, (kb | kk) != 0 ? 1u : 0u);
            else
              tc_mma(d_tmem, ad + 2u * kk, bd + 2u * kk, IDESC, (kb | kk) != 0 ? 1u : 0u);
          }
          tc_commit(empty_bar(stage));  // frees the stage once these MMAs have read it
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit(tfull_bar(acc));  // accumulator ready for the epilogue
        acc ^= 1u;
        if (acc == 0u) acc_phase ^= 1u;
      }
      tc_commit(done_bar);  // every MMA issued above has completed once this fires
      wait_drain(done_bar, 0u, abort_flag, drain_tmo);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Two warps per TMEM lane quadrant, each taking every other 32-column chunk
    const int quad = warp & 3;  // TMEM lanes 32*quad .. 32*quad+31
    const int half = warp >= 7 ? 1 : 0;
    const int r_in_tile = quad * 32 + lane;
    uint32_t acc = 0, acc_phase = 0;
    for (long long tile = blockIdx.x; tile < total; tile += gridDim.x) {
      const TileInfo ti = decode_tile(tile, tiles0, p, s_ts);
      const TcGroup& g = p.g[ti.g];
      if (tile_out_of_bounds(ti.e, ti.nb, ti.row0, BM, g)) continue;
      int ok = 1;
      if (lane == 0) ok = wait_bounded(tfull_bar(acc), acc_phase, abort_flag, tmo) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);  // whole warp converged and agreed
      if (!ok) break;
      tc_fence_after();
      const int row = ti.row0 + r_in_tile;
      const bool row_ok = (g.tile_start != nullptr) || row < g.rows;
      const uint32_t tb = tmem_base + acc * BN + (static_cast<uint32_t>(quad * 32) << 16);
      if (quad * 32 < AR) {
      __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(g.out) + (size_t)row * g.N;
      // E4M3 operands: the A row's scale, and the B scales of this expert
      const float ars = (Q8 && row_ok) ? g.a_scale[row] : 1.f;
      const float* bs0 = Q8 ? g.b_scale0 + (int64_t)ti.e * g.b_scale_stride : nullptr;
      const float* bs1 = Q8 ? g.b_scale1 + (int64_t)ti.e * g.b_scale_stride : nullptr;
      if (EPI == EPI_SWIGLU_TC) {
#pragma unroll 1
        for (int c = half; c < (BN / 2) / 32; c += 2) {
          float gv[32], uv[32];
          __syncwarp();  // tcgen05.ld is warp-collective: reconverge after the stores
          tmem_ld32(tb + c * 32, gv);
          tmem_ld32(tb + BN / 2 + c * 32, uv);
          const int col0 = ti.nb * (BN / 2) + c * 32;
          if (row_ok && col0 < g.N) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              float h[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                float a = gv[q * 8 + i], b = uv[q * 8 + i];
                if (Q8) {
                  const int col = col0 + q * 8 + i;
                  a *= ars * bs0[col];
                  b *= ars * bs1[col];
                }
                h[i] = silu_f32(a) * b;
              }
              if (Q8) {
                // E4M3 operands: H stays fp32, so that the per-row quantiser that
                // follows decides its codes from H itself, not from a bf16 copy
                float* o32 = reinterpret_cast<float*>(g.out) + (size_t)row * g.N + col0 + q * 8;
                st_v4(o32, Vec16<float>::pack(h));
                st_v4(o32 + 4, Vec16<float>::pack(h + 4));
              } else {
                st_v4(out + col0 + q * 8, Vec16<__nv_bfloat16>::pack(h));
              }
            }
          }
        }
      } else {
        const float sc = ((row_ok && g.row_scale != nullptr) ? g.row_scale[row] : 1.f) * ars;
#pragma unroll 1
        for (int c = half; c < BN / 32; c += 2) {
          float v[32];
          __syncwarp();  // tcgen05.ld is warp-collective: reconverge after the stores
          tmem_ld32(tb + c * 32, v);
          const int col0 = ti.nb * BN + c * 32;
          if (row_ok && col0 < g.N) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              float h[8];
#pragma unroll
              for (int i = 0; i < 8; ++i)
                h[i] = Q8 ? sc * (v[q * 8 + i] * bs0[col0 + q * 8 + i]) : sc * v[q * 8 + i];
              st_v4(out + col0 + q * 8, Vec16<__nv_bfloat16>::pack(h));
            }
          }
        }
      }
      }  // quad * 32 < AR
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty_bar(acc));
      acc ^= 1u;
      if (acc == 0u) acc_phase ^= 1u;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  record_call_status(abort_flag, p.call_err);
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace tc
}  // namespace moe
