// Router logits r = x W_r on the 5th-generation tensor cores, keeping fp32
// accuracy, for bf16 activations.
//
// The pages fix the router at float32 (AI Engineering Illustrated "Mixture of
// Experts", "The router is small but it decides everything"). x is exactly
// bf16, and W_r (fp32) is split exactly into three bf16 terms, W_r = hi + mid
// + lo (hi = bf16(W_r), mid = bf16(W_r - hi), lo = W_r - hi - mid, which has
// at most 8 significant bits and is therefore a bf16 value). Every product
// x_j * term is exact in fp32, so the tensor cores (bf16 x bf16 -> fp32) see
// the same products an fp32 FMA would, and only the summation differs: the
// MMAs accumulate one 128-deep K chunk at a time into a fresh TMEM
// accumulator, and the epilogue adds the chunks in fp32 on the CUDA cores, in
// a fixed order. This is the split-precision technique of Markidis et al.
// (2018) and Ootomo and Yokota (2022), with the third term making the split
// exact for fp32.
//
// Tile: 128 tokens x N experts (N = E rounded up to 16, at most 128) over one
// K range (grid.z splits K; the routing kernel sums the split partials in a
// fixed order). Stage: the x box (128 x 64 bf16) and the three terms' boxes
// (N x 64 each), all TMA with the 128-byte swizzle; as many stages as fit
// (3 at N = 128, 8 at small N). Warp 0 = TMA producer,
// warp 1 = TMEM owner and MMA issuer, warps 2..9 = epilogue (two per TMEM lane
// quadrant, each summing half of the N columns in registers). TMEM holds two
// 128 x N accumulators, so one chunk is summed while the next is computed.
// Every wait is bounded as in the expert GEMMs.
#pragma once
#include "tc_gemm.cuh"

namespace moe {
namespace rtc {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int MAX_N = 128;
constexpr int KC = 2;  // K blocks (64 deep) per accumulation chunk
constexpr int MAX_STAGES = 8;
constexpr int NUM_THREADS = 320;
constexpr int EPI_WARPS = 8;
constexpr int A_BYTES = BM * BK * 2;
constexpr int BAR_BYTES = 256;
constexpr int SMEM_LIMIT = 232448;
constexpr uint32_t TMEM_COLS = 256;  // two accumulators of up to 128 columns
static_assert(A_BYTES % 1024 == 0, "1024-byte aligned boxes");

// Stage geometry for tiles of N experts: the x box and the three terms' N-row
// boxes, as many stages as fit (at most MAX_STAGES): 3 at N = 128, 8 at N = 16.
__host__ __device__ constexpr int stage_bytes(int N) { return A_BYTES + 3 * N * BK * 2; }
__host__ __device__ constexpr int stages_for(int N) {
  return (SMEM_LIMIT - 1024 - BAR_BYTES) / stage_bytes(N) < MAX_STAGES
             ? (SMEM_LIMIT - 1024 - BAR_BYTES) / stage_bytes(N)
             : MAX_STAGES;
}
__host__ __device__ constexpr int smem_bytes(int N) {
  return 1024 + stages_for(N) * stage_bytes(N) + BAR_BYTES;
}
static_assert(smem_bytes(MAX_N) <= SMEM_LIMIT && smem_bytes(16) <= SMEM_LIMIT, "shared memory");
static_assert(stages_for(MAX_N) >= 2, "at least double buffering");

struct RtcParams {
  int T, E, N;          // tokens, experts, columns of one tile (multiple of 16, <= MAX_N)
  int k_blocks;         // 64-deep K blocks of each split
  float* logits;        // fp32 [splits][T][E]
  unsigned long long timeout_ns, drain_timeout_ns;
  int* call_err;
};


struct RtcMaps {
  CUtensorMap x;  // bf16 [T][d], box {64, 128}
  CUtensorMap w;  // bf16 [3][E][d], box {64, N, 1}
};

// hi / mid / lo bf16 terms of fp32 router weights, [3][n] (see the top of the file).
__global__ void __launch_bounds__(256) split_router_weights_kernel(const float* __restrict__ w,
                                                                   int64_t n,
                                                                   __nv_bfloat16* __restrict__ out) {
  pdl_wait();
  pdl_launch_dependents();
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const float v = w[i];
    const __nv_bfloat16 hi = __float2bfloat16_rn(v);
    const float r1 = v - __bfloat162float(hi);  // exact
    const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
    const float r2 = r1 - __bfloat162float(mid);  // exact, at most 8 significant bits
    out[i] = hi;
    out[n + i] = mid;
    out[2 * n + i] = __float2bfloat16_rn(r2);  // exact
  }
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
    router_tc_kernel(const __grid_constant__ RtcMaps maps, const RtcParams p) {
  extern __shared__ uint8_t smem_raw[];
  const int STAGES = stages_for(p.N);
  const int STAGE_BYTES = stage_bytes(p.N);
  const uint32_t b_bytes = (uint32_t)p.N * BK * 2;  // one term's box
  const uint32_t raw_addr = tc::smem_addr(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  // bars: full[STAGES], empty[STAGES], tfull[2], tempty[2], done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t stage0 = tc::smem_addr(smem);
  const uint32_t bar0 = tc::smem_addr(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + 2 + a); };
  const uint32_t done_bar = bar0 + 8u * (2 * STAGES + 4);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      tc::mbar_init(full_bar(s), 1);
      tc::mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      tc::mbar_init(tfull_bar(a), 1);
      tc::mbar_init(tempty_bar(a), EPI_WARPS);
    }
    tc::mbar_init(done_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    tc::tmem_alloc(tc::smem_addr(tmem_slot), TMEM_COLS);
    tc::tmem_relinquish();
  }
  pdl_wait();
  pdl_launch_dependents();
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int m0 = blockIdx.x * BM;
  const int n0 = blockIdx.y * p.N;
  const int kb0 = blockIdx.z * p.k_blocks;
  const int nkb = p.k_blocks;
  const int nch = (nkb + KC - 1) / KC;
  const unsigned long long tmo = p.timeout_ns, drain_tmo = p.drain_timeout_ns;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tc::prefetch_map(&maps.x);
      tc::prefetch_map(&maps.w);
      uint32_t issued = 0, last_par = 0;
      bool ok = true;
      for (int kb = 0; kb < nkb; ++kb) {
        const int stage = kb % STAGES;
        const uint32_t phase = (uint32_t)((kb / STAGES) & 1);
        if (!tc::wait_fast(empty_bar(stage), phase ^ 1u, abort_flag, tmo)) { ok = false; break; }
        const uint32_t sa = stage0 + stage * STAGE_BYTES;
        const uint32_t fb = full_bar(stage);
        tc::mbar_expect_tx(fb, A_BYTES + 3 * b_bytes);
        const int kx = (kb0 + kb) * BK;
        tc::tma_load_2d(sa, &maps.x, fb, kx, m0);
#pragma unroll
        for (int t = 0; t < 3; ++t)
          tc::tma_load_3d(sa + A_BYTES + t * b_bytes, &maps.w, fb, kx, n0, t);
        issued |= 1u << stage;
        last_par = (last_par & ~(1u << stage)) | (phase << stage);
      }
      if (!ok)
        for (int s = 0; s < STAGES; ++s)
          if ((issued >> s) & 1u) tc::wait_drain(full_bar(s), (last_par >> s) & 1u, abort_flag, drain_tmo);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = tc::make_idesc(BM, p.N);
      uint32_t acc = 0, acc_phase = 0;
      bool ok = true;
      int kb = 0;
      for (int ch = 0; ok && ch < nch; ++ch) {
        if (!tc::wait_bounded(tempty_bar(acc), acc_phase ^ 1u, abort_flag, tmo)) { ok = false; break; }
        tc::tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * MAX_N;
        const int kend = min(nkb, (ch + 1) * KC);
        for (int first = 1; kb < kend; ++kb, first = 0) {
          const int stage = kb % STAGES;
          if (!tc::wait_fast(full_bar(stage), (uint32_t)((kb / STAGES) & 1), abort_flag, tmo)) {
            ok = false;
            break;
          }
          tc::tc_fence_after();
          const uint32_t sa = stage0 + stage * STAGE_BYTES;
          const uint64_t ad = tc::sw128_kmajor_desc(sa);
          // the smallest term first; a fresh accumulator at the chunk's first MMA
#pragma unroll
          for (int t = 2; t >= 0; --t) {
            const uint64_t bd = tc::sw128_kmajor_desc(sa + A_BYTES + t * b_bytes);
#pragma unroll
            for (int kk = 0; kk < BK / tc::UMMA_K; ++kk)
              tc::tc_mma(d_tmem, ad + 2u * kk, bd + 2u * kk, idesc,
                         (first && t == 2 && kk == 0) ? 0u : 1u);
          }
          tc::tc_commit(empty_bar(stage));
        }
        if (!ok) break;
        tc::tc_commit(tfull_bar(acc));
        acc ^= 1u;
        if (acc == 0u) acc_phase ^= 1u;
      }
      tc::tc_commit(done_bar);
      tc::wait_drain(done_bar, 0u, abort_flag, drain_tmo);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Warp w reads TMEM lanes 32*(w%4).. (its tokens); the two warps of a
    // quadrant take columns [0, N/2) and [N/2, N) of each chunk, and add the
    // chunk to their fp32 sums (chunk order fixed).
    const int quad = warp & 3;
    const int half = warp >= 6 ? 1 : 0;
    const int cols = p.N / 2;  // a multiple of 8
    float sum[MAX_N / 2];
#pragma unroll
    for (int i = 0; i < MAX_N / 2; ++i) sum[i] = 0.f;
    uint32_t acc = 0, acc_phase = 0;
    bool ok = true;
    for (int ch = 0; ch < nch; ++ch) {
      int w = 1;
      if (lane == 0) w = tc::wait_bounded(tfull_bar(acc), acc_phase, abort_flag, tmo) ? 1 : 0;
      if (!__shfl_sync(0xffffffffu, w, 0)) { ok = false; break; }
      tc::tc_fence_after();
      const uint32_t tb = tmem_base + acc * MAX_N + half * cols + (static_cast<uint32_t>(quad * 32) << 16);
#pragma unroll
      for (int c = 0; c < MAX_N / 2; c += 32) {
        if (c < cols) {
          float v[32];
          __syncwarp();
          tc::tmem_ld32(tb + c, v);
#pragma unroll
          for (int i = 0; i < 32; ++i) sum[c + i] += v[i];
        }
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(tempty_bar(acc));
      acc ^= 1u;
      if (acc == 0u) acc_phase ^= 1u;
    }
    const int t = m0 + quad * 32 + lane;
    if (ok && t < p.T) {
      float* out = p.logits + ((size_t)blockIdx.z * p.T + t) * p.E;
      const int e0 = n0 + half * cols;
#pragma unroll
      for (int i = 0; i < MAX_N / 2; ++i)
        if (i < cols && e0 + i < p.E) out[e0 + i] = sum[i];
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

}  // namespace rtc
}  // namespace moe
