// libmoe.so: C ABI of the routed MoE FFN forward pass (include/moe.h).
// Host side: argument checks, workspace layout, TMA descriptors and the launch
// sequence; the kernels live in the included headers (one translation unit).
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <mutex>
#include <utility>
#include <string.h>

#include "moe.h"
#include "common.cuh"
#include "router.cuh"
#include "permute.cuh"
#include "tc_gemm.cuh"
#include "tc2_gemm.cuh"
#include "quant_formats.cuh"
#include "router_tc.cuh"
#include "tc_wq_swap.cuh"
#include "tc_ws_gemm.cuh"

namespace {

using moe::ROW_TILE;

constexpr size_t ALIGN = 1024;
constexpr unsigned long long kWaitTimeoutNs = 4000000000ull;   // 4 s per mbarrier wait
constexpr unsigned long long kDrainTimeoutNs = 2000000000ull;  // teardown waits
// bf16 layers with more than 64 tokens and at most this many routed rows per
// expert (T k / E) run the swapped-operand GEMMs (tc_ws_gemm.cuh)
constexpr int64_t kWsUpMaxRowsPerExpert = 2048;   // gate/up
constexpr int64_t kWsDownMaxRowsPerExpert = 512;  // down
// above that, the down GEMM runs on CTA pairs, with the operands swapped
constexpr bool kPairDownSwap = true;

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }
bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

struct Plan {
  int64_t T;
  int d, de, ds, E, k;
  bool bf16;
  size_t esz;
  int64_t C;  // -1: no limit
  int nblk;   // routing chunks
  int router_split;    // K chunks of the router product
  bool router_narrow;  // few experts, many tokens: warp-per-token-group router kernel
  bool router_tc;      // bf16 x: split-precision tensor-core router
  int router_n;        // tensor-core router: experts per tile
  int64_t rows_max;
  size_t o_logits, o_idx, o_gate, o_lrank, o_slot, o_hist, o_base, o_psum_part, o_probsum,
      o_tile_start, o_pair_start, o_status, o_wsplit, o_rowgate, o_xp, o_h, o_yrows, o_hs, o_ys,
      // E4M3 activations (MOE_WEIGHTS_FP8_W8A8): x codes and scales per token,
      // scales of the permuted x rows, H codes and scales per permuted row
      o_xq, o_sx, o_xsc, o_hq, o_hsc, total;
  bool w8a8;
};

int64_t capacity_of(int64_t T, int E, int k, float cf) {
  if (!(cf > 0.f)) return -1;  // <= 0 (NaN is rejected earlier): no limit
  const double c = floor(static_cast<double>(cf) * static_cast<double>(T) * k / E);
  const double cap = static_cast<double>(T) * k;
  return c >= cap ? static_cast<int64_t>(cap) : static_cast<int64_t>(c);
}

moe_status check_dims(const moe_dims* dims, int E, int k, float cf) {
  if (dims == nullptr) return MOE_ERR_INVALID_ARG;
  if (dims->T < 0 || dims->d <= 0 || dims->d_e <= 0 || dims->d_s < 0) return MOE_ERR_INVALID_ARG;
  if (dims->dtype != MOE_F32 && dims->dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
  if (E < 1 || k < 1 || k > E) return MOE_ERR_INVALID_ARG;
  if (isnan(cf)) return MOE_ERR_INVALID_ARG;
  if (dims->gate_mode < MOE_GATE_RENORM || dims->gate_mode > MOE_GATE_SIGMOID)
    return MOE_ERR_INVALID_ARG;
  if (E > moe::tc::MAX_E || k > 32) return MOE_ERR_UNSUPPORTED;
  if (dims->n_group > 1) {
    if (dims->n_group > 32) return MOE_ERR_UNSUPPORTED;
    if (E % dims->n_group != 0 || dims->topk_group < 1 || dims->topk_group > dims->n_group ||
        static_cast<int64_t>(k) > static_cast<int64_t>(dims->topk_group) * (E / dims->n_group))
      return MOE_ERR_INVALID_ARG;
  } else if (dims->n_group < 0) {
    return MOE_ERR_INVALID_ARG;
  }
  if (dims->T * static_cast<int64_t>(k) >= (int64_t(1) << 31) ||
      dims->T * static_cast<int64_t>(E) >= (int64_t(1) << 40))
    return MOE_ERR_UNSUPPORTED;
  if (dims->weight_format != MOE_WEIGHTS_DTYPE && dims->weight_format != MOE_WEIGHTS_FP8 &&
      dims->weight_format != MOE_WEIGHTS_FP8_W8A8 && dims->weight_format != MOE_WEIGHTS_MXFP4)
    return MOE_ERR_INVALID_ARG;
  if (dims->weight_format != MOE_WEIGHTS_DTYPE && (dims->dtype != MOE_BF16 || dims->d_s != 0))
    return MOE_ERR_UNSUPPORTED;
  // MXFP4: whole 256-deep code stages (eight 32-weight blocks) along both K extents
  if (dims->weight_format == MOE_WEIGHTS_MXFP4 && (dims->d % 256 || dims->d_e % 256))
    return MOE_ERR_UNSUPPORTED;
  const int mult = dims->dtype == MOE_BF16 ? 64 : 32;
  if (dims->d % mult || dims->d_e % mult || dims->d_s % mult) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

// Tensor-core router: experts per tile (E rounded up to the MMA's multiple of
// 16, at most 128).
int router_tc_n(int E) {
  const int n = (E + 15) / 16 * 16;
  return n < moe::rtc::MAX_N ? n : moe::rtc::MAX_N;
}

// Tensor-core router: K splits so that the tiles about fill the 148 SMs of a
// B200 (at most 16, whole 64-deep blocks, at least 8 blocks each). Depends only
// on the shape, so the workspace size does too.
int router_tc_split_k(int64_t T, int E, int d) {
  const int64_t tiles = ((T + moe::rtc::BM - 1) / moe::rtc::BM) *
                        ((E + router_tc_n(E) - 1) / router_tc_n(E));
  const int kb = d / moe::rtc::BK;
  int split = 1;
  while (split < 16 && tiles * split * 2 <= 148 && kb % (2 * split) == 0 && kb / (2 * split) >= 8)
    split *= 2;
  return split;
}

Plan make_plan(const moe_dims* dims, int E, int k, float cf) {
  Plan p{};
  p.T = dims->T;
  p.d = dims->d;
  p.de = dims->d_e;
  p.ds = dims->d_s;
  p.E = E;
  p.k = k;
  p.bf16 = dims->dtype == MOE_BF16;
  p.esz = p.bf16 ? 2 : 4;
  p.C = capacity_of(p.T, E, k, cf);
  p.nblk = static_cast<int>((p.T + moe::ROUTE_CHUNK - 1) / moe::ROUTE_CHUNK);
  p.rows_max = static_cast<int64_t>(
      align_up(static_cast<size_t>(p.T * k + static_cast<int64_t>(ROW_TILE - 1) * E), ROW_TILE));
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, ALIGN);
    return o;
  };
  const size_t T = static_cast<size_t>(p.T), TK = T * k, R = static_cast<size_t>(p.rows_max);
  p.router_tc = p.bf16;
  p.router_narrow = !p.router_tc && E <= 16;
  if (p.router_tc) {
    p.router_n = router_tc_n(E);
    p.router_split = router_tc_split_k(p.T, E, p.d);
  } else {
    p.router_split = p.router_narrow ? moe::narrow_split_k(p.T, E, p.d)
                                     : moe::router_wide_split_k(p.T, E, p.d);
  }
  p.o_logits = take(static_cast<size_t>(p.router_split) * T * E * 4);
  p.o_idx = take(TK * 4);
  p.o_gate = take(TK * 4);
  p.o_lrank = take(TK * 4);
  p.o_slot = take(TK * 4);
  p.o_hist = take(static_cast<size_t>(p.nblk) * E * 4);
  p.o_base = take(static_cast<size_t>(p.nblk) * E * 4);
  p.o_psum_part = take(static_cast<size_t>(p.nblk) * E * 8);
  p.o_probsum = take(static_cast<size_t>(E) * 8);
  p.o_tile_start = take(static_cast<size_t>(E + 1) * 4);
  p.o_pair_start = take(static_cast<size_t>(E + 1) * 4);
  p.o_status = take(4);  // the call's own device status word
  // tensor-core router: the hi / mid / lo bf16 terms of W_r, [3][E][d]
  p.o_wsplit = take(p.router_tc ? static_cast<size_t>(3) * E * p.d * 2 : 0);
  p.o_rowgate = take(R * 4);
  p.o_xp = take(R * p.d * p.esz);
  // H: fp32 with E4M3 activations (quantised per row from its fp32 value)
  p.o_h = take(R * p.de * (dims->weight_format == MOE_WEIGHTS_FP8_W8A8 ? 4 : p.esz));
  p.o_yrows = take(R * p.d * p.esz);
  p.o_hs = take(p.ds ? T * p.ds * p.esz : 0);
  p.o_ys = take(p.ds ? T * p.d * p.esz : 0);
  p.w8a8 = dims->weight_format == MOE_WEIGHTS_FP8_W8A8;
  p.o_xq = take(p.w8a8 ? T * p.d : 0);
  p.o_sx = take(p.w8a8 ? T * 4 : 0);
  p.o_xsc = take(p.w8a8 ? R * 4 : 0);
  p.o_hq = take(p.w8a8 ? R * p.de : 0);
  p.o_hsc = take(p.w8a8 ? R * 4 : 0);
  p.total = off;
  return p;
}

// ---------------------------------------------------------------------------
// Per-device one-time set-up: SM count and kernel attributes.
// ---------------------------------------------------------------------------
struct DeviceInfo {
  bool ready = false;
  int num_sms = 0;
  int pair_clusters[2] = {0, 0};  // co-resident 2-CTA clusters of each pair GEMM kernel
};
constexpr int kMaxDevices = 64;
DeviceInfo g_devices[kMaxDevices];
std::mutex g_dev_mutex;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

template <int EPI, int AR, bool Q8 = false>
bool tc_attr() {
  return cudaFuncSetAttribute(moe::tc::tc_grouped_gemm_kernel<EPI, AR, Q8>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              moe::tc::TcShape<AR>::SMEM_BYTES) == cudaSuccess;
}

// Launch a kernel of the forward pass with programmatic dependent launch: it
// may start launching while the previous kernel in the stream finishes, and
// waits in the kernel (pdl_wait) before touching memory that kernel may use.
// A failure is left for launched() to report.
template <typename... KArgs, typename... Args>
void launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  (void)cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Quantised-weight grouped GEMM (operands swapped, decoded weights in TMEM)
// with token boxes of `nb` rows (32, 64 or 128).
template <int EPI, int WQ>
bool wq_attr() {
  return cudaFuncSetAttribute(moe::wqs::tc_wq_swap_kernel<EPI, 32, WQ>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              moe::wqs::WqShape<32, WQ>::SMEM_BYTES) == cudaSuccess &&
         cudaFuncSetAttribute(moe::wqs::tc_wq_swap_kernel<EPI, 64, WQ>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              moe::wqs::WqShape<64, WQ>::SMEM_BYTES) == cudaSuccess &&
         cudaFuncSetAttribute(moe::wqs::tc_wq_swap_kernel<EPI, 128, WQ>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              moe::wqs::WqShape<128, WQ>::SMEM_BYTES) == cudaSuccess;
}

template <int EPI, int WQ>
void launch_wq(int nb, int grid, cudaStream_t st, const moe::tc::TcMaps& maps,
               const moe::wqs::WqParams& wp) {
  using namespace moe::wqs;
  if (nb == 32)
    launch_pdl(tc_wq_swap_kernel<EPI, 32, WQ>, grid, NUM_THREADS, WqShape<32, WQ>::SMEM_BYTES, st,
               maps, wp);
  else if (nb == 64)
    launch_pdl(tc_wq_swap_kernel<EPI, 64, WQ>, grid, NUM_THREADS, WqShape<64, WQ>::SMEM_BYTES, st,
               maps, wp);
  else
    launch_pdl(tc_wq_swap_kernel<EPI, 128, WQ>, grid, NUM_THREADS, WqShape<128, WQ>::SMEM_BYTES,
               st, maps, wp);
}

// 1-CTA grouped GEMM with an activation box of `ar` rows (128, 64 or 32);
// Q8: E4M3 operands.
template <int EPI, bool Q8 = false>
void launch_tc(int ar, int grid, cudaStream_t st, const moe::tc::TcMaps& maps,
               const moe::tc::TcParams& tp) {
  using namespace moe::tc;
  if (ar == 32)
    launch_pdl(tc_grouped_gemm_kernel<EPI, 32, Q8>, grid, NUM_THREADS, TcShape<32>::SMEM_BYTES, st, maps, tp);
  else if (ar == 64)
    launch_pdl(tc_grouped_gemm_kernel<EPI, 64, Q8>, grid, NUM_THREADS, TcShape<64>::SMEM_BYTES, st, maps, tp);
  else
    launch_pdl(tc_grouped_gemm_kernel<EPI, 128, Q8>, grid, NUM_THREADS, TcShape<128>::SMEM_BYTES, st, maps, tp);
}

// Launch configuration of the CTA-pair kernels: clusters of two; with `pdl`,
// also programmatic dependent launch (see launch_pdl). attr holds 2 entries.
template <int EPI>
cudaLaunchConfig_t pair_config(int clusters, cudaStream_t st, cudaLaunchAttribute* attr,
                               bool pdl = false) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(2 * clusters, 1, 1);
  cfg.blockDim = dim3(moe::tc2::NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = moe::tc2::SMEM_BYTES;
  cfg.stream = st;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  return cfg;
}

template <int EPI, bool SWAP = false>
bool pair_setup(int num_sms, int* clusters) {
  auto kern = moe::tc2::tc2_grouped_gemm_kernel<EPI, SWAP>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           moe::tc2::SMEM_BYTES) != cudaSuccess)
    return false;
  cudaLaunchAttribute attr[2];
  cudaLaunchConfig_t cfg = pair_config<EPI>(num_sms / 2, nullptr, attr);
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) return false;
  *clusters = n < num_sms / 2 ? n : num_sms / 2;
  return true;
}

moe_status device_setup(int* num_sms, int* pair_clusters = nullptr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_dev_mutex);
  DeviceInfo& di = g_devices[dev];
  if (!di.ready) {
    if (cudaDeviceGetAttribute(&di.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return MOE_ERR_CUDA;
    if (g_encode == nullptr) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault,
                                           &q) != cudaSuccess ||
          q != cudaDriverEntryPointSuccess || fn == nullptr)
        return MOE_ERR_CUDA;
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    if (!tc_attr<moe::tc::EPI_SWIGLU_TC, 128>() || !tc_attr<moe::tc::EPI_SCALE_TC, 128>() ||
        !tc_attr<moe::tc::EPI_SWIGLU_TC, 64>() || !tc_attr<moe::tc::EPI_SCALE_TC, 64>() ||
        !tc_attr<moe::tc::EPI_SWIGLU_TC, 32>() || !tc_attr<moe::tc::EPI_SCALE_TC, 32>())
      return MOE_ERR_CUDA;
    if (!tc_attr<moe::tc::EPI_SWIGLU_TC, 128, true>() ||
        !tc_attr<moe::tc::EPI_SCALE_TC, 128, true>() ||
        !tc_attr<moe::tc::EPI_SWIGLU_TC, 64, true>() || !tc_attr<moe::tc::EPI_SCALE_TC, 64, true>() ||
        !tc_attr<moe::tc::EPI_SWIGLU_TC, 32, true>() || !tc_attr<moe::tc::EPI_SCALE_TC, 32, true>())
      return MOE_ERR_CUDA;
    if (cudaFuncSetAttribute(moe::tcws::tc_ws_grouped_gemm_kernel<moe::tc::EPI_SWIGLU_TC>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             moe::tcws::SMEM_BYTES) != cudaSuccess ||
        cudaFuncSetAttribute(moe::tcws::tc_ws_grouped_gemm_kernel<moe::tc::EPI_SCALE_TC>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             moe::tcws::SMEM_BYTES) != cudaSuccess)
      return MOE_ERR_CUDA;
    if (!wq_attr<moe::tc::EPI_SWIGLU_TC, moe::tcf8::WQ_FP8>() ||
        !wq_attr<moe::tc::EPI_SCALE_TC, moe::tcf8::WQ_FP8>() ||
        !wq_attr<moe::tc::EPI_SWIGLU_TC, moe::tcf8::WQ_MXFP4>() ||
        !wq_attr<moe::tc::EPI_SCALE_TC, moe::tcf8::WQ_MXFP4>())
      return MOE_ERR_CUDA;
    int swap_clusters = 0;
    if (!pair_setup<moe::tc::EPI_SWIGLU_TC>(di.num_sms, &di.pair_clusters[0]) ||
        !pair_setup<moe::tc::EPI_SCALE_TC>(di.num_sms, &di.pair_clusters[1]) ||
        !pair_setup<moe::tc::EPI_SCALE_TC, true>(di.num_sms, &swap_clusters) ||
        swap_clusters != di.pair_clusters[1])
      return MOE_ERR_CUDA;
    if (cudaFuncSetAttribute(moe::rtc::router_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             moe::rtc::SMEM_LIMIT) != cudaSuccess)
      return MOE_ERR_CUDA;
    const int rs = static_cast<int>(moe::route_smem_bytes(moe::tc::MAX_E));
    if (cudaFuncSetAttribute(moe::route_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             rs) != cudaSuccess ||
        cudaFuncSetAttribute(moe::route_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             rs) != cudaSuccess)
      return MOE_ERR_CUDA;
    di.ready = true;
  }
  *num_sms = di.num_sms;
  if (pair_clusters != nullptr) {
    pair_clusters[0] = di.pair_clusters[0];
    pair_clusters[1] = di.pair_clusters[1];
  }
  return MOE_OK;
}

// ---------------------------------------------------------------------------
// Scratch of moe_forward_no_alloc: a statically sized device array, so the
// call itself allocates nothing. In host code `g_no_alloc_scratch` only names
// the symbol; its device address comes from cudaGetSymbolAddress, looked up
// once per device with that device current.
// ---------------------------------------------------------------------------
static __device__ __align__(256) uint8_t g_no_alloc_scratch[MOE_NO_ALLOC_WORKSPACE_BYTES];
void* g_no_alloc_ptr[kMaxDevices] = {};

moe_status no_alloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_dev_mutex);
  if (g_no_alloc_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_no_alloc_scratch) != cudaSuccess || ptr == nullptr)
      return MOE_ERR_CUDA;
    g_no_alloc_ptr[dev] = ptr;
  }
  *out = g_no_alloc_ptr[dev];
  return MOE_OK;
}

// bf16 tensor map over a row-major [outer][mid][inner] array (mid = 1 for 2D),
// 128-byte swizzle, box {64, box_rows(, 1)}; out-of-range rows read as zero.
bool encode_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t mid, uint64_t outer,
                uint32_t box_rows, int rank) {
  cuuint64_t dims[3] = {inner, mid, outer};
  cuuint64_t strides[2] = {inner * 2, inner * mid * 2};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(moe::tc::BK), box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r =
      g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Weight-code tensor map over [outer][mid][inner] bytes (inner a multiple of
// 16: FP8 codes, or MXFP4 codes two per byte), box {128 bytes, box_rows, 1}
// (full 128-byte lines), 128-byte swizzle. The bytes are described to the TMA
// unit as 32-bit words: they land exactly where a uint8 map would put them, in
// a quarter of the elements.
bool encode_map_u8(CUtensorMap* m, const void* base, uint64_t inner, uint64_t mid, uint64_t outer,
                   uint32_t box_rows) {
  cuuint64_t dims[3] = {inner / 4, mid, outer};
  cuuint64_t strides[2] = {inner, inner * mid};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(moe::wqs::Q_ROW / 4), box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r =
      g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<void*>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

struct Timer {
  void* const* ev;
  cudaStream_t s;
  void at(int i) const {
    if (ev != nullptr && ev[i] != nullptr) cudaEventRecord(static_cast<cudaEvent_t>(ev[i]), s);
  }
};

moe_status launched() { return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }



template <typename TX>
moe_status launch_route_and_permute(const Plan& P, const moe_dims* dims, const TX* x,
                                    const float* W_r, uint8_t* ws, int32_t* counts, float* aux,
                                    cudaStream_t st, const Timer& tm,
                                    unsigned long long wait_tmo) {
  float* logits = reinterpret_cast<float*>(ws + P.o_logits);
  int32_t* idx = reinterpret_cast<int32_t*>(ws + P.o_idx);
  float* gate = reinterpret_cast<float*>(ws + P.o_gate);
  int32_t* lrank = reinterpret_cast<int32_t*>(ws + P.o_lrank);
  int32_t* slot = reinterpret_cast<int32_t*>(ws + P.o_slot);
  int32_t* hist = reinterpret_cast<int32_t*>(ws + P.o_hist);
  int32_t* base = reinterpret_cast<int32_t*>(ws + P.o_base);
  double* psum_part = reinterpret_cast<double*>(ws + P.o_psum_part);
  double* probsum = reinterpret_cast<double*>(ws + P.o_probsum);
  int32_t* tile_start = reinterpret_cast<int32_t*>(ws + P.o_tile_start);
  int32_t* pair_start = reinterpret_cast<int32_t*>(ws + P.o_pair_start);
  float* rowgate = reinterpret_cast<float*>(ws + P.o_rowgate);
  TX* xp = reinterpret_cast<TX*>(ws + P.o_xp);
  const int T = static_cast<int>(P.T);

  // (0) router logits: split-precision tensor cores (bf16 x), or fp32 FMA
  tm.at(0);
  if (P.router_tc) {
    __nv_bfloat16* wsplit = reinterpret_cast<__nv_bfloat16*>(ws + P.o_wsplit);
    const int64_t n = static_cast<int64_t>(P.E) * P.d;
    const int64_t blocks = (n + 255) / 256;
    launch_pdl(moe::rtc::split_router_weights_kernel, static_cast<unsigned>(blocks < 4096 ? blocks : 4096), 256, 0, st, W_r, n, wsplit);
    moe::rtc::RtcMaps maps;
    memset(&maps, 0, sizeof(maps));
    if (!encode_map(&maps.x, x, P.d, P.T, 1, moe::rtc::BM, 2) ||
        !encode_map(&maps.w, wsplit, P.d, P.E, 3, P.router_n, 3))
      return MOE_ERR_CUDA;
    moe::rtc::RtcParams rp{};
    rp.T = T;
    rp.E = P.E;
    rp.N = P.router_n;
    rp.k_blocks = P.d / moe::rtc::BK / P.router_split;
    rp.logits = logits;
    rp.timeout_ns = wait_tmo;
    rp.drain_timeout_ns = kDrainTimeoutNs;
    rp.call_err = reinterpret_cast<int*>(ws + P.o_status);
    dim3 grid((T + moe::rtc::BM - 1) / moe::rtc::BM, (P.E + P.router_n - 1) / P.router_n,
              P.router_split);
    launch_pdl(moe::rtc::router_tc_kernel, grid, moe::rtc::NUM_THREADS, moe::rtc::smem_bytes(P.router_n), st, maps,
                                                                                          rp);
  } else if (P.router_narrow) {
    if (P.E <= 8) {
      dim3 grid((T + moe::NarrowShape<8>::TB - 1) / moe::NarrowShape<8>::TB, P.router_split);
      launch_pdl(moe::router_narrow_kernel<TX, 8>, grid, 256, 0, st, x, W_r, T, P.d, P.E, P.router_split, logits);
    } else {
      dim3 grid((T + moe::NarrowShape<16>::TB - 1) / moe::NarrowShape<16>::TB, P.router_split);
      launch_pdl(moe::router_narrow_kernel<TX, 16>, grid, 256, 0, st, x, W_r, T, P.d, P.E, P.router_split, logits);
    }
  } else {
    dim3 grid((P.E + moe::RW_BN - 1) / moe::RW_BN, (T + moe::RW_BM - 1) / moe::RW_BM,
              P.router_split);
    launch_pdl(moe::router_wide_kernel<TX>, grid, 256, 0, st, x, W_r, T, P.d, P.E, P.router_split,
                                                       logits);
  }
  tm.at(1);
  if (launched() != MOE_OK) return MOE_ERR_CUDA;

  // (1) routing; a batch of one 64-token chunk with at most 256 experts also
  // runs the scan (step 2) in the same kernel
  const bool fused_scan = P.nblk == 1 && P.E <= 256;
  moe::ScanArgs sa{};
  sa.fused = fused_scan;
  sa.C = P.C;
  sa.rows_max = P.rows_max;
  sa.counts = counts;
  sa.base = base;
  sa.tile_start = tile_start;
  sa.pair_start = pair_start;
  sa.probsum = probsum;
  sa.aux = aux;
  sa.call_err = reinterpret_cast<int*>(ws + P.o_status);
  tm.at(2);
  {
    const size_t smem = moe::route_smem_bytes(P.E);
    const int nv = (P.E + 31) / 32;
#define MOE_ROUTE(NV)                                                                         \
  launch_pdl(moe::route_kernel<NV>, P.nblk, 256, smem, st, \
      logits, P.router_split, dims->router_bias, dims->selection_bias, dims->gate_mode,       \
      dims->n_group, dims->topk_group, T, P.E, P.k, idx, gate, lrank, hist, psum_part, sa)
    if (nv <= 1) MOE_ROUTE(1);
    else if (nv <= 2) MOE_ROUTE(2);
    else if (nv <= 4) MOE_ROUTE(4);
    else if (nv <= 8) MOE_ROUTE(8);
    else if (nv <= 16) MOE_ROUTE(16);
    else MOE_ROUTE(32);
#undef MOE_ROUTE
  }
  tm.at(3);
  if (launched() != MOE_OK) return MOE_ERR_CUDA;

  // (2) scan: counts, capacity, segment offsets, aux
  tm.at(4);
  if (!fused_scan)
    launch_pdl(moe::scan_kernel, 1, moe::scan_kernel_threads(P.E), 0, st, hist, P.nblk, psum_part, P.nblk, P.E, P.T, P.k, P.C, counts, base, tile_start, pair_start,
        probsum, aux, sa.call_err, P.rows_max);
  tm.at(5);
  if (launched() != MOE_OK) return MOE_ERR_CUDA;

  // (3) scatter rows into expert segments
  tm.at(6);
  {
    const int nvec = static_cast<int>(static_cast<size_t>(P.d) * sizeof(TX) / 16);
    dim3 grid((T + 7) / 8, (nvec + moe::PERMUTE_CHUNK_VECS - 1) / moe::PERMUTE_CHUNK_VECS);
    if (P.w8a8) {
      // E4M3 activations: quantise each token row once (scale per token), then
      // scatter the code rows and carry each row's scale to its slots
      uint8_t* xq = ws + P.o_xq;
      float* sx = reinterpret_cast<float*>(ws + P.o_sx);
      launch_pdl(moe::tcf8::quantize_rows_fp8_kernel<TX>, static_cast<unsigned>(T < 8192 ? T : 8192),
                 256, 0, st, x, T, P.d, xq, sx, nullptr, nullptr, 0, int64_t(-1));
      const int qvec = P.d / 16;
      dim3 qgrid((T + 7) / 8, (qvec + moe::PERMUTE_CHUNK_VECS - 1) / moe::PERMUTE_CHUNK_VECS);
      launch_pdl(moe::scatter_kernel<uint8_t>, qgrid, 256, 0, st, xq, P.d, T, P.k, P.E, P.C, idx, gate, lrank, base, tile_start, slot, rowgate,
          reinterpret_cast<uint8_t*>(xp), P.rows_max, sx, reinterpret_cast<float*>(ws + P.o_xsc));
    } else if (dims->weight_format == MOE_WEIGHTS_FP8 || dims->weight_format == MOE_WEIGHTS_MXFP4) {
      // the quantised-weight GEMMs read fp16 rows
      launch_pdl(moe::scatter_kernel<TX, true>, grid, 256, 0, st, x, P.d, T, P.k, P.E, P.C, idx, gate,
                                                          lrank, base, tile_start, slot, rowgate,
                                                          xp, P.rows_max, nullptr, nullptr);
    } else
      launch_pdl(moe::scatter_kernel<TX>, grid, 256, 0, st, x, P.d, T, P.k, P.E, P.C, idx, gate, lrank,
                                                    base, tile_start, slot, rowgate, xp,
                                                    P.rows_max, nullptr, nullptr);
  }
  tm.at(7);
  return launched();
}

moe_status forward_impl(const moe_dims* dims, const void* x, const float* W_r, const void* W_g,
                        const void* W_u, const void* W_d, const void* W_shared, int E, int k,
                        float cf, void* y, float* aux, int32_t* counts) {
  moe_status s = check_dims(dims, E, k, cf);
  if (s != MOE_OK) return s;
  if (aux == nullptr || counts == nullptr) return MOE_ERR_INVALID_ARG;
  if (!aligned(aux, 4) || !aligned(counts, 4)) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(dims->stream);
  if (dims->T == 0) {
    if (cudaMemsetAsync(counts, 0, sizeof(int32_t) * E, st) != cudaSuccess ||
        cudaMemsetAsync(aux, 0, sizeof(float), st) != cudaSuccess)
      return MOE_ERR_CUDA;
    return MOE_OK;
  }
  if (x == nullptr || W_r == nullptr || W_g == nullptr || W_u == nullptr || W_d == nullptr ||
      y == nullptr || (dims->d_s > 0 && W_shared == nullptr))
    return MOE_ERR_INVALID_ARG;
  const void* ptrs[] = {x, W_r, W_g, W_u, W_d, y};
  for (const void* q : ptrs)
    if (!aligned(q, 16)) return MOE_ERR_INVALID_ARG;
  if (dims->d_s > 0 && !aligned(W_shared, 16)) return MOE_ERR_INVALID_ARG;
  if (dims->router_bias != nullptr && !aligned(dims->router_bias, 16)) return MOE_ERR_INVALID_ARG;
  if (dims->selection_bias != nullptr && !aligned(dims->selection_bias, 16))
    return MOE_ERR_INVALID_ARG;
  if (dims->weight_format != MOE_WEIGHTS_DTYPE &&
      (dims->weight_scales == nullptr || !aligned(dims->weight_scales, 4)))
    return MOE_ERR_INVALID_ARG;
  if (dims->weight_format == MOE_WEIGHTS_MXFP4 &&
      (dims->weight_block_scales == nullptr || !aligned(dims->weight_block_scales, 16)))
    return MOE_ERR_INVALID_ARG;

  const Plan P = make_plan(dims, E, k, cf);
  if (dims->workspace == nullptr || !aligned(dims->workspace, 256) ||
      dims->workspace_bytes < P.total)
    return MOE_ERR_WORKSPACE;
  int num_sms = 0, pair_clusters[2] = {0, 0};
  s = device_setup(&num_sms, pair_clusters);
  if (s != MOE_OK) return s;

  uint8_t* ws = static_cast<uint8_t*>(dims->workspace);
  const Timer tm{dims->events, st};
  const unsigned long long wait_tmo =
      dims->wait_timeout_ns != 0 ? static_cast<unsigned long long>(dims->wait_timeout_ns)
                                 : kWaitTimeoutNs;
  const int T = static_cast<int>(P.T);
  int32_t* slot = reinterpret_cast<int32_t*>(ws + P.o_slot);
  int32_t* tile_start = reinterpret_cast<int32_t*>(ws + P.o_tile_start);
  float* rowgate = reinterpret_cast<float*>(ws + P.o_rowgate);
  int* call_err = reinterpret_cast<int*>(ws + P.o_status);
  const int rows_cap = static_cast<int>(P.rows_max);  // permuted rows (debug bounds checks)

  if (P.bf16) {
    using bf16 = __nv_bfloat16;
    s = launch_route_and_permute<bf16>(P, dims, static_cast<const bf16*>(x), W_r, ws, counts, aux,
                                       st, tm, wait_tmo);
    if (s != MOE_OK) return s;
    const bf16* xp = reinterpret_cast<const bf16*>(ws + P.o_xp);
    bf16* h = reinterpret_cast<bf16*>(ws + P.o_h);
    bf16* yrows = reinterpret_cast<bf16*>(ws + P.o_yrows);
    bf16* hs = P.ds ? reinterpret_cast<bf16*>(ws + P.o_hs) : nullptr;
    bf16* ys = P.ds ? reinterpret_cast<bf16*>(ws + P.o_ys) : nullptr;
    const bf16* sg = static_cast<const bf16*>(W_shared);
    const size_t sh_n = static_cast<size_t>(P.ds) * P.d;
    const int ng = P.ds ? 2 : 1;

    if (P.w8a8) {
      // E4M3 x E4M3 (kind::f8f6f4) on the 1-CTA kernels; H is quantised per row
      // between the two GEMMs
      const int arows = P.T <= 32 ? 32 : (P.T <= 64 ? 64 : 128);
      const float* sc = dims->weight_scales;
      const size_t gsz = static_cast<size_t>(E) * P.de;
      uint8_t* hq = ws + P.o_hq;
      float* xsc = reinterpret_cast<float*>(ws + P.o_xsc);
      float* hsc = reinterpret_cast<float*>(ws + P.o_hsc);
      constexpr int K8 = 128;  // codes per K step
      moe::tc::TcMaps up, dn;
      memset(&up, 0, sizeof(up));
      memset(&dn, 0, sizeof(dn));
      // the code rows are described to TMA as 16-bit elements (2 codes each),
      // with the same boxes as the bf16 path: 128-byte lines, 128-byte swizzle
      const bool ok = encode_map(&up.a[0], xp, P.d / 2, P.rows_max, 1, arows, 2) &&
                      encode_map(&up.b0[0], W_g, P.d / 2, P.de, E, moe::tc::BN / 2, 3) &&
                      encode_map(&up.b1[0], W_u, P.d / 2, P.de, E, moe::tc::BN / 2, 3) &&
                      encode_map(&dn.a[0], hq, P.de / 2, P.rows_max, 1, arows, 2) &&
                      encode_map(&dn.b0[0], W_d, P.de / 2, P.d, E, moe::tc::BN, 3);
      if (!ok) return MOE_ERR_CUDA;
      dn.b1[0] = dn.b0[0];
      moe::tc::TcParams tu{};
      tu.num_groups = 1;
      tu.timeout_ns = wait_tmo;
      tu.drain_timeout_ns = kDrainTimeoutNs;
      tu.call_err = call_err;
      tu.g[0] = {tile_start, E, rows_cap, (P.de + moe::tc::BN / 2 - 1) / (moe::tc::BN / 2),
                 (P.d + K8 - 1) / K8, P.de, h, nullptr, xsc, sc, sc + gsz, P.de};
      moe::tc::TcParams td{};
      td.num_groups = 1;
      td.timeout_ns = wait_tmo;
      td.drain_timeout_ns = kDrainTimeoutNs;
      td.call_err = call_err;
      td.g[0] = {tile_start, E, rows_cap, (P.d + moe::tc::BN - 1) / moe::tc::BN, (P.de + K8 - 1) / K8,
                 P.d, yrows, rowgate, hsc, sc + 2 * gsz, sc + 2 * gsz, P.d};
      tm.at(8);
      launch_tc<moe::tc::EPI_SWIGLU_TC, true>(arows, num_sms, st, up, tu);
      tm.at(9);
      if (launched() != MOE_OK) return MOE_ERR_CUDA;
      tm.at(10);
      launch_pdl(moe::tcf8::quantize_rows_fp8_kernel<float>, static_cast<unsigned>(P.rows_max < 8192 ? P.rows_max : 8192), 256, 0, st, reinterpret_cast<const float*>(h), P.rows_max, P.de, hq, hsc, tile_start, counts, E,
              P.C);
      launch_tc<moe::tc::EPI_SCALE_TC, true>(arows, num_sms, st, dn, td);
      tm.at(11);
      if (launched() != MOE_OK) return MOE_ERR_CUDA;
    } else if (dims->weight_format == MOE_WEIGHTS_FP8 || dims->weight_format == MOE_WEIGHTS_MXFP4) {
      // FP8 or MXFP4 expert weights: operands swapped (weights are the M = 128
      // side), decoded on chip into TMEM; token boxes of 32, 64 or 128 rows
      const bool mx = dims->weight_format == MOE_WEIGHTS_MXFP4;
      {
        const int nb = P.T <= 32 ? 32 : (P.T <= 64 ? 64 : 128);
        const float* sc = dims->weight_scales;
        const size_t gsz = static_cast<size_t>(E) * P.de;
        const int cpb = mx ? 2 : 1;  // codes per byte
        moe::tc::TcMaps up, dn;
        memset(&up, 0, sizeof(up));
        memset(&dn, 0, sizeof(dn));
        const bool ok = encode_map(&up.a[0], xp, P.d, P.rows_max, 1, nb, 2) &&
                        encode_map_u8(&up.b0[0], W_g, P.d / cpb, P.de, E, moe::tc::BM) &&
                        encode_map_u8(&up.b1[0], W_u, P.d / cpb, P.de, E, moe::tc::BM) &&
                        encode_map(&dn.a[0], h, P.de, P.rows_max, 1, nb, 2) &&
                        encode_map_u8(&dn.b0[0], W_d, P.de / cpb, P.d, E, moe::tc::BM);
        if (!ok) return MOE_ERR_CUDA;
        const uint8_t* bs = dims->weight_block_scales;
        const size_t gbs = gsz * (P.d / 32);
        moe::wqs::WqParams wu{}, wd{};
        wu.timeout_ns = wd.timeout_ns = wait_tmo;
        wu.drain_timeout_ns = wd.drain_timeout_ns = kDrainTimeoutNs;
        wu.call_err = wd.call_err = call_err;
        wu.grp.tile_start = wd.grp.tile_start = tile_start;
        wu.grp.E = wd.grp.E = E;
        wu.grp.rows = wd.grp.rows = rows_cap;
        wu.grp.n_tiles = (P.de + moe::tc::BM - 1) / moe::tc::BM;
        wu.grp.k_blocks = P.d / moe::tc::BK;
        wu.grp.N = P.de;
        wu.grp.out = h;
        wu.grp.scale0 = sc;
        wu.grp.scale1 = sc + gsz;
        wu.grp.scale_stride = P.de;
        wd.grp.n_tiles = (P.d + 2 * moe::tc::BM - 1) / (2 * moe::tc::BM);
        wd.grp.k_blocks = P.de / moe::tc::BK;
        wd.grp.N = P.d;
        wd.grp.out = yrows;
        wd.grp.row_gate = rowgate;
        wd.grp.scale0 = wd.grp.scale1 = sc + 2 * gsz;
        wd.grp.scale_stride = P.d;
        if (mx) {
          wu.grp.bscale0 = bs;
          wu.grp.bscale1 = bs + gbs;
          wu.grp.bscale_stride = static_cast<int64_t>(P.de) * (P.d / 32);
          wu.grp.kblk = P.d / 32;
          wd.grp.bscale0 = wd.grp.bscale1 = bs + 2 * gbs;
          wd.grp.bscale_stride = static_cast<int64_t>(P.d) * (P.de / 32);
          wd.grp.kblk = P.de / 32;
        }
        tm.at(8);
        if (mx)
          launch_wq<moe::tc::EPI_SWIGLU_TC, moe::tcf8::WQ_MXFP4>(nb, num_sms, st, up, wu);
        else
          launch_wq<moe::tc::EPI_SWIGLU_TC, moe::tcf8::WQ_FP8>(nb, num_sms, st, up, wu);
        tm.at(9);
        if (launched() != MOE_OK) return MOE_ERR_CUDA;
        tm.at(10);
        if (mx)
          launch_wq<moe::tc::EPI_SCALE_TC, moe::tcf8::WQ_MXFP4>(nb, num_sms, st, dn, wd);
        else
          launch_wq<moe::tc::EPI_SCALE_TC, moe::tcf8::WQ_FP8>(nb, num_sms, st, dn, wd);
        tm.at(11);
        if (launched() != MOE_OK) return MOE_ERR_CUDA;
      }
    } else {
    // (4) gate/up projection + SwiGLU, (5) down projection scaled by the gates.
    // CTA-pair tiles (256 rows) cut the operand traffic per SM by a third but
    // pair up the 128-row tiles of each expert, so an expert with an odd tile
    // count computes one idle half-tile. They are used where experts get many
    // rows: down (long K, few N tiles) from 512 rows per expert, gate/up from 2048.
    const int64_t rows_per_expert = P.T * P.k / E;
#if defined(MOE_FORCE_1CTA)
    const bool pair_up = false, pair_down = false;
#elif defined(MOE_FORCE_PAIR)
    const bool pair_up = true, pair_down = true;
#else
    const bool pair_up = rows_per_expert >= 2048;
    const bool pair_down = rows_per_expert >= 512;
#endif
    // activation box of the 1-CTA kernel: no expert (and no dense group) holds more
    // than T rows, so small batches load only that many
    const int arows = P.T <= 32 ? 32 : (P.T <= 64 ? 64 : 128);
    int32_t* pair_start = reinterpret_cast<int32_t*>(ws + P.o_pair_start);
    constexpr int HB = 128;  // rows of B each CTA of a pair loads
    constexpr int BNp = moe::tc2::BN;
    cudaLaunchAttribute attr[2];
    // Swapped operands (tc_ws_gemm.cuh: weights as the M side, token tiles sized
    // to their valid rows, so the 128-row segment padding is not multiplied):
    // measured faster for gate/up up to 2048 routed rows per expert, and for
    // down up to 512 (above that the CTA-pair down kernel wins).
    const bool ws_up = P.T > 64 && rows_per_expert <= kWsUpMaxRowsPerExpert;
    const bool ws_down = P.T > 64 && rows_per_expert <= kWsDownMaxRowsPerExpert;
    constexpr int WB = moe::tc::BM;  // weight rows per box of the swapped kernel
    if (ws_up) {
      moe::tc::TcMaps up;
      memset(&up, 0, sizeof(up));
      bool ok = encode_map(&up.a[0], xp, P.d, P.rows_max, 1, moe::tcws::NB, 2) &&
                encode_map(&up.b0[0], W_g, P.d, P.de, E, WB, 3) &&
                encode_map(&up.b1[0], W_u, P.d, P.de, E, WB, 3);
      if (P.ds)
        ok = ok && encode_map(&up.a[1], x, P.d, P.T, 1, moe::tcws::NB, 2) &&
             encode_map(&up.b0[1], sg, P.d, P.ds, 1, WB, 3) &&
             encode_map(&up.b1[1], sg + sh_n, P.d, P.ds, 1, WB, 3);
      if (!ok) return MOE_ERR_CUDA;
      moe::tc::TcParams tu{};
      tu.num_groups = ng;
      tu.timeout_ns = wait_tmo;
      tu.drain_timeout_ns = kDrainTimeoutNs;
      tu.call_err = call_err;
      tu.g[0] = {tile_start, E, rows_cap, (P.de + WB - 1) / WB, P.d / moe::tc::BK, P.de, h, nullptr};
      tu.g[0].counts = counts;
      tu.g[0].cap = P.C;
      if (P.ds)
        tu.g[1] = {nullptr, 1, T, (P.ds + WB - 1) / WB, P.d / moe::tc::BK, P.ds, hs, nullptr};
      tm.at(8);
      launch_pdl(moe::tcws::tc_ws_grouped_gemm_kernel<moe::tc::EPI_SWIGLU_TC>, num_sms,
                 moe::tcws::NUM_THREADS, moe::tcws::SMEM_BYTES, st, up, tu);
      tm.at(9);
      if (launched() != MOE_OK) return MOE_ERR_CUDA;
    } else {
      const int brows = pair_up ? HB : moe::tc::BN / 2;
      const int abox = pair_up ? moe::tc::BM : arows;
      moe::tc::TcMaps up;
      memset(&up, 0, sizeof(up));
      bool ok = encode_map(&up.a[0], xp, P.d, P.rows_max, 1, abox, 2) &&
                encode_map(&up.b0[0], W_g, P.d, P.de, E, brows, 3) &&
                encode_map(&up.b1[0], W_u, P.d, P.de, E, brows, 3);
      if (P.ds)
        ok = ok && encode_map(&up.a[1], x, P.d, P.T, 1, abox, 2) &&
             encode_map(&up.b0[1], sg, P.d, P.ds, 1, brows, 3) &&
             encode_map(&up.b1[1], sg + sh_n, P.d, P.ds, 1, brows, 3);
      if (!ok) return MOE_ERR_CUDA;
      tm.at(8);
      if (pair_up) {
        moe::tc2::Tc2Params tu{};
        tu.num_groups = ng;
        tu.timeout_ns = wait_tmo;
        tu.drain_timeout_ns = kDrainTimeoutNs;
        tu.call_err = call_err;
        tu.g[0] = {tile_start, pair_start, E, rows_cap, (P.de + BNp / 2 - 1) / (BNp / 2),
                   P.d / moe::tc::BK, P.de, h, nullptr};
        if (P.ds)
          tu.g[1] = {nullptr, nullptr, 1, T, (P.ds + BNp / 2 - 1) / (BNp / 2), P.d / moe::tc::BK,
                     P.ds, hs, nullptr};
        cudaLaunchConfig_t cfg = pair_config<moe::tc::EPI_SWIGLU_TC>(pair_clusters[0], st, attr, true);
        if (cudaLaunchKernelEx(&cfg, moe::tc2::tc2_grouped_gemm_kernel<moe::tc::EPI_SWIGLU_TC>,
                               up, tu) != cudaSuccess)
          return MOE_ERR_CUDA;
      } else {
        moe::tc::TcParams tp{};
        tp.num_groups = ng;
        tp.timeout_ns = wait_tmo;
        tp.drain_timeout_ns = kDrainTimeoutNs;
        tp.call_err = call_err;
        tp.g[0] = {tile_start, E, rows_cap, (P.de + moe::tc::BN / 2 - 1) / (moe::tc::BN / 2),
                   P.d / moe::tc::BK, P.de, h, nullptr};
        if (P.ds)
          tp.g[1] = {nullptr, 1, T, (P.ds + moe::tc::BN / 2 - 1) / (moe::tc::BN / 2),
                     P.d / moe::tc::BK, P.ds, hs, nullptr};
        launch_tc<moe::tc::EPI_SWIGLU_TC>(arows, num_sms, st, up, tp);
      }
      tm.at(9);
      if (launched() != MOE_OK) return MOE_ERR_CUDA;
    }
    if (ws_down) {
      moe::tc::TcMaps dn;
      memset(&dn, 0, sizeof(dn));
      bool ok = encode_map(&dn.a[0], h, P.de, P.rows_max, 1, moe::tcws::NB, 2) &&
                encode_map(&dn.b0[0], W_d, P.de, P.d, E, WB, 3);
      if (P.ds)
        ok = ok && encode_map(&dn.a[1], hs, P.ds, P.T, 1, moe::tcws::NB, 2) &&
             encode_map(&dn.b0[1], sg + 2 * sh_n, P.ds, P.d, 1, WB, 3);
      if (!ok) return MOE_ERR_CUDA;
      dn.b1[0] = dn.b0[0];
      dn.b1[1] = dn.b0[1];
      moe::tc::TcParams td{};
      td.num_groups = ng;
      td.timeout_ns = wait_tmo;
      td.drain_timeout_ns = kDrainTimeoutNs;
      td.call_err = call_err;
      td.g[0] = {tile_start, E, rows_cap, (P.d + 2 * WB - 1) / (2 * WB), P.de / moe::tc::BK, P.d,
                 yrows, rowgate};
      td.g[0].counts = counts;
      td.g[0].cap = P.C;
      if (P.ds)
        td.g[1] = {nullptr, 1, T, (P.d + 2 * WB - 1) / (2 * WB), P.ds / moe::tc::BK, P.d, ys,
                   nullptr};
      tm.at(10);
      launch_pdl(moe::tcws::tc_ws_grouped_gemm_kernel<moe::tc::EPI_SCALE_TC>, num_sms,
                 moe::tcws::NUM_THREADS, moe::tcws::SMEM_BYTES, st, dn, td);
      tm.at(11);
      if (launched() != MOE_OK) return MOE_ERR_CUDA;
    } else {
      const int brows = pair_down ? HB : moe::tc::BN;
      const int abox = pair_down ? moe::tc::BM : arows;
      moe::tc::TcMaps dn;
      memset(&dn, 0, sizeof(dn));
      // swapped pairs: the weight map is A and the rows' map B
      const bool swap = pair_down && kPairDownSwap;
      const void* dn_rows[2] = {h, hs};
      bool ok = swap ? encode_map(&dn.a[0], W_d, P.de, P.d, E, HB, 3) &&
                           encode_map(&dn.b0[0], h, P.de, P.rows_max, 1, HB, 2)
                     : encode_map(&dn.a[0], h, P.de, P.rows_max, 1, abox, 2) &&
                           encode_map(&dn.b0[0], W_d, P.de, P.d, E, brows, 3);
      if (P.ds)
        ok = ok && (swap ? encode_map(&dn.a[1], sg + 2 * sh_n, P.ds, P.d, 1, HB, 3) &&
                               encode_map(&dn.b0[1], dn_rows[1], P.ds, P.T, 1, HB, 2)
                         : encode_map(&dn.a[1], hs, P.ds, P.T, 1, abox, 2) &&
                               encode_map(&dn.b0[1], sg + 2 * sh_n, P.ds, P.d, 1, brows, 3));
      if (!ok) return MOE_ERR_CUDA;
      dn.b1[0] = dn.b0[0];
      dn.b1[1] = dn.b0[1];
      tm.at(10);
      if (pair_down) {
        moe::tc2::Tc2Params td{};
        td.num_groups = ng;
        td.timeout_ns = wait_tmo;
        td.drain_timeout_ns = kDrainTimeoutNs;
        td.call_err = call_err;
        td.g[0] = {tile_start, pair_start, E, rows_cap, (P.d + BNp - 1) / BNp, P.de / moe::tc::BK, P.d,
                   yrows, rowgate};
        td.g[0].counts = counts;
        td.g[0].cap = P.C;
        if (P.ds)
          td.g[1] = {nullptr, nullptr, 1, T, (P.d + BNp - 1) / BNp, P.ds / moe::tc::BK, P.d, ys,
                     nullptr};
        cudaLaunchConfig_t cfg = pair_config<moe::tc::EPI_SCALE_TC>(pair_clusters[1], st, attr, true);
        const cudaError_t le =
            swap ? cudaLaunchKernelEx(&cfg, moe::tc2::tc2_grouped_gemm_kernel<moe::tc::EPI_SCALE_TC, true>,
                                      dn, td)
                 : cudaLaunchKernelEx(&cfg, moe::tc2::tc2_grouped_gemm_kernel<moe::tc::EPI_SCALE_TC>,
                                      dn, td);
        if (le != cudaSuccess) return MOE_ERR_CUDA;
      } else {
        moe::tc::TcParams tp{};
        tp.num_groups = ng;
        tp.timeout_ns = wait_tmo;
        tp.drain_timeout_ns = kDrainTimeoutNs;
        tp.call_err = call_err;
        tp.g[0] = {tile_start, E, rows_cap, (P.d + moe::tc::BN - 1) / moe::tc::BN, P.de / moe::tc::BK,
                   P.d, yrows, rowgate};
        if (P.ds)
          tp.g[1] = {nullptr, 1, T, (P.d + moe::tc::BN - 1) / moe::tc::BN, P.ds / moe::tc::BK,
                     P.d, ys, nullptr};
        launch_tc<moe::tc::EPI_SCALE_TC>(arows, num_sms, st, dn, tp);
      }
      tm.at(11);
      if (launched() != MOE_OK) return MOE_ERR_CUDA;
    }
    }  // bf16 weights
    // (6) combine
    tm.at(12);
    {
      const int nvec = P.d * 2 / 16;
      dim3 grid((T + 7) / 8, (nvec + moe::PERMUTE_CHUNK_VECS - 1) / moe::PERMUTE_CHUNK_VECS);
      launch_pdl(moe::combine_kernel<bf16>, grid, 256, 0, st, yrows, ys, slot, T, P.k, P.d,
                                                      static_cast<bf16*>(y), P.rows_max);
    }
    tm.at(13);
    return launched();
  }

  // fp32 layer: the same pipeline with fp32 FMA expert products
  const float* xf = static_cast<const float*>(x);
  s = launch_route_and_permute<float>(P, dims, xf, W_r, ws, counts, aux, st, tm, wait_tmo);
  if (s != MOE_OK) return s;
  const float* xp = reinterpret_cast<const float*>(ws + P.o_xp);
  float* h = reinterpret_cast<float*>(ws + P.o_h);
  float* yrows = reinterpret_cast<float*>(ws + P.o_yrows);
  float* hs = P.ds ? reinterpret_cast<float*>(ws + P.o_hs) : nullptr;
  float* ys = P.ds ? reinterpret_cast<float*>(ws + P.o_ys) : nullptr;
  const float* sg = static_cast<const float*>(W_shared);
  const size_t sh_n = static_cast<size_t>(P.ds) * P.d;
  const int64_t gy = (P.rows_max > P.T ? P.rows_max : P.T);
  {
    moe::SimtGroup a{}, b{};
    a = {xp, W_g, W_u, static_cast<int64_t>(P.de) * P.d, h, nullptr, tile_start, E, 0, P.de, P.d,
         1};
    if (P.ds) b = {xf, sg, sg + sh_n, 0, hs, nullptr, nullptr, 1, P.T, P.ds, P.d, 1};
    const int nmax = P.de > P.ds ? P.de : P.ds;
    dim3 grid((nmax + moe::SG_BN - 1) / moe::SG_BN,
              static_cast<unsigned>((gy + moe::SG_BM - 1) / moe::SG_BM), P.ds ? 2 : 1);
    tm.at(8);
    launch_pdl(moe::simt_gemm_kernel<float, float, float, moe::EPI_SWIGLU>, grid, 256, 0, st, a, b);
    tm.at(9);
    if (launched() != MOE_OK) return MOE_ERR_CUDA;
  }
  {
    moe::SimtGroup a{}, b{};
    a = {h, W_d, nullptr, static_cast<int64_t>(P.d) * P.de, yrows, rowgate, tile_start, E, 0, P.d,
         P.de, 1};
    if (P.ds) b = {hs, sg + 2 * sh_n, nullptr, 0, ys, nullptr, nullptr, 1, P.T, P.d, P.ds, 1};
    dim3 grid((P.d + moe::SG_BN - 1) / moe::SG_BN,
              static_cast<unsigned>((gy + moe::SG_BM - 1) / moe::SG_BM), P.ds ? 2 : 1);
    tm.at(10);
    launch_pdl(moe::simt_gemm_kernel<float, float, float, moe::EPI_SCALE>, grid, 256, 0, st, a, b);
    tm.at(11);
    if (launched() != MOE_OK) return MOE_ERR_CUDA;
  }
  tm.at(12);
  {
    const int nvec = P.d * 4 / 16;
    dim3 grid((T + 7) / 8, (nvec + moe::PERMUTE_CHUNK_VECS - 1) / moe::PERMUTE_CHUNK_VECS);
    launch_pdl(moe::combine_kernel<float>, grid, 256, 0, st, yrows, ys, slot, T, P.k, P.d,
                                                     static_cast<float*>(y), P.rows_max);
  }
  tm.at(13);
  return launched();
}

}  // namespace

extern "C" {

size_t moe_workspace_size(const moe_dims* dims, int E, int k, float capacity_factor) {
  if (check_dims(dims, E, k, capacity_factor) != MOE_OK) return 0;
  return make_plan(dims, E, k, capacity_factor).total;
}

int64_t moe_capacity(int64_t T, int E, int k, float capacity_factor) {
  if (T < 0 || E < 1 || k < 1) return -1;
  return capacity_of(T, E, k, capacity_factor);
}

moe_status moe_workspace_layout(const moe_dims* dims, int E, int k, float capacity_factor,
                                moe_workspace_layout_t* out) {
  const moe_status s = check_dims(dims, E, k, capacity_factor);
  if (s != MOE_OK) return s;
  if (out == nullptr) return MOE_ERR_INVALID_ARG;
  const Plan P = make_plan(dims, E, k, capacity_factor);
  out->logits = P.o_logits;
  out->topk_idx = P.o_idx;
  out->gates = P.o_gate;
  out->slot_pos = P.o_slot;
  out->probsum = P.o_probsum;
  out->tile_start = P.o_tile_start;
  out->xp = P.o_xp;
  out->h = P.o_h;
  out->yrows = P.o_yrows;
  out->rows_max = P.rows_max;
  out->capacity = P.C;
  out->xscale = P.o_xsc;
  out->hq = P.o_hq;
  out->hscale = P.o_hsc;
  out->status = P.o_status;
  return MOE_OK;
}

moe_status moe_forward(const moe_dims* dims, const void* x, const float* W_r, const void* W_g,
                       const void* W_u, const void* W_d, const void* W_shared, int E, int k,
                       float capacity_factor, void* y, float* aux, int32_t* counts) {
  return forward_impl(dims, x, W_r, W_g, W_u, W_d, W_shared, E, k, capacity_factor, y, aux,
                      counts);
}

moe_status moe_get_device_status(void) {
  // one atomic exchange on the device takes the word out and clears it; the
  // synchronous copy on the legacy default stream then reads what it took
  moe::take_device_error_kernel<<<1, 1>>>();
  if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, moe::g_dev_error_taken, sizeof(int)) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (v & moe::DEVERR_TIMEOUT) return MOE_ERR_DEVICE_TIMEOUT;
  if (v & moe::DEVERR_BOUNDS) return MOE_ERR_DEVICE_BOUNDS;
  return MOE_OK;
}

moe_status moe_forward_host_io(const moe_dims* dims, const void* x_host, void* x_dev,
                               const float* W_r, const void* W_g, const void* W_u, const void* W_d,
                               const void* W_shared, int E, int k, float capacity_factor,
                               void* y_dev, void* y_host, float* aux_dev, float* aux_host,
                               int32_t* counts_dev, int32_t* counts_host) {
  moe_status s = check_dims(dims, E, k, capacity_factor);
  if (s != MOE_OK) return s;
  if (aux_host == nullptr || counts_host == nullptr) return MOE_ERR_INVALID_ARG;
  if (dims->T > 0 && (x_host == nullptr || y_host == nullptr)) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(dims->stream);
  const size_t esz = dims->dtype == MOE_BF16 ? 2 : 4;
  const size_t bytes = static_cast<size_t>(dims->T) * dims->d * esz;
  if (bytes && cudaMemcpyAsync(x_dev, x_host, bytes, cudaMemcpyHostToDevice, st) != cudaSuccess)
    return MOE_ERR_CUDA;
  s = forward_impl(dims, x_dev, W_r, W_g, W_u, W_d, W_shared, E, k, capacity_factor, y_dev,
                   aux_dev, counts_dev);
  if (s != MOE_OK) return s;
  if ((bytes && cudaMemcpyAsync(y_host, y_dev, bytes, cudaMemcpyDeviceToHost, st) != cudaSuccess) ||
      cudaMemcpyAsync(aux_host, aux_dev, sizeof(float), cudaMemcpyDeviceToHost, st) !=
          cudaSuccess ||
      cudaMemcpyAsync(counts_host, counts_dev, sizeof(int32_t) * E, cudaMemcpyDeviceToHost, st) !=
          cudaSuccess)
    return MOE_ERR_CUDA;
  // this call's own status word (in its workspace), read in order on its stream:
  // concurrent callers on other streams neither wait on it nor see its timeouts
  int v = 0;
  if (dims->T > 0) {
    const Plan P = make_plan(dims, E, k, capacity_factor);
    const uint8_t* ws = static_cast<const uint8_t*>(dims->workspace);
    if (cudaMemcpyAsync(&v, ws + P.o_status, sizeof(int), cudaMemcpyDeviceToHost, st) !=
        cudaSuccess)
      return MOE_ERR_CUDA;
  }
  if (cudaStreamSynchronize(st) != cudaSuccess) return MOE_ERR_CUDA;
  return v != 0 ? MOE_ERR_DEVICE_TIMEOUT : MOE_OK;
}

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_DEVICE_TIMEOUT: return "MOE_ERR_DEVICE_TIMEOUT";
    case MOE_ERR_SCRATCH_LIMIT: return "MOE_ERR_SCRATCH_LIMIT";
    case MOE_ERR_DEVICE_BOUNDS: return "MOE_ERR_DEVICE_BOUNDS";
  }
  return "MOE_STATUS_UNKNOWN";
}

moe_status moe_quantize_fp8(const void* w, int32_t dtype, int64_t rows, int32_t cols,
                            uint8_t* codes, float* scales, void* stream) {
  if (w == nullptr || codes == nullptr || scales == nullptr || rows < 0 || cols < 1 ||
      cols % 16 != 0 || (dtype != MOE_BF16 && dtype != MOE_F32) || !aligned(scales, 4) ||
      !aligned(w, 16) || !aligned(codes, 16))
    return MOE_ERR_INVALID_ARG;
  if (rows == 0) return MOE_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const unsigned grid = static_cast<unsigned>(rows < 8192 ? rows : 8192);
  if (dtype == MOE_BF16)
    moe::tcf8::quantize_rows_fp8_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(w), rows, cols, codes, scales);
  else
    moe::tcf8::quantize_rows_fp8_kernel<float><<<grid, 256, 0, st>>>(
        static_cast<const float*>(w), rows, cols, codes, scales);
  return launched();
}

moe_status moe_dequantize_fp8(const uint8_t* codes, const float* scales, int64_t rows,
                              int32_t cols, float* out, void* stream) {
  if (codes == nullptr || scales == nullptr || out == nullptr || rows < 0 || cols < 1 ||
      cols % 16 != 0 || !aligned(codes, 16) || !aligned(out, 16) || !aligned(scales, 4))
    return MOE_ERR_INVALID_ARG;
  if (rows == 0) return MOE_OK;
  const int64_t n = rows * (cols / 16);
  const int64_t blocks = (n + 255) / 256;
  moe::tcf8::dequantize_rows_fp8_kernel<<<static_cast<unsigned>(blocks < 16384 ? blocks : 16384),
                                          256, 0, static_cast<cudaStream_t>(stream)>>>(
      codes, scales, rows, cols, out);
  return launched();
}

moe_status moe_quantize_mxfp4(const void* w, int32_t dtype, int64_t rows, int32_t cols,
                              uint8_t* codes, uint8_t* block_scales, float* row_factors,
                              void* stream) {
  if (w == nullptr || codes == nullptr || block_scales == nullptr || row_factors == nullptr ||
      rows < 0 || cols < 1 || cols % 32 != 0 || (dtype != MOE_BF16 && dtype != MOE_F32) ||
      !aligned(w, 16) || !aligned(codes, 16) || !aligned(row_factors, 4))
    return MOE_ERR_INVALID_ARG;
  if (rows == 0) return MOE_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const unsigned grid = static_cast<unsigned>(rows < 8192 ? rows : 8192);
  if (dtype == MOE_BF16)
    moe::tcf8::quantize_rows_mxfp4_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(w), rows, cols, codes, block_scales, row_factors);
  else
    moe::tcf8::quantize_rows_mxfp4_kernel<float><<<grid, 256, 0, st>>>(
        static_cast<const float*>(w), rows, cols, codes, block_scales, row_factors);
  return launched();
}

moe_status moe_dequantize_mxfp4(const uint8_t* codes, const uint8_t* block_scales,
                                const float* row_factors, int64_t rows, int32_t cols, float* out,
                                void* stream) {
  if (codes == nullptr || block_scales == nullptr || row_factors == nullptr || out == nullptr ||
      rows < 0 || cols < 1 || cols % 32 != 0 || !aligned(codes, 16) || !aligned(out, 16) ||
      !aligned(row_factors, 4))
    return MOE_ERR_INVALID_ARG;
  if (rows == 0) return MOE_OK;
  const int64_t n = rows * (cols / 16);
  const int64_t blocks = (n + 255) / 256;
  moe::tcf8::dequantize_rows_mxfp4_kernel<<<static_cast<unsigned>(blocks < 16384 ? blocks : 16384),
                                            256, 0, static_cast<cudaStream_t>(stream)>>>(
      codes, block_scales, row_factors, rows, cols, out);
  return launched();
}

moe_status moe_forward_no_alloc(const moe_dims* dims, const void* x, const float* W_r,
                                const void* W_g, const void* W_u, const void* W_d,
                                const void* W_shared, int E, int k, float capacity_factor,
                                void* y, float* aux, int32_t* counts) {
  const moe_status s = check_dims(dims, E, k, capacity_factor);
  if (s != MOE_OK) return s;
  if (make_plan(dims, E, k, capacity_factor).total > MOE_NO_ALLOC_WORKSPACE_BYTES)
    return MOE_ERR_SCRATCH_LIMIT;
  void* scratch = nullptr;
  const moe_status ss = no_alloc_scratch(&scratch);
  if (ss != MOE_OK) return ss;
  moe_dims d2 = *dims;
  d2.workspace = scratch;
  d2.workspace_bytes = MOE_NO_ALLOC_WORKSPACE_BYTES;
  return forward_impl(&d2, x, W_r, W_g, W_u, W_d, W_shared, E, k, capacity_factor, y, aux,
                      counts);
}

}  // extern "C"
