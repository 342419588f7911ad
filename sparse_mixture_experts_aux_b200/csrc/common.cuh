// Device helpers shared by the MoE kernels (one translation unit: moe_api.cu).
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace moe {

// Device-side error word of this device, shared by every call on it; read and
// cleared in one atomic exchange by moe_get_device_status(). Each call also has
// a status word of its own in its workspace (cleared by the scan kernel, set by
// a GEMM CTA that gave up), which attributes a timeout to the call that hit it.
// Bit 0: an mbarrier wait in a GEMM kernel gave up after its time limit.
// Bit 1 (builds with MOE_DEBUG only): a device-side bounds check failed and
// the access was skipped.
__device__ int g_dev_error;
__device__ int g_dev_error_taken;  // the value the last exchange took out
constexpr int DEVERR_TIMEOUT = 1;
constexpr int DEVERR_BOUNDS = 2;

// Read and clear the device error word in one step, so that a bit set by a
// kernel between a separate read and clear cannot be lost.
__global__ void take_device_error_kernel() { g_dev_error_taken = atomicExch(&g_dev_error, 0); }

// Programmatic dependent launch: the kernels of a forward pass are launched
// while the previous kernel in the stream is still finishing, so that launch
// latency and set-up (barriers, TMEM, tensor-map prefetch) overlap its tail.
// pdl_wait() blocks until the previous kernel has completed and its memory is
// visible; every kernel calls it in all threads before its first global
// memory access that another kernel (of this pass, the previous pass, or the
// caller's work before it) may make. pdl_launch_dependents() then lets the
// next kernel start launching. Both are no-ops for a plain launch.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Record a failed bounds check (MOE_DEBUG builds).
__device__ __forceinline__ void flag_bounds() { atomicOr(&g_dev_error, DEVERR_BOUNDS); }

// Rows of the permuted buffers are grouped per expert in segments padded to
// this many rows, so that no GEMM M-tile straddles two experts.
constexpr int ROW_TILE = 128;

// Tokens handled by one block of the routing kernel (8 warps x 8 tokens); the
// stable ranks are counted per chunk, so this is also the rank-base granule.
constexpr int ROUTE_CHUNK = 64;
constexpr int ROUTE_WARPS = 8;

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

// 16-byte vector unpack / pack: 8 bf16 or 4 fp32 lanes as float.
template <typename T> struct Vec16;
template <> struct Vec16<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ __forceinline__ static void unpack(const uint4& u, float* f) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 t = __bfloat1622float2(h[i]);
      f[2 * i] = t.x;
      f[2 * i + 1] = t.y;
    }
  }
  __device__ __forceinline__ static uint4 pack(const float* f) {
    uint4 u;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
    return u;
  }
};
template <> struct Vec16<float> {
  static constexpr int N = 4;
  __device__ __forceinline__ static void unpack(const uint4& u, float* f) {
    f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
  }
  __device__ __forceinline__ static uint4 pack(const float* f) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                      __float_as_uint(f[3]));
  }
};

__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}
__device__ __forceinline__ uint4 ld_v4(const void* p) {
  return *reinterpret_cast<const uint4*>(p);
}
__device__ __forceinline__ void st_v4(void* p, const uint4& v) {
  *reinterpret_cast<uint4*>(p) = v;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Cycle budget for a wait limited to `ns` nanoseconds, counted on the SM's own
// cycle counter (a cheap register read, unlike %globaltimer, whose read sits on
// the critical path of every wait that does not succeed at once). 2 cycles per
// ns is above the SM's top clock, so the limit in wall time is never shorter
// than asked; at lower clocks it is longer.
__device__ __forceinline__ uint64_t wait_cycles(unsigned long long ns) {
  return ns > (1ull << 61) ? (1ull << 62) : 2ull * ns;
}

// SiLU(a) = a * sigmoid(a). __expf and the fast divide keep the error within a
// few ulp of fp32 (far inside bf16 and the fp32 path's tolerance); the IEEE
// divide costs the epilogues more instructions than the rest of their math.
// For a << 0 the denominator overflows to inf and the quotient is 0.
__device__ __forceinline__ float silu_f32(float a) { return __fdividef(a, 1.0f + __expf(-a)); }

}  // namespace moe
