// Shared device helpers: the device error word, storage-type conversion,
// warp reductions, and small host helpers used by every entry point.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <utility>

#include "mla.h"

namespace mla {

using bf16 = __nv_bfloat16;

// First device-side error since the last mla_get_device_error: [code, a, b, c].
// One copy per device that loads the library; kernels only ever set it once
// (compare-and-swap from zero), so a later error never hides the first one.
__device__ int g_err[4];

__device__ __forceinline__ void report(int code, int a, int b, int c) {
  if (atomicCAS(&g_err[0], 0, code) == 0) {
    g_err[1] = a;
    g_err[2] = b;
    g_err[3] = c;
  }
}

// ------------------------------------------------------------ launch chaining
// Kernels of a decode step are launched with programmatic stream
// serialization: a kernel may start while the previous one in the stream is
// finishing.  Each such kernel runs its prologue (barriers, TMEM, descriptor
// prefetch), then pdl_wait() before it touches global memory the previous
// kernels write or read, and pdl_trigger() to let the next one start.  Both
// are no-ops for a normal launch.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ------------------------------------------------------------ storage types
template <typename T> struct Store;

template <> struct Store<float> {
  static __device__ __forceinline__ float ld(const float* p) { return *p; }
  static __device__ __forceinline__ float cvt(float v) { return v; }
  static __device__ __forceinline__ void st(float* p, float v) { *p = v; }
  // round a double once to the storage type (nearest, ties to even)
  static __device__ __forceinline__ void st64(float* p, double v) { *p = __double2float_rn(v); }
};

template <> struct Store<bf16> {
  static __device__ __forceinline__ float ld(const bf16* p) { return __bfloat162float(*p); }
  static __device__ __forceinline__ float cvt(bf16 v) { return __bfloat162float(v); }
  static __device__ __forceinline__ void st(bf16* p, float v) { *p = __float2bfloat16_rn(v); }
  static __device__ __forceinline__ void st64(bf16* p, double v) { *p = __double2bfloat16(v); }
};

// E4M3 codes of the FP8 cache (the scale of the row is applied by the reader).
template <> struct Store<__nv_fp8_e4m3> {
  static __device__ __forceinline__ float ld(const __nv_fp8_e4m3* p) { return static_cast<float>(*p); }
  // nearest E4M3, ties to even, straight from the double; saturating at +-448
  static __device__ __forceinline__ void st64(__nv_fp8_e4m3* p, double v) {
    p->__x = __nv_cvt_double_to_fp8(v, __NV_SATFINITE, __NV_E4M3);
  }
};

template <typename T> __device__ __forceinline__ double to_f64(T v);
template <> __device__ __forceinline__ double to_f64<float>(float v) { return (double)v; }
template <> __device__ __forceinline__ double to_f64<bf16>(bf16 v) { return (double)__bfloat162float(v); }

// ------------------------------------------------------------ reductions
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// RoPE inverse frequency of pair i for a rotary width d: theta^(-2i/d), in fp64.
__device__ __forceinline__ double rope_inv_freq(double theta, int i, int d) {
  return pow(theta, -2.0 * (double)i / (double)d);
}

// ------------------------------------------------------------ host helpers
// Kernel launches issued by this library in this process (all devices).
inline std::atomic<long long>& launch_counter() {
  static std::atomic<long long> n{0};
  return n;
}
static inline void note_launch(long long n = 1) { launch_counter().fetch_add(n, std::memory_order_relaxed); }

static inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Launch `kernel` so that it may overlap the tail of the previous kernel in
// `s` (the kernel itself must call pdl_wait() before reading or writing
// anything that kernel touches).
template <typename... KArgs, typename... Args>
static inline cudaError_t launch_chained(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                                         Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  note_launch();
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

static inline int elem_bytes(const mla_config* cfg) { return cfg->dtype == MLA_BF16 ? 2 : 4; }

static inline float scale_of(const mla_config* cfg) {
  return cfg->softmax_scale > 0.f ? cfg->softmax_scale
                                  : (float)(1.0 / sqrt((double)(cfg->qk_nope + cfg->d_r)));
}

}  // namespace mla
