// Device helpers shared by every kernel of libmla: storage-type conversion, the per-device status
// word, RoPE angles and block reductions.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <atomic>
#include <utility>

#include "mla.h"

namespace mla {

// Host-side count of kernel launches made by the library (reported by mla_launch_count).
inline std::atomic<uint64_t> g_launches{0};

// Every kernel of the library is launched through here, so that the launches can be counted.
template <typename... KArgs, typename... Args>
void launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args&&... args) {
  kernel<<<grid, block, smem, st>>>(std::forward<Args>(args)...);
  g_launches.fetch_add(1, std::memory_order_relaxed);
}

// Same, with programmatic dependent launch allowed: the kernel may be scheduled while the previous
// kernel of the stream is still running, and runs its prologue (barrier setup, TMEM allocation) in
// its shadow. Such a kernel calls grid_dependency_wait() before it touches global memory and
// allow_dependents() once its own successor may be scheduled.
template <typename... KArgs, typename... Args>
void launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  g_launches.fetch_add(1, std::memory_order_relaxed);
}
// Waits until the kernels this one depends on have completed and their writes are visible.
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Lets the next kernel of the stream be scheduled (it still waits for this one in its own
// grid_dependency_wait before reading anything).
__device__ __forceinline__ void allow_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Per-device status word: the first error a kernel records wins; mla_check_status() clears it.
__device__ int g_status;

__device__ __forceinline__ void report(int code) { atomicCAS(&g_status, 0, code); }

// ---- storage types ---------------------------------------------------------------------------
template <typename T> struct Store;
template <> struct Store<float> {
  static __device__ __forceinline__ float load(const float* p) { return *p; }
  static __device__ __forceinline__ void store(float* p, float v) { *p = v; }
};
template <> struct Store<__nv_bfloat16> {
  static __device__ __forceinline__ float load(const __nv_bfloat16* p) { return __bfloat162float(*p); }
  static __device__ __forceinline__ void store(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }
};
template <typename T> __device__ __forceinline__ float ld(const T* p) { return Store<T>::load(p); }
template <typename T> __device__ __forceinline__ void st(T* p, float v) { Store<T>::store(p, v); }

// ---- RoPE ------------------------------------------------------------------------------------
// Pair (2i, 2i+1) of a d_r vector turns by pos * base^(-2i/d_r). The angle is formed in double
// precision (at pos ~ 1e5 an fp32 product would already be off by ~1e-2 rad), reduced modulo 2π
// in double by the Cody-Waite method with 2π split into a double head and tail, and the remainder
// (|r| <= π) is evaluated with fp32 sincosf.
__device__ __forceinline__ double rope_inv_freq(int i, int d_r, float base) {
  return exp2(-(2.0 * (double)i / (double)d_r) * log2((double)base));
}
__device__ __forceinline__ void rope_cos_sin_at(int pos, double inv_freq, float* c, float* s) {
  constexpr double kTwoPiHi = 6.283185307179586;        // 2π rounded to double
  constexpr double kTwoPiLo = 2.4492935982947064e-16;   // 2π minus kTwoPiHi
  constexpr double kInvTwoPi = 0.15915494309189535;
  const double a = (double)pos * inv_freq;
  const double k = rint(a * kInvTwoPi);
  const double r = fma(-k, kTwoPiLo, fma(-k, kTwoPiHi, a));
  sincosf((float)r, s, c);
}
__device__ __forceinline__ void rope_cos_sin(int pos, int i, int d_r, float base, float* c, float* s) {
  rope_cos_sin_at(pos, rope_inv_freq(i, d_r, base), c, s);
}
// The same angle and reduction, the remainder evaluated by the SFU (__sincosf): on |r| <= π its
// absolute error is a few 1e-7, far below one rounding of a bf16 output (2^-9 relative), at a few
// instructions instead of sincosf's polynomial. For the bf16-only tensor-core paths.
__device__ __forceinline__ void rope_cos_sin_at_sfu(int pos, double inv_freq, float* c, float* s) {
  constexpr double kTwoPiHi = 6.283185307179586;
  constexpr double kTwoPiLo = 2.4492935982947064e-16;
  constexpr double kInvTwoPi = 0.15915494309189535;
  const double a = (double)pos * inv_freq;
  const double k = rint(a * kInvTwoPi);
  const double r = fma(-k, kTwoPiLo, fma(-k, kTwoPiHi, a));
  __sincosf((float)r, s, c);
}

// ---- reductions --------------------------------------------------------------------------------
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
// Sum over the whole block; `red` needs blockDim.x/32 floats of shared memory.
__device__ __forceinline__ float block_sum(float v, float* red) {
  v = warp_sum(v);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31, nw = blockDim.x >> 5;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float t = (threadIdx.x < (unsigned)nw) ? red[threadIdx.x] : 0.f;
  if (w == 0) t = warp_sum(t);
  if (threadIdx.x == 0) red[0] = t;
  __syncthreads();
  return red[0];
}

// Page-table lookup with a range check: returns the pool row of position p, or -1 (and records
// MLA_ERR_DEVICE_CHECK) when the page id is outside the pool.
__device__ __forceinline__ int64_t cache_row(const int32_t* table_row, int p, int num_pages) {
  int page = table_row[p >> 6];
  if (page < 0 || page >= num_pages) {
    report(MLA_ERR_DEVICE_CHECK);
    return -1;
  }
  return (int64_t)page * 64 + (p & 63);
}

}  // namespace mla
