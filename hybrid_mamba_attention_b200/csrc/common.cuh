// Internal helpers shared by the libhspec kernels (not part of the C-ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace hspec {

using bf16 = __nv_bfloat16;

// Device error bits (OR-ed into the library's device error word).
enum : int {
  kErrPageOOB = 1,    // a page id outside [0, num_pages)
  kErrCtxOOB = 2,     // a context length < 0 or > max_pages * page_size
  kErrTokenOOB = 4,   // a token id outside [0, vocab)
};

__device__ __forceinline__ float to_f(float v) { return v; }
__device__ __forceinline__ float to_f(bf16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ bf16 from_f<bf16>(float v) { return __float2bfloat16_rn(v); }

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

// Block-wide sum for blockDim.x a multiple of 32 (<= 1024); `red` holds >= 32 floats.
__device__ __forceinline__ float block_sum(float v, float* red) {
  v = warp_sum(v);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31, nw = blockDim.x >> 5;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float t = (l < nw) ? red[l] : 0.f;
  t = warp_sum(t);
  return t;
}

__device__ __forceinline__ float silu(float v) { return v / (1.f + __expf(-v)); }

__device__ __forceinline__ float softplus(float v) { return v > 20.f ? v : log1pf(__expf(v)); }

__device__ __forceinline__ void flag_error(int* err, int bits) {
  if (err) atomicOr(err, bits);
}

// Programmatic dependent launch.  A kernel launched with launch_pdl() may start while
// the previous kernel on its stream is still running: it does its own set-up (shared
// memory barriers, TMEM, descriptor prefetch), then every thread passes pdl_wait()
// -- which returns once the previous grid has completed and its memory is visible --
// before it reads or writes any global memory.  pdl_trigger() lets the next kernel
// launch (its threads still wait for this grid to complete).  Both are no-ops when the
// kernel was launched without the attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---------------------------------------------------------------- host side

// Counts a kernel launch of this library (reported by hspec_launch_count).
void note_launch(int n = 1);

// Records the message of the current thread's most recent failure.
void set_error(const char* fmt, ...);

inline int cdiv(long a, long b) { return (int)((a + b - 1) / b); }

// Whether launch_pdl() sets the programmatic-serialization attribute (HSPEC_PDL=1 in the
// environment; off by default).
bool pdl_enabled();

// Launches `kernel` on `s`, allowed to start before the previous kernel on the stream
// has finished (the kernel must call pdl_wait() before touching global memory).
template <typename... KArgs, typename... Args>
void launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl_enabled() ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

}  // namespace hspec
