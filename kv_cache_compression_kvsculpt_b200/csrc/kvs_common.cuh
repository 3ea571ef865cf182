// Shared device/host helpers of the KVSculpt B200 library.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "kvsculpt.h"

namespace kvs {

// Per-thread text of the last CUDA error (kvs_last_cuda_error).
void set_cuda_error(cudaError_t e, const char *where);
// The same for a driver-API failure (CUresult code).
void set_driver_error(int code, const char *where);
// Counts kernel launches (kvs_launch_count); called once per launch.
void count_launch();
// Cycles a kernel's pipeline wait may spin before the kernel gives up
// (kvs_set_wait_limit; about 2 s by default).
long long wait_limit();
// The default of wait_limit() (the tensor-core kernels' kWaitCycles).
constexpr long long tc_wait_default() { return 4000000000LL; }

#define KVS_CUDA_TRY(expr)                                     \
  do {                                                         \
    cudaError_t _e = (expr);                                   \
    if (_e != cudaSuccess) {                                   \
      ::kvs::set_cuda_error(_e, #expr);                        \
      (void)cudaGetLastError(); /* do not leak into later checks */ \
      return KVS_ECUDA;                                        \
    }                                                          \
  } while (0)

#define KVS_LAUNCH_CHECK(where)                                \
  do {                                                         \
    ::kvs::count_launch();                                     \
    cudaError_t _e = cudaGetLastError();                       \
    if (_e != cudaSuccess) {                                   \
      ::kvs::set_cuda_error(_e, where);                        \
      return KVS_ECUDA;                                        \
    }                                                          \
  } while (0)

// A row-major float matrix family over the problems of a batch: problem b's
// block starts at row `off[b]` (or b * bstride when off is null) of `base`,
// with leading dimension `ld` floats.
struct Mat {
  const float *base;
  const int64_t *off;
  int64_t bstride;
  int64_t ld;
  __device__ __forceinline__ const float *at(int b) const {
    return base + (off ? off[b] : (int64_t)b * bstride) * ld;
  }
};

// A per-problem extent: off[b+1] - off[b], or a fixed value when off is null.
struct Dim {
  const int64_t *off;
  int fixed;
  __device__ __forceinline__ int of(int b) const {
    return off ? (int)(off[b + 1] - off[b]) : fixed;
  }
};

// Selects the problems a launch works on: all of them when p is null, else
// those whose int at p[b * stride] equals want (an L-BFGS phase).
struct Filter {
  const int *p;
  int stride;
  int want;
  __device__ __forceinline__ bool skip(int b) const { return p && p[(int64_t)b * stride] != want; }
};

// Problem geometry read from the host copies of the offsets.
struct HostGeom {
  int B = 0, d = 0;
  int64_t sum_q = 0, sum_z = 0, sum_c = 0;
  int max_q = 0, max_z = 0, max_c = 0;
  int64_t sum_qpad = 0;  // sum over problems of n_q rounded up to 128
  int64_t sum_zpad = 0;  // ... of z rounded up to 128
  int64_t sum_cpad = 0;  // ... of k rounded up to 128
  int64_t ld_a = 0;      // columns of the attention-weight buffer (max_c rounded up to 128)
  int64_t ld_g = 0;      // columns of the Gram / factor buffer (max_c rounded up to 4)
};

int geom_from_batch(const kvs_batch *b, HostGeom *g, bool need_c);

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Deterministic block-wide sum (fixed tree order); `red` holds >= 32 floats.
// Every thread of the block must call it; all receive the total.
__device__ __forceinline__ float block_sum(float v, float *red) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) red[w] = v;
  __syncthreads();
  float t = (threadIdx.x < nw) ? red[threadIdx.x] : 0.f;
  if (w == 0) t = warp_sum(t);
  if (threadIdx.x == 0) red[0] = t;
  __syncthreads();
  float r = red[0];
  __syncthreads();
  return r;
}
__device__ __forceinline__ double block_sum_d(double v, double *red) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  v = warp_sum_d(v);
  __syncthreads();
  if (lane == 0) red[w] = v;
  __syncthreads();
  double t = (threadIdx.x < nw) ? red[threadIdx.x] : 0.0;
  if (w == 0) t = warp_sum_d(t);
  if (threadIdx.x == 0) red[0] = t;
  __syncthreads();
  double r = red[0];
  __syncthreads();
  return r;
}
__device__ __forceinline__ float block_max(float v, float *red) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  v = warp_max(v);
  __syncthreads();
  if (lane == 0) red[w] = v;
  __syncthreads();
  float t = (threadIdx.x < nw) ? red[threadIdx.x] : -INFINITY;
  if (w == 0) t = warp_max(t);
  if (threadIdx.x == 0) red[0] = t;
  __syncthreads();
  float r = red[0];
  __syncthreads();
  return r;
}

inline int64_t align_up(int64_t x, int64_t a) { return (x + a - 1) / a * a; }

// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) once per kernel and device.
cudaError_t set_smem_once_impl(const void *kern, int bytes);
template <class F>
cudaError_t set_smem_once(F *kern, int bytes) {
  return set_smem_once_impl(reinterpret_cast<const void *>(kern), bytes);
}

}  // namespace kvs
