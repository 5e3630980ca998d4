// mlg_common.cuh -- small device helpers shared by the build and attention
// kernels of libmlg.so (sm_100a).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "mlg.h"

namespace mlg {

constexpr int kWarp = 32;
constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ unsigned lane_id() { return threadIdx.x & 31u; }

__device__ __forceinline__ unsigned lanemask_lt() {
  return (1u << lane_id()) - 1u;
}

template <typename T>
__device__ __forceinline__ T warp_sum(T v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  return v;
}

template <typename T>
__device__ __forceinline__ T warp_max(T v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(kFull, v, o));
  return v;
}

// inclusive warp scan of ints
__device__ __forceinline__ int warp_incl_scan(int v) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int u = __shfl_up_sync(kFull, v, o);
    if ((int)lane_id() >= o) v += u;
  }
  return v;
}

// floor division and the matching non-negative remainder
__device__ __forceinline__ int floordiv(int a, int b) {
  int q = a / b;
  return (a % b != 0 && ((a < 0) != (b < 0))) ? q - 1 : q;
}

// Order-preserving map of a double to uint64 (for atomicMin / atomicMax).
__device__ __forceinline__ unsigned long long ordered_bits(double v) {
  long long b = __double_as_longlong(v);
  return b >= 0 ? (unsigned long long)b ^ 0x8000000000000000ull : ~(unsigned long long)b;
}
__device__ __forceinline__ double from_ordered_bits(unsigned long long u) {
  long long b = (u & 0x8000000000000000ull) ? (long long)(u ^ 0x8000000000000000ull)
                                             : (long long)~u;
  return __longlong_as_double(b);
}

}  // namespace mlg
