// Shared device/host helpers of libegnn (CUDA path only).
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "egnn.h"

// Device status codes written into egnn_graph::status (first writer wins): the
// EGNN_DEV_* values of egnn.h.
enum : int32_t { EGNN_DEV_OK = 0 };

__device__ __forceinline__ void egnn_flag(int32_t* status, int32_t code) {
  if (status) atomicCAS(status, 0, code);
}

__device__ __forceinline__ float egnn_ld(const float* p, int64_t i) { return __ldg(p + i); }
__device__ __forceinline__ float egnn_ld(const __nv_bfloat16* p, int64_t i) {
  return __bfloat162float(p[i]);
}
__device__ __forceinline__ void egnn_st(float* p, int64_t i, float v) { p[i] = v; }
__device__ __forceinline__ void egnn_st(__nv_bfloat16* p, int64_t i, float v) {
  p[i] = __float2bfloat16_rn(v);
}

__device__ __forceinline__ float egnn_silu(float x) { return x / (1.0f + __expf(-x)); }

#define EGNN_CUDA_TRY(expr)                          \
  do {                                               \
    cudaError_t _e = (expr);                         \
    if (_e != cudaSuccess) return EGNN_ERR_CUDA;     \
  } while (0)

// Per-edge Wigner float count and l-block offsets (same layout as egnn.h).
__host__ __device__ __forceinline__ int egnn_wig_off(int l, int mmax) {
  int o = 0;
  for (int k = 0; k < l; ++k) {
    int mk = k < mmax ? k : mmax;
    o += (2 * mk + 1) * (2 * k + 1);
  }
  return o;
}
// Kept-row index of (l, m): rows ordered by l, then m = -min(l,mmax)..min(l,mmax).
__host__ __device__ __forceinline__ int egnn_row_off(int l, int mmax) {
  int o = 0;
  for (int k = 0; k < l; ++k) o += 2 * (k < mmax ? k : mmax) + 1;
  return o;
}
