// Shared device/host helpers of libegnn (CUDA path only).
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "egnn.h"

// Device status codes written into egnn_graph::status (first writer wins).
enum : int32_t {
  EGNN_DEV_OK = 0,
  EGNN_DEV_BAD_POSITION = 1,      // coordinate outside [0, box) or not finite
  EGNN_DEV_SEGMENT_TOO_LARGE = 2, // more than the per-atom edge limit
  EGNN_DEV_INDEX_RANGE = 3,       // a source index outside [0, n_atoms)
  EGNN_DEV_COUNT_MISMATCH = 4,    // fill pass disagreed with count pass
  EGNN_DEV_EDGE_OVERFLOW = 5,     // more than 2^31-1 edges
  EGNN_DEV_WAIT_TIMEOUT = 6,      // a bounded wait in a pipelined kernel ran out
  EGNN_DEV_BAD_GRAPH = 7          // row_ptr not monotone / out of range
};

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
