// Internal definitions shared by the kernels of the Compressor library.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "cmp.h"

namespace cmp {

// Bits of the device error word (one per workspace, so per device and stream).
enum : unsigned {
  kErrIndex = 1u,    // a bad table entry / block index / cu_seqlens / start_pos
  kErrTimeout = 2u,  // a pipeline wait gave up
};

// Everything a kernel of one call needs, passed by value.
struct Params {
  // operator arguments (device pointers)
  const __nv_bfloat16* x;       // [T, H]
  float* kv_state;              // [block_num, bs, C]
  float* score_state;           // [block_num, bs, C]
  const int32_t* kv_tbl;        // [B, stride]
  const int32_t* sc_tbl;        // [B, stride]
  const __nv_bfloat16* sin;     // [n_out, rope]
  const __nv_bfloat16* cos;     // [n_out, rope]
  const __nv_bfloat16* wkv;     // [C, H]
  const __nv_bfloat16* wgate;   // [C, H]
  const float* ape;             // [ratio, C]
  const __nv_bfloat16* norm_w;  // [D]
  const __nv_bfloat16* had;     // [D, D] or null
  const int32_t* start_pos;     // [B] or null
  const int32_t* cu_in;         // [B+1]
  __nv_bfloat16* out;           // [n_out, D]
  // shapes
  int B, T, H, D, C, coff, ratio, rope, rotate, block_num, bs, stride;
  int n_out;
  // workspace
  unsigned* err;   // device error word
  int32_t* m_cu;   // [B+1] validated token offsets (all 0 when the call is rejected)
  int32_t* m_s;    // [B]   start positions
  int32_t* m_off;  // [B+1] first output row of each sequence
  float* proj;     // [T, 2C]: kv in columns [0, C), score (with ape) in [C, 2C)
};

// Largest b in [0, n] with a[b] <= v, for a non-decreasing a[0..n] with a[0] <= v.
__device__ __forceinline__ int upper_index(const int32_t* __restrict__ a, int n, int v) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(a + mid) <= v) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Pool row of block (p / bs) of sequence b in a table, or -1 (and the error bit)
// if the block index or the entry is out of range.
__device__ __forceinline__ int table_row(const Params& p, const int32_t* __restrict__ tbl, int b,
                                         int pos) {
  const int blk = pos / p.bs;
  if (blk < 0 || blk >= p.stride) {
    atomicOr(p.err, kErrIndex);
    return -1;
  }
  const int r = __ldg(tbl + (int64_t)b * p.stride + blk);
  if (r < 0 || r >= p.block_num) {
    atomicOr(p.err, kErrIndex);
    return -1;
  }
  return r;
}

// The tail threshold: positions >= this are kept in the state after a call
// that ends at position e (exclusive).
__device__ __forceinline__ int tail_threshold(int e, int ratio, int coff) {
  return (e / ratio - coff + 1) * ratio;
}

// Raise a kernel's dynamic shared-memory limit once per device (the attribute
// belongs to the function on the current device).
template <class K>
inline cudaError_t smem_attr_once(K* kernel, size_t bytes, int (&done)[64]) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 64 && done[dev]) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess && dev < 64) done[dev] = 1;
  return e;
}

// Kernel launchers (each file defines its own).
cudaError_t launch_sched(const Params& p, cudaStream_t s);
cudaError_t launch_proj_mma(const Params& p, cudaStream_t s);
cudaError_t launch_pool(const Params& p, cudaStream_t s);

}  // namespace cmp
