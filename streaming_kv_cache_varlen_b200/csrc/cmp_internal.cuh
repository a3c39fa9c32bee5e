// Internal definitions shared by the kernels of the Compressor library.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

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
  float* proj;     // [T, 2C]: kv in columns [0, C), raw score in [C, 2C) (non-fused paths)
  int32_t* m_tile; // [B+1] first fused work tile of each sequence (fused path), else null
  float* ystat;    // [n_out, coff, D] pooled halves (fused path)
  float* ylse;     // [n_out, coff, D] log-sum-exp of each half's scores (fused path, coff = 2)
  int32_t* had_sylv;  // rotate: per kHadChunk entries of hadamard, 1 if they are those of
                      // hadamard[0][0] * (Sylvester H_D) (the scheduler kernel checks), else 0;
                      // null: not checked (the dense product is used)
  unsigned* tile_cnt; // fused path in one kernel: per work tile, the arrivals of its items
                      // (zero between calls), else null (scheduler and finish kernels run)
  int single_cta;     // tcgen05 projection: 1 = on single CTAs even where CTA pairs would run
};

// Entries of the hadamard matrix each checking CTA of the scheduler kernel covers.
constexpr int kHadChunk = 65536;
__host__ __device__ inline int had_chunks(int D) { return (D * D + kHadChunk - 1) / kHadChunk; }

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

// Programmatic dependent launch. A kernel launched with launch_chained may start
// while the kernel before it in the stream is still running; it must call
// pdl_wait() before it touches anything that kernel (or an earlier one of the
// same call) writes, and may read the call's inputs before that. pdl_trigger()
// lets the next kernel of the chain be scheduled early. Without the launch
// attribute both are no-ops.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Launch `kernel` on `s` as a programmatic dependent of the previous launch in
// the stream, optionally as clusters of cluster_x CTAs.
template <class... KArgs, class... Args>
inline cudaError_t launch_chained(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                  cudaStream_t s, int cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  int n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster_x > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
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

// One NsaCompressWithCache call (the second workload), device pointers.
struct NsaParams {
  const uint16_t* input;   // paged [tokens = block_num, pbs, N, D] or packed [tokens = T, N, D]
  const uint16_t* weight;  // [cbs, N]
  const int32_t* slot;     // [B]
  const int64_t* len;      // [B] per-batch lengths
  const int32_t* table;    // [B, table_stride] (paged)
  uint16_t* out;           // [result_len, N, D]
  int64_t* starts;         // [B] packed: first row of each batch (-1: a negative length before it)
  unsigned* err;           // device error word
  int B, N, D, cbs, stride, pbs, packed, bf16;
  int64_t tokens, table_stride, result_len;
};

// Kernel launchers (each file defines its own).
cudaError_t launch_sched(const Params& p, cudaStream_t s);
cudaError_t launch_proj_mma(const Params& p, cudaStream_t s);
cudaError_t launch_pool(const Params& p, cudaStream_t s);
cudaError_t launch_finish(const Params& p, cudaStream_t s);
cudaError_t launch_fused(const Params& p, cudaStream_t s, int sm_count);
bool fused_supported(const Params& p);
// Whether the fused path can run as one kernel (metadata and row finish inside):
// no rotation, few enough sequences and work tiles.
bool fused_fold_supported(const Params& p);
constexpr int kFusedTile = 256;  // positions per fused work tile
constexpr int kFusedTileCounters = 8192;  // arrival counters of the one-kernel fused path

}  // namespace cmp
