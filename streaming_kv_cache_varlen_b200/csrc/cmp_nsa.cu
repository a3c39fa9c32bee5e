// NsaCompressWithCache: for each batch whose length just reached a compression
// step, the weighted sum of its last compress_block_size cached tokens, written
// to its slot of the output cache ("CANN ops-transformer 算子解析
// NsaCompressWithCache", 计算公式 and 算法流程: trigger s >= compress_block_size
// and (s - compress_block_size) % stride == 0; tokens s - compress_block_size
// .. s - 1 found through the block table (paged) or packed by batch (TND);
// values cast to fp32, multiplied by weight[j, n], summed, cast back to
// fp16 / bf16 with round-to-nearest-even).
//
// HBM bound: every byte of the window's tokens is read once. Grid = (batch,
// chunk of the N*D plane); a thread owns 8 consecutive elements (16 bytes, one
// head since D is a multiple of 16) and streams the window's tokens with 8
// 16-byte loads in flight, so a warp reads 512 contiguous bytes of one token
// per instruction. The sum runs over the tokens in order (deterministic).
#include "cmp_internal.cuh"

#include <cuda_fp16.h>

namespace cmp {

namespace {

constexpr int kThreads = 128;
constexpr int kElems = 8;  // per thread

__device__ __forceinline__ float to_f32(uint16_t v, bool bf16) {
  return bf16 ? __bfloat162float(__ushort_as_bfloat16(v)) : __half2float(__ushort_as_half(v));
}

__device__ __forceinline__ uint16_t from_f32(float v, bool bf16) {
  return bf16 ? __bfloat16_as_ushort(__float2bfloat16_rn(v)) : __half_as_ushort(__float2half_rn(v));
}

__global__ void __launch_bounds__(kThreads) nsa_kernel(NsaParams p) {
  const int b = blockIdx.x;
  const int64_t s = p.len[b];
  if (s < p.cbs || (s - p.cbs) % p.stride != 0) return;  // not a compression step
  __shared__ int ok;
  __shared__ int64_t row0;  // packed: the batch's first row
  if (threadIdx.x == 0) {
    const int slot = p.slot[b];
    bool good = slot >= 0 && slot < p.result_len;
    int64_t start = 0;
    if (p.packed) {
      for (int i = 0; i < b; ++i) {
        const int64_t li = p.len[i];
        good = good && li >= 0;
        start += li > 0 ? li : 0;
      }
      good = good && start + s <= p.tokens;
    } else {
      // the window spans at most two pages (cbs <= page size)
      const int64_t first = s - p.cbs, last = s - 1;
      for (int64_t pg = first / p.pbs; pg <= last / p.pbs; ++pg) {
        const int32_t blk = pg < p.table_stride ? p.table[(int64_t)b * p.table_stride + pg] : -1;
        good = good && blk >= 0 && blk < p.tokens;
      }
    }
    if (!good) atomicOr(p.err, kErrIndex);
    ok = good ? 1 : 0;
    row0 = start;
  }
  __syncthreads();
  if (!ok) return;

  const int64_t plane = (int64_t)p.N * p.D;
  const int64_t e0 = ((int64_t)blockIdx.y * kThreads + threadIdx.x) * kElems;
  if (e0 >= plane) return;
  const int n = (int)(e0 / p.D);
  const bool bf = p.bf16 != 0;
  const int64_t first = s - p.cbs;
  float acc[kElems];
#pragma unroll
  for (int k = 0; k < kElems; ++k) acc[k] = 0.f;
  for (int j0 = 0; j0 < p.cbs; j0 += 8) {  // cbs is a multiple of 16
    uint4 v[8];
    float w[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int64_t pos = first + j0 + u;
      int64_t row;
      if (p.packed) {
        row = row0 + pos;
      } else {
        const int32_t blk = p.table[(int64_t)b * p.table_stride + pos / p.pbs];
        row = (int64_t)blk * p.pbs + pos % p.pbs;
      }
      v[u] = __ldg(reinterpret_cast<const uint4*>(p.input + row * plane + e0));
      w[u] = to_f32(__ldg(p.weight + (int64_t)(j0 + u) * p.N + n), bf);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const uint32_t q[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        acc[2 * k] = fmaf(to_f32((uint16_t)(q[k] & 0xFFFFu), bf), w[u], acc[2 * k]);
        acc[2 * k + 1] = fmaf(to_f32((uint16_t)(q[k] >> 16), bf), w[u], acc[2 * k + 1]);
      }
    }
  }
  uint32_t o[4];
#pragma unroll
  for (int k = 0; k < 4; ++k)
    o[k] = (uint32_t)from_f32(acc[2 * k], bf) | ((uint32_t)from_f32(acc[2 * k + 1], bf) << 16);
  *reinterpret_cast<uint4*>(p.out + (int64_t)p.slot[b] * plane + e0) = make_uint4(o[0], o[1], o[2], o[3]);
}

}  // namespace

cudaError_t launch_nsa(const NsaParams& p, cudaStream_t s) {
  const int64_t plane = (int64_t)p.N * p.D;
  const unsigned chunks = (unsigned)((plane / kElems + kThreads - 1) / kThreads);
  nsa_kernel<<<dim3((unsigned)p.B, chunks), kThreads, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace cmp
