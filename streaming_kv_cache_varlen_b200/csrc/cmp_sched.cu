// Varlen scheduler: turns cu_seqlens / start_pos into the per-sequence metadata
// the projection and pooling kernels read (validated token offsets, start
// positions and first output rows). It runs on the device so a call needs no
// host synchronisation; this is the role the value-dependent AICPU scheduler
// plays on "NPU DeepSeek-V4 Ascend C 融合算子优化" (AICPU Scheduler).
//
// With rotation it also checks, once per call, whether the hadamard matrix is
// a scaled Sylvester matrix (classify_hadamard).
//
// Output-row layout ("CANN PyPTO 算子实战", 返回值说明 fixes only the row count
// min(T, T//ratio + B)): sequence b reserves cap_b = min(L_b, L_b / ratio + 1)
// rows after those of sequences 0..b-1. A sequence covering positions [s, e)
// completes e/ratio - s/ratio <= cap_b windows, and sum(cap_b) <= the row count.
#include "cmp_internal.cuh"

namespace cmp {
namespace {

constexpr int kThreads = 1024;

__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_tot, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += n;
  }
  if (lane == 31) warp_tot[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    int w = lane < (kThreads / 32) ? warp_tot[lane] : 0;
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += n;
    }
    warp_tot[lane] = wi - w;  // exclusive prefix of warp totals
    if (lane == 31) *total = wi;
  }
  __syncthreads();
  const int r = warp_tot[warp] + inc - v;
  __syncthreads();
  return r;
}

// CTAs 1.. of a rotating call: is the hadamard matrix c * H_D in natural
// Sylvester order, c = hadamard[0][0]? Entry (k, j) of H_D is
// (-1)^popcount(k & j), so its bf16 pattern must be c's with the sign bit
// flipped by the parity of popcount(k & j). Each CTA checks kHadChunk entries
// and writes its verdict; the pooling kernels use the in-register fast
// Walsh-Hadamard transform only if every chunk passed.
__device__ void classify_hadamard(const Params& p, int chunk) {
  const int D = p.D;
  const int64_t lo = (int64_t)chunk * kHadChunk;
  const int64_t hi = min((int64_t)D * D, lo + kHadChunk);
  const uint16_t* h = reinterpret_cast<const uint16_t*>(p.had);
  const uint32_t c = __ldg(h);
  bool ok = true;
  for (int64_t e = lo + threadIdx.x * 4; e < hi; e += kThreads * 4) {  // 4 entries of one row
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(h + e));
    const int k = (int)(e / D), j0 = (int)(e % D);
    const uint32_t got[4] = {v.x & 0xFFFFu, v.x >> 16, v.y & 0xFFFFu, v.y >> 16};
#pragma unroll
    for (int i = 0; i < 4; ++i) ok = ok && got[i] == (c ^ ((uint32_t)(__popc(k & (j0 + i)) & 1) << 15));
  }
  ok = __syncthreads_and(ok);
  if (threadIdx.x == 0) p.had_sylv[chunk] = ok ? 1 : 0;
}

__global__ void __launch_bounds__(kThreads) sched_kernel(Params p) {
  __shared__ int bad;
  __shared__ int warp_tot[32];
  __shared__ int chunk_total;
  pdl_trigger();  // the projection kernel may start streaming its inputs now
  if (blockIdx.x > 0) {
    classify_hadamard(p, blockIdx.x - 1);
    return;
  }
  if (threadIdx.x == 0) bad = 0;
  __syncthreads();
  const int B = p.B;
  // 1) validate: cu rises from 0 to T, start_pos >= 0, positions fit in int32
  for (int b = threadIdx.x; b <= B; b += kThreads) {
    const int c = p.cu_in[b];
    bool ok = c >= 0 && c <= p.T;
    if (b == 0) ok = ok && c == 0;
    if (b == B) ok = ok && c == p.T;
    if (b < B) {
      const int c1 = p.cu_in[b + 1];
      const int s = p.start_pos ? p.start_pos[b] : 0;
      ok = ok && c1 >= c && s >= 0 && (int64_t)s + (int64_t)(c1 - c) <= (int64_t)INT32_MAX;
    }
    if (!ok) atomicOr(&bad, 1);
  }
  __syncthreads();
  const bool rejected = bad != 0;
  if (rejected && threadIdx.x == 0) atomicOr(p.err, kErrIndex);
  // 2) metadata; a rejected call gets empty sequences (every output row 0).
  // Fused path: sequence b's work tiles cover positions from its first
  // window's start (start_pos rounded down to the ratio) to its end.
  int carry = 0, tcarry = 0;
  for (int base = 0; base < B; base += kThreads) {
    const int b = base + threadIdx.x;
    int c = 0, s = 0, cap = 0, tiles = 0;
    if (b < B && !rejected) {
      c = p.cu_in[b];
      const int L = p.cu_in[b + 1] - c;
      s = p.start_pos ? p.start_pos[b] : 0;
      cap = min(L, L / p.ratio + 1);
      if (L > 0) tiles = (s + L - (s / p.ratio) * p.ratio + kFusedTile - 1) / kFusedTile;
    }
    const int ex = block_exclusive_scan(cap, warp_tot, &chunk_total);
    const int cap_total = chunk_total;
    const int tex = block_exclusive_scan(tiles, warp_tot, &chunk_total);
    if (b < B) {
      p.m_cu[b] = c;
      p.m_s[b] = s;
      p.m_off[b] = carry + ex;
      if (p.m_tile) p.m_tile[b] = tcarry + tex;
    }
    carry += cap_total;
    tcarry += chunk_total;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    p.m_cu[B] = rejected ? 0 : p.T;
    p.m_off[B] = carry;
    if (p.m_tile) p.m_tile[B] = tcarry;
  }
}

}  // namespace

cudaError_t launch_sched(const Params& p, cudaStream_t s) {
  const int grid = 1 + ((p.rotate && p.had_sylv) ? had_chunks(p.D) : 0);
  sched_kernel<<<grid, kThreads, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace cmp
