// The per-row tail of the Compressor shared by the pooling and finish kernels:
// RMSNorm over the D channels, interleaved RoPE on the last rope_head_dim
// channels, the optional Hadamard product and the bf16 store
// ("CANN PyPTO 算子实战", 压缩窗口与状态更新: rms_norm (eps 1e-6, fp32), kv_rope
// through interleaved_rope_2d, then out @ hadamard when rotate).
#pragma once

#include "cmp_internal.cuh"

namespace cmp {

constexpr float kRmsEps = 1e-6f;

// Threads 0 .. D/4-1 of the CTA hold the pooled values y of channels
// c = 4i .. 4i+3 of output row n (thread i); any further threads only take part
// in the barriers. red: >= D/128 floats of shared memory, zs: >= D floats of
// shared memory. Every thread of the CTA must call it.
__device__ __forceinline__ void finish_row(const Params& p, int n, int c, const float (&y)[4], float* red,
                                           float* zs) {
  const int D = p.D;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = D / 128;
  const bool active = (int)threadIdx.x < D / 4;
  // RMSNorm over the D channels of the row
  float ss = active ? y[0] * y[0] + y[1] * y[1] + y[2] * y[2] + y[3] * y[3] : 0.f;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if (lane == 0 && warp < nwarps) red[warp] = ss;
  __syncthreads();
  float tot = 0.f;
  for (int i = 0; i < nwarps; ++i) tot += red[i];
  const float inv = rsqrtf(tot / (float)D + kRmsEps);
  if (!active) {
    if (p.rotate) __syncthreads();  // the Hadamard product's barrier
    return;
  }
  const uint2 wraw = *reinterpret_cast<const uint2*>(p.norm_w + c);
  const __nv_bfloat162 w01 = *reinterpret_cast<const __nv_bfloat162*>(&wraw.x);
  const __nv_bfloat162 w23 = *reinterpret_cast<const __nv_bfloat162*>(&wraw.y);
  float z[4] = {y[0] * inv * __low2float(w01), y[1] * inv * __high2float(w01),
                y[2] * inv * __low2float(w23), y[3] * inv * __high2float(w23)};

  // interleaved RoPE on the last rope channels
  const int r0 = D - p.rope;
  if (c >= r0) {
    const int half = p.rope / 2;
    const __nv_bfloat16* cs = p.cos + (int64_t)n * p.rope;
    const __nv_bfloat16* sn = p.sin + (int64_t)n * p.rope;
#pragma unroll
    for (int i = 0; i < 4; i += 2) {
      const int j = (c + i - r0) >> 1;
      const float ce = __bfloat162float(cs[j]), se = __bfloat162float(sn[j]);
      const float co = __bfloat162float(cs[half + j]), so = __bfloat162float(sn[half + j]);
      const float ev = z[i], od = z[i + 1];
      z[i] = ev * ce - od * se;
      z[i + 1] = od * co + ev * so;
    }
  }

  if (p.rotate) {  // out = z @ hadamard (dense product, any D x D matrix)
#pragma unroll
    for (int i = 0; i < 4; ++i) zs[c + i] = z[i];
    __syncthreads();
    float o[4] = {0.f, 0.f, 0.f, 0.f};
    for (int k = 0; k < D; ++k) {
      const float zk = zs[k];
      const uint2 hr = *reinterpret_cast<const uint2*>(p.had + (int64_t)k * D + c);
      const __nv_bfloat162 h01 = *reinterpret_cast<const __nv_bfloat162*>(&hr.x);
      const __nv_bfloat162 h23 = *reinterpret_cast<const __nv_bfloat162*>(&hr.y);
      o[0] = fmaf(zk, __low2float(h01), o[0]);
      o[1] = fmaf(zk, __high2float(h01), o[1]);
      o[2] = fmaf(zk, __low2float(h23), o[2]);
      o[3] = fmaf(zk, __high2float(h23), o[3]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) z[i] = o[i];
  }

  __nv_bfloat162 o01 = __floats2bfloat162_rn(z[0], z[1]);
  __nv_bfloat162 o23 = __floats2bfloat162_rn(z[2], z[3]);
  uint2 v;
  v.x = *reinterpret_cast<uint32_t*>(&o01);
  v.y = *reinterpret_cast<uint32_t*>(&o23);
  *reinterpret_cast<uint2*>(p.out + (int64_t)n * D + c) = v;
}


}  // namespace cmp
