// The per-row tail of the Compressor shared by the pooling and finish kernels:
// RMSNorm over the D channels, interleaved RoPE on the last rope_head_dim
// channels, the optional Hadamard product and the bf16 store
// ("CANN PyPTO 算子实战", 压缩窗口与状态更新: rms_norm (eps 1e-6, fp32), kv_rope
// through interleaved_rope_2d, then out @ hadamard when rotate).
#pragma once

#include "cmp_internal.cuh"

namespace cmp {

constexpr float kRmsEps = 1e-6f;

// Whether the scheduler kernel found the hadamard matrix to be hadamard[0][0]
// times the Sylvester matrix H_D (every checked chunk passed). Same answer in
// every thread of a call.
__device__ __forceinline__ bool hadamard_is_sylvester(const Params& p) {
  if (!p.rotate || !p.had_sylv) return false;
  bool ok = true;
  for (int i = 0; i < had_chunks(p.D); ++i) ok = ok && p.had_sylv[i] != 0;
  return ok;
}

// z @ (c * H_D) for the D values of a row held 4 per thread (thread t of the
// first D/4: channels 4t .. 4t+3), with the fast Walsh-Hadamard transform in
// natural order: for every bit b of the channel index, the pair (i, i + 2^b)
// with bit b clear in i becomes (u + v, u - v); entry (k, j) of the product of
// those butterflies is (-1)^popcount(k & j), which is H_D. Bits 0-1 are inside
// a thread, 2-6 across the lanes of a warp (shuffles), 7-8 (D = 512) across
// warps through shared memory (xs: 2 D floats, two barriers, which every
// thread of the CTA takes). The result is scaled by c.
__device__ __forceinline__ void fwht_row(float (&z)[4], int D, bool active, float* xs, float c) {
  const float a0 = z[0] + z[1], a1 = z[0] - z[1], a2 = z[2] + z[3], a3 = z[2] - z[3];
  z[0] = a0 + a2;
  z[1] = a1 + a3;
  z[2] = a0 - a2;
  z[3] = a1 - a3;
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float v = __shfl_xor_sync(0xffffffffu, z[i], m);
      z[i] = (lane & m) ? v - z[i] : z[i] + v;
    }
  }
  if (D > 128) {
    const int c0 = threadIdx.x * 4;
#pragma unroll
    for (int r = 0; r < 2; ++r) {  // index bits 7, 8 = bits 0, 1 of the warp
      const int m = 128 << r;
      float* buf = xs + r * D;
      if (active) *reinterpret_cast<float4*>(buf + c0) = make_float4(z[0], z[1], z[2], z[3]);
      __syncthreads();
      if (active) {
        const float4 v = *reinterpret_cast<const float4*>(buf + (c0 ^ m));
        const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) z[i] = (c0 & m) ? vv[i] - z[i] : z[i] + vv[i];
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) z[i] *= c;
}

// What the row tail of channels c .. c+3 of output row n reads besides the
// pooled values: norm_weight, and the RoPE table entries when c lies in the
// last rope_head_dim channels. Loaded before the pooled values are known, so
// these loads overlap the pooling's.
struct RowAux {
  uint2 w;                         // norm_weight[c .. c+3] (bf16)
  __nv_bfloat162 c_lo, c_hi;       // cos[j], cos[j+1] and cos[rope/2 + j], cos[rope/2 + j + 1]
  __nv_bfloat162 s_lo, s_hi;       // the same for sin; j = (c - (D - rope)) / 2
  bool sylv;                       // hadamard_is_sylvester (the same in every thread)
};

// Every thread of the CTA calls it (sylv must agree across the CTA); the
// channel loads are made by the threads that hold channels (active).
__device__ __forceinline__ RowAux load_row_aux(const Params& p, int n, int c, bool active = true) {
  RowAux a{};
  a.sylv = hadamard_is_sylvester(p);
  if (!active) return a;
  a.w = *reinterpret_cast<const uint2*>(p.norm_w + c);
  const int r0 = p.D - p.rope;
  if (c >= r0) {
    const int j = (c - r0) >> 1;  // even: c - r0 is a multiple of 4
    const __nv_bfloat16* cs = p.cos + (int64_t)n * p.rope;
    const __nv_bfloat16* sn = p.sin + (int64_t)n * p.rope;
    a.c_lo = *reinterpret_cast<const __nv_bfloat162*>(cs + j);
    a.c_hi = *reinterpret_cast<const __nv_bfloat162*>(cs + p.rope / 2 + j);
    a.s_lo = *reinterpret_cast<const __nv_bfloat162*>(sn + j);
    a.s_hi = *reinterpret_cast<const __nv_bfloat162*>(sn + p.rope / 2 + j);
  }
  return a;
}

// Threads 0 .. D/4-1 of the CTA hold the pooled values y of channels
// c = 4i .. 4i+3 of output row n (thread i) and their RowAux; any further
// threads only take part in the barriers. red: >= D/128 floats of shared
// memory, zs: >= 2 D floats of shared memory. Every thread of the CTA must
// call it.
__device__ __forceinline__ void finish_row(const Params& p, int n, int c, const float (&y)[4], float* red,
                                           float* zs, const RowAux& aux) {
  const int D = p.D;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = D / 128;
  const bool active = (int)threadIdx.x < D / 4;
  const bool sylv = aux.sylv;
  // RMSNorm over the D channels of the row
  float ss = active ? y[0] * y[0] + y[1] * y[1] + y[2] * y[2] + y[3] * y[3] : 0.f;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if (lane == 0 && warp < nwarps) red[warp] = ss;
  __syncthreads();
  float tot = 0.f;
  for (int i = 0; i < nwarps; ++i) tot += red[i];
  const float inv = rsqrtf(tot / (float)D + kRmsEps);
  if (!active) {  // the Hadamard product's barriers
    if (sylv) {
      float z[4] = {0.f, 0.f, 0.f, 0.f};
      if (D > 128) fwht_row(z, D, false, zs, 0.f);
    } else if (p.rotate) {
      __syncthreads();
    }
    return;
  }
  const __nv_bfloat162 w01 = *reinterpret_cast<const __nv_bfloat162*>(&aux.w.x);
  const __nv_bfloat162 w23 = *reinterpret_cast<const __nv_bfloat162*>(&aux.w.y);
  float z[4] = {y[0] * inv * __low2float(w01), y[1] * inv * __high2float(w01),
                y[2] * inv * __low2float(w23), y[3] * inv * __high2float(w23)};

  // interleaved RoPE on the last rope channels: pair (c + i, c + i + 1) takes
  // table columns j + i/2 and rope/2 + j + i/2
  if (c >= D - p.rope) {
    const float ce[2] = {__low2float(aux.c_lo), __high2float(aux.c_lo)};
    const float co[2] = {__low2float(aux.c_hi), __high2float(aux.c_hi)};
    const float se[2] = {__low2float(aux.s_lo), __high2float(aux.s_lo)};
    const float so[2] = {__low2float(aux.s_hi), __high2float(aux.s_hi)};
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const float ev = z[2 * i], od = z[2 * i + 1];
      z[2 * i] = ev * ce[i] - od * se[i];
      z[2 * i + 1] = od * co[i] + ev * so[i];
    }
  }

  if (sylv) {  // out = z @ hadamard with hadamard = c * H_D: the fast transform
    fwht_row(z, D, true, zs, __bfloat162float(p.had[0]));
  } else if (p.rotate) {  // out = z @ hadamard (dense product, any D x D matrix)
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

// The same with the RowAux loads issued here (only the active threads load).
__device__ __forceinline__ void finish_row(const Params& p, int n, int c, const float (&y)[4], float* red,
                                           float* zs) {
  const RowAux aux = load_row_aux(p, n, c, (int)threadIdx.x < p.D / 4);
  finish_row(p, n, c, y, red, zs, aux);
}


}  // namespace cmp
