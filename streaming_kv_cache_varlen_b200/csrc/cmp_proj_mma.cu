// Dual projection with warp-level mma.sync (bf16 x bf16 -> fp32).
//
//   proj[t][n] = sum_k x[t][k] * W[n][k],  W = wkv (n < C) or wgate (n >= C)
// ("compressor torch_extension API", 计算公式 1-2). The epilogue also writes
// the state tail rows (positions p >= (e/ratio - coff + 1)*ratio of their
// sequence) into the paged fp32 kv_state / score_state, the score rows with
// ape[p mod ratio] added (the pooling kernel adds ape to the projection rows
// it reads, so the projection buffer holds raw scores).
//
// This is the portable tensor-core path (mma.sync runs on every architecture
// since sm_80); the sm_100a tcgen05 kernel is the fast prefill path and this one
// serves as its cross-check and as the path for shapes that kernel does not take.
#include "cmp_internal.cuh"

namespace cmp {
namespace {

constexpr int BM = 128, BN = 128, BK = 32, STAGES = 3, PAD = 8;
constexpr int LDS = BK + PAD;  // smem row pitch in bf16 elements (80 bytes: ldmatrix conflict-free)
constexpr int kThreads = 256;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;  // zero-fill rows past the end
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(n));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void mma_bf16(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Epilogue for two adjacent columns (n, n+1) of token t.
__device__ __forceinline__ void store_pair(const Params& p, int t, int n, float v0, float v1) {
  if (t >= p.T) return;
  const int b = upper_index(p.m_cu, p.B, t);
  const bool seq = b < p.B;
  int pos = 0, thr = 0;
  if (seq) {
    const int s = p.m_s[b];
    pos = s + (t - p.m_cu[b]);
    const int e = s + (p.m_cu[b + 1] - p.m_cu[b]);
    thr = tail_threshold(e, p.ratio, p.coff);
  }
  const bool score = n >= p.C;
  const int col = score ? n - p.C : n;
  *reinterpret_cast<float2*>(p.proj + (int64_t)t * (2 * p.C) + n) = make_float2(v0, v1);
  if (seq && pos >= thr) {
    if (score) {  // the state holds score + ape
      const float2 a = *reinterpret_cast<const float2*>(p.ape + (int64_t)(pos % p.ratio) * p.C + col);
      v0 += a.x;
      v1 += a.y;
    }
    const int r = table_row(p, score ? p.sc_tbl : p.kv_tbl, b, pos);
    if (r >= 0) {
      float* st = score ? p.score_state : p.kv_state;
      *reinterpret_cast<float2*>(st + ((int64_t)r * p.bs + pos % p.bs) * p.C + col) =
          make_float2(v0, v1);
    }
  }
}

__global__ void __launch_bounds__(kThreads) proj_mma_kernel(Params p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  pdl_wait();
  pdl_trigger();
  __nv_bfloat16* As = reinterpret_cast<__nv_bfloat16*>(smem_raw);
  __nv_bfloat16* Bs = As + STAGES * BM * LDS;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int wm = warp >> 2, wn = warp & 3;  // 2 x 4 warps, warp tile 64 x 32
  const int t0 = blockIdx.x * BM;
  const int n0 = blockIdx.y * BN;
  const __nv_bfloat16* W = n0 < p.C ? p.wkv + (int64_t)n0 * p.H : p.wgate + (int64_t)(n0 - p.C) * p.H;
  const int K = p.H;
  const int ktiles = K / BK;

  auto load_stage = [&](int stage, int kt) {
    const int k0 = kt * BK;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int c = tid + i * kThreads;  // 512 chunks of 16 bytes per operand
      const int r = c >> 2, kc = (c & 3) * 8;
      const int t = t0 + r;
      const bool ok = t < p.T;
      const __nv_bfloat16* src = p.x + (int64_t)(ok ? t : 0) * K + k0 + kc;
      cp_async16(smem_u32(As + (stage * BM + r) * LDS + kc), src, ok);
      cp_async16(smem_u32(Bs + (stage * BN + r) * LDS + kc), W + (int64_t)r * K + k0 + kc, true);
    }
  };

  float acc[4][4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[i][j][e] = 0.f;

#pragma unroll
  for (int s = 0; s < STAGES - 1; ++s) {
    if (s < ktiles) load_stage(s, s);
    asm volatile("cp.async.commit_group;\n" ::);
  }

  for (int kt = 0; kt < ktiles; ++kt) {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(STAGES - 2));
    __syncthreads();
    const int nk = kt + STAGES - 1;
    if (nk < ktiles) load_stage(nk % STAGES, nk);
    asm volatile("cp.async.commit_group;\n" ::);
    const int st = kt % STAGES;
#pragma unroll
    for (int kk = 0; kk < BK; kk += 16) {
      uint32_t a[4][4], bfr[2][4];
#pragma unroll
      for (int mi = 0; mi < 4; ++mi) {
        const int r = wm * 64 + mi * 16 + (lane & 15);
        const int c = kk + (lane >> 4) * 8;
        ldsm_x4(smem_u32(As + (st * BM + r) * LDS + c), a[mi][0], a[mi][1], a[mi][2], a[mi][3]);
      }
#pragma unroll
      for (int nj = 0; nj < 2; ++nj) {
        const int r = wn * 32 + nj * 16 + (lane & 7) + (lane >> 4) * 8;
        const int c = kk + ((lane >> 3) & 1) * 8;
        ldsm_x4(smem_u32(Bs + (st * BN + r) * LDS + c), bfr[nj][0], bfr[nj][1], bfr[nj][2],
                bfr[nj][3]);
      }
#pragma unroll
      for (int mi = 0; mi < 4; ++mi)
#pragma unroll
        for (int ni = 0; ni < 4; ++ni)
          mma_bf16(acc[mi][ni], a[mi], bfr[ni >> 1][(ni & 1) * 2], bfr[ni >> 1][(ni & 1) * 2 + 1]);
    }
  }
  asm volatile("cp.async.wait_group 0;\n" ::);

  const int g = lane >> 2, q = lane & 3;
#pragma unroll
  for (int mi = 0; mi < 4; ++mi)
#pragma unroll
    for (int ni = 0; ni < 4; ++ni) {
      const int t = t0 + wm * 64 + mi * 16 + g;
      const int n = n0 + wn * 32 + ni * 8 + 2 * q;
      store_pair(p, t, n, acc[mi][ni][0], acc[mi][ni][1]);
      store_pair(p, t + 8, n, acc[mi][ni][2], acc[mi][ni][3]);
    }
}

}  // namespace

cudaError_t launch_proj_mma(const Params& p, cudaStream_t s) {
  const size_t smem = (size_t)STAGES * (BM + BN) * LDS * sizeof(__nv_bfloat16);
  static int configured[64] = {0};
  const cudaError_t e = smem_attr_once(proj_mma_kernel, smem, configured);
  if (e != cudaSuccess) return e;
  dim3 grid((p.T + BM - 1) / BM, (2 * p.C) / BN);
  return launch_chained(proj_mma_kernel, grid, dim3(kThreads), smem, s, 1, p);
}

}  // namespace cmp
