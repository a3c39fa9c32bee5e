// Finish kernel of the fused prefill path: one CTA of D/4 threads per output
// row turns the fused kernel's pooled halves into the output row.
//
// coff = 1: y is the pooled row. coff = 2: the window's softmax runs over the
// previous window's 4 rows (half 0, columns [0, D)) and its own 4 rows (half 1,
// columns [D, 2D)) ("compressor torch_extension API", 计算公式 2-5). The fused
// kernel pooled each 4-row half separately and kept the log of its exp-sum, so
//   y = (y_a e^{lse_a} + y_b e^{lse_b}) / (e^{lse_a} + e^{lse_b}),
// which is the 8-row softmax-weighted sum exactly. Half 0 of window w was
// pooled as part of window w-1's row; for the first window of a sequence in a
// call it comes from the paged state, and window 0 has none ("CANN PyPTO 算子实战",
// 压缩窗口与状态更新: the missing previous window counts as 0 / -inf).
// Then RMSNorm, RoPE, Hadamard and the bf16 store (cmp_rowpost.cuh).
#include "cmp_internal.cuh"
#include "cmp_rowpost.cuh"

namespace cmp {
namespace {

constexpr int kMaxStagedSeqs = 256;

__global__ void __launch_bounds__(128) finish_kernel(Params p) {
  __shared__ float red[32];
  __shared__ float zs[1024];  // 2 D floats: the Hadamard product's exchange buffers
  __shared__ int32_t off_s[kMaxStagedSeqs + 1];
  const int n = blockIdx.x;
  const int D = p.D, r = p.ratio;
  const int c = threadIdx.x * 4;
  pdl_wait();

  int b;
  if (p.B <= kMaxStagedSeqs) {
    for (int i = threadIdx.x; i <= p.B; i += blockDim.x) off_s[i] = p.m_off[i];
    __syncthreads();
    int lo = 0, hi = p.B;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (off_s[mid] <= n) lo = mid; else hi = mid - 1;
    }
    b = lo;
  } else {
    b = upper_index(p.m_off, p.B, n);
  }
  int w = -1, k = 0, s = 0;
  if (b < p.B) {
    s = p.m_s[b];
    const int e = s + (p.m_cu[b + 1] - p.m_cu[b]);
    k = n - p.m_off[b];
    if (k < e / r - s / r) w = s / r + k;
  }
  if (w < 0) {
    *reinterpret_cast<uint2*>(p.out + (int64_t)n * D + c) = make_uint2(0u, 0u);
    return;
  }
  const RowAux aux = load_row_aux(p, n, c);  // in flight while the halves load

  float y[4];
  if (p.coff == 1) {
    const float4 v = *reinterpret_cast<const float4*>(p.ystat + (int64_t)n * D + c);
    y[0] = v.x; y[1] = v.y; y[2] = v.z; y[3] = v.w;
  } else {
    const int64_t rb = ((int64_t)n * 2 + 1) * D + c;
    const float4 yb = *reinterpret_cast<const float4*>(p.ystat + rb);
    const float4 lb = *reinterpret_cast<const float4*>(p.ylse + rb);
    float ya[4] = {0.f, 0.f, 0.f, 0.f}, la[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
    if (w > 0 && k > 0) {  // half 0 of window w-1, pooled with the previous row
      const int64_t ra = ((int64_t)(n - 1) * 2) * D + c;
      const float4 v = *reinterpret_cast<const float4*>(p.ystat + ra);
      const float4 g = *reinterpret_cast<const float4*>(p.ylse + ra);
      ya[0] = v.x; ya[1] = v.y; ya[2] = v.z; ya[3] = v.w;
      la[0] = g.x; la[1] = g.y; la[2] = g.z; la[3] = g.w;
    } else if (w > 0) {  // window w-1 lies wholly before start_pos: pool it from the state
      float m[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY}, l[4] = {0.f, 0.f, 0.f, 0.f},
            a[4] = {0.f, 0.f, 0.f, 0.f};
      for (int j = 0; j < r; ++j) {
        const int q = (w - 1) * r + j;
        const int rk = table_row(p, p.kv_tbl, b, q);
        const int rs = table_row(p, p.sc_tbl, b, q);
        if (rk < 0 || rs < 0) continue;
        const float4 kv = *reinterpret_cast<const float4*>(p.kv_state + ((int64_t)rk * p.bs + q % p.bs) * p.C + c);
        const float4 sc = *reinterpret_cast<const float4*>(p.score_state + ((int64_t)rs * p.bs + q % p.bs) * p.C + c);
        const float kk[4] = {kv.x, kv.y, kv.z, kv.w}, zz[4] = {sc.x, sc.y, sc.z, sc.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float mn = fmaxf(m[i], zz[i]);
          const float f = __expf(m[i] - mn), pz = __expf(zz[i] - mn);
          l[i] = l[i] * f + pz;
          a[i] = a[i] * f + pz * kk[i];
          m[i] = mn;
        }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (l[i] > 0.f) {
          ya[i] = a[i] / l[i];
          la[i] = m[i] + __logf(l[i]);
        }
    }
    const float ybv[4] = {yb.x, yb.y, yb.z, yb.w}, lbv[4] = {lb.x, lb.y, lb.z, lb.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float M = fmaxf(la[i], lbv[i]);
      const float wa = __expf(la[i] - M), wb = __expf(lbv[i] - M);
      y[i] = (ya[i] * wa + ybv[i] * wb) / (wa + wb);
    }
  }
  finish_row(p, n, c, y, red, zs, aux);
}

}  // namespace

cudaError_t launch_finish(const Params& p, cudaStream_t s) {
  if (p.n_out <= 0) return cudaSuccess;
  return launch_chained(finish_kernel, dim3(p.n_out), dim3(p.D / 4), 0, s, 1, p);
}

}  // namespace cmp
