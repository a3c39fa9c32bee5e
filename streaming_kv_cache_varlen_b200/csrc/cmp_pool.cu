// Pooling and epilogue: one CTA per output row, D/4 threads, each thread owns
// four consecutive channels.
//
// For the window the row holds:
//  * gather its rows: coff = 1: the ratio rows of the window; coff = 2: the
//    ratio rows of the previous window, columns [0, D), then the ratio rows of
//    the window, columns [D, 2D); the first window of a sequence has no
//    previous rows ("compressor torch_extension API", 计算公式 2-4; "CANN PyPTO
//    算子实战", 压缩窗口与状态更新: 0 and -inf fill the missing previous window).
//    A row at a position inside this call comes from the projection buffer
//    (raw score, plus ape[position mod ratio] here), an earlier one from the
//    paged state (which already holds score + ape);
//  * per-channel softmax over those rows weighting a sum of the kv rows
//    (计算公式 3-5), as an online (running max) softmax in fp32;
//  * RMSNorm, eps 1e-6, times norm_weight; interleaved RoPE on the last
//    rope_head_dim channels (pair (2j, 2j+1) uses table columns j and
//    rope_head_dim/2 + j); optional product with the hadamard matrix
//    ("CANN PyPTO 算子实战", 压缩窗口与状态更新, 算子级辅助函数, kernel 派发逻辑);
//  * bf16 round-to-nearest-even store. Rows that hold no window are stored as 0
//    ("CANN PyPTO 算子实战", 返回值说明).
#include "cmp_internal.cuh"
#include "cmp_rowpost.cuh"

namespace cmp {
namespace {

__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }

__device__ __forceinline__ void online(float& m, float& l, float& a, float z, float k) {
  const float mn = fmaxf(m, z);
  const float sc = __expf(m - mn);  // m = -inf on the first row: exp(-inf) = 0
  const float pz = __expf(z - mn);
  l = l * sc + pz;
  a = a * sc + pz * k;
  m = mn;
}

// Where row j of a window comes from: this call's projection row t (raw score,
// ape row given) or an earlier call's state rows (score already with ape), or
// nowhere (masked / bad table entry).
struct RowSrc {
  int64_t kv;    // element offset of the row start: proj row (2C wide) or kv_state row (C wide)
  int64_t sc;    // proj row again, or score_state row
  int32_t ape;   // ape row for projection rows, -1 for state rows, -2 for skipped rows
  int32_t half;  // column offset of the half this row contributes (0 or D)
};

constexpr int kMaxRows = 256;  // coff * ratio <= 256
constexpr int kMaxStagedSeqs = 256;

__global__ void __launch_bounds__(128) pool_kernel(Params p) {
  __shared__ float red[32];
  __shared__ float zs[1024];  // 2 D floats: the Hadamard product's exchange buffers
  __shared__ RowSrc src[kMaxRows];
  __shared__ int32_t off_s[kMaxStagedSeqs + 1];
  __shared__ int32_t cu_s[kMaxStagedSeqs + 1];
  __shared__ int32_t s_s[kMaxStagedSeqs];
  const int n = blockIdx.x;
  const int D = p.D, C = p.C, r = p.ratio;
  const int c = threadIdx.x * 4;
  pdl_wait();  // everything below reads what the earlier kernels of the call wrote

  // which sequence owns row n: its metadata is staged in one round trip of
  // independent loads (when B is small), then searched in shared memory
  int b, s = 0, cu = 0, e = 0;
  const bool staged = p.B <= kMaxStagedSeqs;
  if (staged) {
    for (int i = threadIdx.x; i <= p.B; i += blockDim.x) {
      off_s[i] = p.m_off[i];
      cu_s[i] = p.m_cu[i];
      if (i < p.B) s_s[i] = p.m_s[i];
    }
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
  int w = -1, off = 0;
  if (b < p.B) {
    s = staged ? s_s[b] : p.m_s[b];
    cu = staged ? cu_s[b] : p.m_cu[b];
    e = s + ((staged ? cu_s[b + 1] : p.m_cu[b + 1]) - cu);
    off = staged ? off_s[b] : p.m_off[b];
    const int k = n - off;
    if (k < e / r - s / r) w = s / r + k;
  }
  uint2* dst = reinterpret_cast<uint2*>(p.out + (int64_t)n * D + c);
  if (w < 0) {
    *dst = make_uint2(0u, 0u);
    return;
  }
  const RowAux aux = load_row_aux(p, n, c);  // independent of the pooling: in flight meanwhile

  // 1) resolve every row of the window (table lookups only for rows before
  //    start_pos, i.e. the first window of the sequence)
  const int rows = p.coff * r;
  for (int j = threadIdx.x; j < rows; j += blockDim.x) {
    const bool bhalf = p.coff == 1 || j >= r;
    const int q = p.coff == 1 ? w * r + j : (j < r ? (w - 1) * r + j : w * r + (j - r));
    RowSrc rs{0, 0, -2, (p.coff == 2 && bhalf) ? D : 0};
    if (q >= s) {
      rs.kv = (int64_t)(cu + (q - s)) * (2 * C);
      rs.sc = rs.kv + C;
      rs.ape = q % r;
    } else if (q >= 0) {  // q < 0: the first window has no previous window
      const int rk = table_row(p, p.kv_tbl, b, q);
      const int rv = table_row(p, p.sc_tbl, b, q);
      if (rk >= 0 && rv >= 0) {
        rs.kv = ((int64_t)rk * p.bs + q % p.bs) * C;
        rs.sc = ((int64_t)rv * p.bs + q % p.bs) * C;
        rs.ape = -1;
      }
    }
    src[j] = rs;
  }
  __syncthreads();

  // 2) online softmax over the rows, 8 rows' loads in flight at a time
  float m[4], l[4], a[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) { m[i] = -INFINITY; l[i] = 0.f; a[i] = 0.f; }
  for (int j0 = 0; j0 < rows; j0 += 8) {
    float4 kv[8], sc[8];
    bool use[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      use[u] = false;
      if (j0 + u < rows) {
        const RowSrc rs = src[j0 + u];
        const int col = rs.half + c;
        if (rs.ape >= 0) {
          kv[u] = ld4(p.proj + rs.kv + col);
          sc[u] = ld4(p.proj + rs.sc + col);
          const float4 ap = ld4(p.ape + (int64_t)rs.ape * C + col);
          sc[u].x += ap.x;
          sc[u].y += ap.y;
          sc[u].z += ap.z;
          sc[u].w += ap.w;
          use[u] = true;
        } else if (rs.ape == -1) {
          kv[u] = ld4(p.kv_state + rs.kv + col);
          sc[u] = ld4(p.score_state + rs.sc + col);
          use[u] = true;
        }
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (use[u]) {
        online(m[0], l[0], a[0], sc[u].x, kv[u].x);
        online(m[1], l[1], a[1], sc[u].y, kv[u].y);
        online(m[2], l[2], a[2], sc[u].z, kv[u].z);
        online(m[3], l[3], a[3], sc[u].w, kv[u].w);
      }
    }
  }
  float y[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) y[i] = l[i] > 0.f ? a[i] / l[i] : 0.f;

  finish_row(p, n, c, y, red, zs, aux);
}

}  // namespace

cudaError_t launch_pool(const Params& p, cudaStream_t s) {
  if (p.n_out <= 0) return cudaSuccess;
  return launch_chained(pool_kernel, dim3(p.n_out), dim3(p.D / 4), 0, s, 1, p);
}

}  // namespace cmp
