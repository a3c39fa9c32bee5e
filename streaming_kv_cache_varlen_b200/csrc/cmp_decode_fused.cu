// Decode in one kernel (T <= 64 tokens, B <= 256 sequences): no separate
// scheduler or pooling launch, one grid-wide barrier.
//
// The cost of a decode call is reading the two weight matrices once, so all
// CTAs start streaming them at once. The grid is (weight tiles of 128 rows) x
// (K slices), sized to fill the GPU, launched cooperatively so that every CTA
// is resident (the launch fails otherwise) and the grid barrier cannot wait on
// a CTA that never runs.
//
//  1. Every CTA streams its 128-row x K-slice of wkv or wgate and the matching
//     x slice with TMA (4 stages), accumulates 128 x N (N = T rounded up to 16)
//     in TMEM with tcgen05.mma, and stores the partial product in a global
//     (L2-resident) buffer part[kslice][token][2C]. Meanwhile warps 2-3 read
//     cu_seqlens / start_pos and compute, in shared memory, what the varlen
//     scheduler kernel computes on the other paths (validation, per-sequence
//     output-row offsets, each token's position and state slots).
//  2. Grid barrier (bounded: a CTA that waits too long records a timeout and
//     skips the rest).
//  3. CTAs 0 .. n_out-1 each build one output row: the window's rows come from
//     the paged state (positions before start_pos) or, for this call's tokens,
//     from the sum of the K-slice partials (in slice order: bitwise
//     reproducible) plus ape; then the per-channel softmax-weighted sum,
//     RMSNorm, RoPE, Hadamard and the bf16 store ("compressor torch_extension
//     API", 计算公式 1-5; "CANN PyPTO 算子实战", 压缩窗口与状态更新). Rows with no
//     window are stored as 0. The other CTAs sum the partials of the state tail
//     rows and write kv and score + ape to the paged state.
// This call writes state slots of positions >= start_pos only and reads those
// below, so step 3's readers and writers never touch the same slot.
#include <cstddef>
#include <mutex>

#include "cmp_internal.cuh"
#include "cmp_rowpost.cuh"
#include "cmp_sm100.cuh"

namespace cmp {
namespace {

using namespace sm100;

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int kThreads = 192;        // warps 0-3: TMEM quadrants; warps 4-5: call metadata
constexpr int kMaxSeqs = 256;
constexpr int kMaxRowsPerWindow = 256;
constexpr int kHistRows = 8;         // state rows of a window prefetched into shared memory

template <int MAXT>
struct Stages {
  // enough stages that a C4A-sized CTA requests its whole weight slice at once
  static constexpr int value = MAXT <= 32 ? 8 : 6;
};

struct TokInfo {
  int32_t b;        // sequence, or -1
  int32_t pos;      // absolute position
  int64_t kv_off;   // kv_state element offset of its row if it is a tail row, else -1
  int64_t sc_off;   // score_state element offset, else -1
};

template <int MAXT>
struct Smem {
  static constexpr int S = Stages<MAXT>::value;
  __nv_bfloat16 w[S][BM * BK];     // 16 KB per stage
  __nv_bfloat16 x[S][MAXT * BK];   // MAXT * 128 bytes per stage
  alignas(16) float hist_kv[kHistRows][512];  // the window's state rows (float4 access)
  alignas(16) float hist_sc[kHistRows][512];
  TokInfo tok[MAXT];
  int32_t cu[kMaxSeqs + 1];
  int32_t sp[kMaxSeqs];
  int32_t off[kMaxSeqs + 1];
  int32_t src_t[kMaxRowsPerWindow];     // per window row: token (>= 0), -1 (state row) or INT32_MIN (skip)
  int64_t src_kv[kMaxRowsPerWindow];
  int64_t src_sc[kMaxRowsPerWindow];
  int32_t row_w;                        // window of this CTA's output row, or -1
  int32_t nhist;                        // state rows 0..nhist-1 of the window are in hist_*, or -1
  float red[32];
  float zs[1024];  // 2 D floats: the Hadamard product's exchange buffers
  uint64_t full[S];
  uint64_t empty[S];
  uint64_t acc_full;
  uint32_t tmem_base;
  int abort;
  int rejected;
  int grid_ok;
  uint32_t bar_gen;   // generation seen at arrival (thread 0)
  int bar_last;       // this CTA released the barrier
};

static_assert(offsetof(Smem<32>, hist_kv) % 16 == 0 && offsetof(Smem<32>, hist_sc) % 16 == 0,
              "float4 shared-memory rows must be 16-byte aligned");
static_assert(offsetof(Smem<64>, hist_kv) % 16 == 0 && offsetof(Smem<64>, hist_sc) % 16 == 0,
              "float4 shared-memory rows must be 16-byte aligned");
static_assert(offsetof(Smem<32>, x) % 1024 == 0 && offsetof(Smem<64>, x) % 1024 == 0,
              "TMA swizzled tiles must be 1024-byte aligned");
static_assert(sizeof(Smem<32>) + 1024 <= 232448 && sizeof(Smem<64>) + 1024 <= 232448,
              "shared memory per CTA");

struct GridBar {
  unsigned count;
  unsigned pad0[31];  // count and generation on different 128-byte lines
  unsigned gen;
};

// Split grid barrier for a cooperative launch. grid_arrive: thread 0 of each
// CTA, after the CTA's stores; the last arrival resets the count and bumps the
// generation. grid_wait: thread 0 waits (bounded: ~1 s, then a timeout is
// recorded and the CTA goes on without the data) for the generation to move.
__device__ __forceinline__ void grid_arrive(GridBar* bar, unsigned nblocks, uint32_t* gen_seen, int* last) {
  unsigned g;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(g) : "l"(&bar->gen) : "memory");
  __threadfence();
  *gen_seen = g;
  *last = 0;
  if (atomicAdd(&bar->count, 1u) == nblocks - 1) {
    atomicExch(&bar->count, 0u);
    __threadfence();
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(&bar->gen), "r"(g + 1) : "memory");
    *last = 1;
  }
}

__device__ __forceinline__ bool grid_wait(GridBar* bar, uint32_t g, unsigned* err) {
  const uint64_t t0 = globaltimer();
  for (;;) {
    unsigned now;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(now) : "l"(&bar->gen) : "memory");
    if (now != g) return true;
    if (globaltimer() - t0 > 1000000000ull) {
      atomicOr(err, kErrTimeout);
      return false;
    }
    __nanosleep(32);
  }
}

// sum over the K slices of part[q][t][col .. col+3], in slice order, with up to
// eight loads in flight (the partials were written by other CTAs: L2 loads).
__device__ __forceinline__ float4 sum_slices(const float* part, int KS, int64_t slice_stride, int64_t off) {
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int q0 = 0; q0 < KS; q0 += 8) {
    float4 u[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      u[i] = q0 + i < KS ? __ldcg(reinterpret_cast<const float4*>(part + (q0 + i) * slice_stride + off))
                         : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (q0 + i < KS) {
        acc.x += u[i].x;
        acc.y += u[i].y;
        acc.z += u[i].z;
        acc.w += u[i].w;
      }
    }
  }
  return acc;
}

struct DecodeArgs {
  float* part;      // [ks][T][2C] partial products
  GridBar* bar;
  int ks;           // K slices
};

// Window row j of window w: its absolute position.
__device__ __forceinline__ int window_pos(int w, int j, int r, int coff) {
  return coff == 1 ? w * r + j : (j < r ? (w - 1) * r + j : w * r + (j - r));
}

// Warps 4-5: validate the call, output-row offsets, per-token facts, and the
// sources of this CTA's output row (what the varlen scheduler kernel does on
// the other paths), while warps 0-3 stream and multiply.
template <int MAXT>
__device__ void call_metadata(const Params& p, Smem<MAXT>& sm, int NT) {
  const int et = threadIdx.x - 128;  // 0..63
  const int B = p.B;
  bool bad = false;
  for (int i = et; i <= B; i += 64) {
    const int c = p.cu_in[i];
    const int c1 = i < B ? p.cu_in[i + 1] : c;
    const int s = (i < B && p.start_pos) ? p.start_pos[i] : 0;
    sm.cu[i] = c;
    if (i < B) sm.sp[i] = s;
    bool ok = c >= 0 && c <= p.T && (i != 0 || c == 0) && (i != B || c == p.T);
    if (i < B) ok = ok && c1 >= c && s >= 0 && (int64_t)s + (c1 - c) <= (int64_t)INT32_MAX;
    bad = bad || !ok;
  }
  if (bad) atomicOr(&sm.rejected, 1);
  asm volatile("bar.sync 2, 64;" ::: "memory");
  const bool rejected = sm.rejected != 0;
  if (et < 32) {  // output-row offsets: sequence b reserves min(L, L/ratio + 1) rows
    int carry = 0;
    for (int b0 = 0; b0 < B; b0 += 32) {
      const int b = b0 + et;
      int cap = 0;
      if (b < B && !rejected) {
        const int L = sm.cu[b + 1] - sm.cu[b];
        cap = min(L, L / p.ratio + 1);
      }
      int inc = cap;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, inc, o);
        if (et >= o) inc += v;
      }
      if (b < B) sm.off[b] = carry + inc - cap;
      carry += __shfl_sync(0xffffffffu, inc, 31);
    }
    if (et == 0) {
      sm.off[B] = carry;
      if (rejected) atomicOr(p.err, kErrIndex);
    }
  }
  asm volatile("bar.sync 2, 64;" ::: "memory");
  if (rejected) {
    for (int i = et; i <= B; i += 64) sm.cu[i] = 0;
    asm volatile("bar.sync 2, 64;" ::: "memory");
  }
  for (int t = et; t < NT; t += 64) {
    TokInfo ti{-1, 0, -1, -1};
    if (t < p.T && !rejected) {
      int lo = 0, hi = B;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (sm.cu[mid] <= t) lo = mid; else hi = mid - 1;
      }
      if (lo < B) {
        const int s = sm.sp[lo];
        const int pos = s + (t - sm.cu[lo]);
        const int e = s + (sm.cu[lo + 1] - sm.cu[lo]);
        ti.b = lo;
        ti.pos = pos;
        if (pos >= tail_threshold(e, p.ratio, p.coff)) {
          const int rk = table_row(p, p.kv_tbl, lo, pos);
          const int rs = table_row(p, p.sc_tbl, lo, pos);
          if (rk >= 0) ti.kv_off = ((int64_t)rk * p.bs + pos % p.bs) * p.C;
          if (rs >= 0) ti.sc_off = ((int64_t)rs * p.bs + pos % p.bs) * p.C;
        }
      }
    }
    sm.tok[t] = ti;
  }
  // this CTA's output row: its window and where each window row comes from
  if ((int)blockIdx.x < p.n_out) {
    const int n = blockIdx.x, r = p.ratio;
    int lo = 0, hi = B;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (sm.off[mid] <= n) lo = mid; else hi = mid - 1;
    }
    int w = -1, s = 0, cu = 0;
    if (lo < B && !rejected) {
      s = sm.sp[lo];
      cu = sm.cu[lo];
      const int e = s + (sm.cu[lo + 1] - cu);
      const int k = n - sm.off[lo];
      if (k < e / r - s / r) w = s / r + k;
    }
    const int rows = p.coff * r;
    int nh = 0;
    if (w >= 0) {
      for (int j = et; j < rows; j += 64) {
        const int q = window_pos(w, j, r, p.coff);
        int st = INT32_MIN;
        int64_t okv = 0, osc = 0;
        if (q >= s) {
          st = cu + (q - s);
        } else if (q >= 0) {
          const int rk = table_row(p, p.kv_tbl, lo, q);
          const int rs = table_row(p, p.sc_tbl, lo, q);
          if (rk >= 0 && rs >= 0) {
            st = -1;
            okv = ((int64_t)rk * p.bs + q % p.bs) * p.C;
            osc = ((int64_t)rs * p.bs + q % p.bs) * p.C;
          }
        }
        sm.src_t[j] = st;
        sm.src_kv[j] = okv;
        sm.src_sc[j] = osc;
      }
      for (int j = 0; j < rows; ++j)
        if (window_pos(w, j, r, p.coff) < s) nh = j + 1;  // state rows are the window's first rows
    }
    if (et == 0) {
      sm.row_w = w;
      sm.nhist = (w >= 0 && nh <= kHistRows && p.D <= 512) ? nh : -1;
    }
  }
}

template <int MAXT>
__global__ void __launch_bounds__(kThreads, 1)
    decode_fused_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_wkv,
                        const __grid_constant__ CUtensorMap map_wg, Params p, DecodeArgs a, int NT) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  using SM = Smem<MAXT>;
  constexpr int STAGES = SM::S;
  SM& sm = *reinterpret_cast<SM*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x / a.ks, ks = blockIdx.x % a.ks;
  const int m0 = tile * BM;  // first of the 128 weight rows (of the 2C)
  const bool score_rows = m0 >= p.C;
  const CUtensorMap* wmap = score_rows ? &map_wg : &map_wkv;
  const int wrow = score_rows ? m0 - p.C : m0;
  const int kb_total = p.H / BK;
  const int kb_lo = ks * kb_total / a.ks, kb_hi = (ks + 1) * kb_total / a.ks;
  const uint32_t x_bytes = (uint32_t)NT * BK * 2;
  const uint32_t tmem_cols = NT <= 32 ? 32 : 64;
  const int C2 = 2 * p.C;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    mbar_init(&sm.acc_full, 1);
    sm.abort = 0;
    sm.rejected = 0;
    sm.row_w = -1;
    sm.nhist = -1;
    fence_barrier_init();
    prefetch_tmap(wmap);
    prefetch_tmap(&map_x);
  }
  if (warp == 1) tmem_alloc(&sm.tmem_base, tmem_cols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort = &sm.abort;

  // ---- 1) stream + MMA (warps 0, 1) / call metadata (warps 4, 5) ----
  if (warp == 0 && lane == 0) {
    int stage = 0;
    uint32_t phase = 0;
    Armed armed;
    for (int kb = kb_lo; kb < kb_hi; ++kb) {
      if (!mbar_wait(&sm.empty[stage], phase ^ 1u, abort)) break;
      mbar_arrive_expect_tx(&sm.full[stage], BM * BK * 2 + x_bytes);
      armed.note(stage, phase);
      tma_load_2d(sm.w[stage], wmap, &sm.full[stage], kb * BK, wrow);
      tma_load_2d(sm.x[stage], &map_x, &sm.full[stage], kb * BK, 0);
      if (++stage == STAGES) { stage = 0; phase ^= 1u; }
    }
    drain_armed(sm.full, STAGES, armed);  // no copy still landing when the CTA leaves
  } else if (warp == 1 && lane == 0) {
    int stage = 0;
    uint32_t phase = 0;
    const uint32_t idesc = idesc_bf16_f32(BM, NT);
    bool ok = true;
    for (int kb = kb_lo; kb < kb_hi; ++kb) {
      if (!mbar_wait(&sm.full[stage], phase, abort)) { ok = false; break; }
      tc_fence_after();
      const uint32_t a0 = smem_u32(sm.w[stage]);
      const uint32_t b0 = smem_u32(sm.x[stage]);
#pragma unroll
      for (int k = 0; k < BK / 16; ++k)
        mma_bf16(tmem, sw128_kmajor_desc(a0 + k * 32), sw128_kmajor_desc(b0 + k * 32), idesc,
                 (kb > kb_lo || k > 0) ? 1u : 0u);
      mma_commit(&sm.empty[stage]);
      if (++stage == STAGES) { stage = 0; phase ^= 1u; }
    }
    if (ok) mma_commit(&sm.acc_full);
  } else if (warp >= 4) {
    call_metadata<MAXT>(p, sm, NT);
  }

  if (warp < 4) {
    // the partial product of this CTA's 128 rows -> part[ks][t][m0 + row]
    const bool have = mbar_wait(&sm.acc_full, 0, abort);
    if (__all_sync(0xffffffffu, have)) {
      tc_fence_after();
      const int row = warp * 32 + lane;
      float* dst = a.part + (int64_t)ks * p.T * C2 + m0 + row;
      for (int c0 = 0; c0 < NT; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + c0, r);
        tmem_ld_wait(r);
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (c0 + j < p.T) dst[(int64_t)(c0 + j) * C2] = __uint_as_float(r[j]);
      }
    }
    tc_fence_before();
    asm volatile("bar.sync 1, 128;" ::: "memory");  // all partial stores of the CTA issued
    if (threadIdx.x == 0) grid_arrive(a.bar, gridDim.x, &sm.bar_gen, &sm.bar_last);
  }
  __syncthreads();  // metadata (warps 4-5) done

  // ---- 2) while the other CTAs arrive: this CTA's window rows from the state ----
  const int nh = sm.nhist;
  if ((int)blockIdx.x < p.n_out && nh > 0) {
    const int q4 = p.D / 4;
    for (int i0 = threadIdx.x; i0 < nh * q4; i0 += 2 * kThreads) {
      float4 kv[2], sc[2];
      bool use[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {  // two rows' loads in flight per thread
        const int i = i0 + u * kThreads;
        const int j = i / q4;
        use[u] = i < nh * q4 && sm.src_t[j] == -1;
        if (use[u]) {
          const int c = (i % q4) * 4;
          const int col = ((p.coff == 2 && j >= p.ratio) ? p.D : 0) + c;
          kv[u] = *reinterpret_cast<const float4*>(p.kv_state + sm.src_kv[j] + col);
          sc[u] = *reinterpret_cast<const float4*>(p.score_state + sm.src_sc[j] + col);
        }
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        if (use[u]) {
          const int i = i0 + u * kThreads;
          const int j = i / q4, c = (i % q4) * 4;
          *reinterpret_cast<float4*>(&sm.hist_kv[j][c]) = kv[u];
          *reinterpret_cast<float4*>(&sm.hist_sc[j][c]) = sc[u];
        }
      }
    }
  }
  if (threadIdx.x == 0) sm.grid_ok = sm.bar_last ? 1 : (grid_wait(a.bar, sm.bar_gen, p.err) ? 1 : 0);
  __syncthreads();
  const bool ok = sm.grid_ok && !*abort;

  // ---- 3) output rows / state tails ----
  const int n_out = p.n_out;
  const int KS = a.ks;
  const int64_t slice = (int64_t)p.T * C2;
  if ((int)blockIdx.x < n_out) {
    const int n = blockIdx.x;
    const int D = p.D, r = p.ratio, c = threadIdx.x * 4;
    const bool active = c < D;
    const int w = ok ? sm.row_w : -1;
    if (w < 0) {
      if (active) *reinterpret_cast<uint2*>(p.out + (int64_t)n * D + c) = make_uint2(0u, 0u);
    } else {
      const int rows = p.coff * r;
      float y[4] = {0.f, 0.f, 0.f, 0.f};
      if (active) {
        float m[4], l[4], ac[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) { m[i] = -INFINITY; l[i] = 0.f; ac[i] = 0.f; }
        for (int j = 0; j < rows; ++j) {
          const int st = sm.src_t[j];
          if (st == INT32_MIN) continue;
          const int col = ((p.coff == 2 && j >= r) ? D : 0) + c;
          float4 kv, sc;
          if (st >= 0) {  // this call's token: the K-slice partials plus ape
            const int q = window_pos(w, j, r, p.coff);
            kv = sum_slices(a.part, KS, slice, (int64_t)st * C2 + col);
            sc = sum_slices(a.part, KS, slice, (int64_t)st * C2 + p.C + col);
            const float4 ap = *reinterpret_cast<const float4*>(p.ape + (int64_t)(q % r) * p.C + col);
            sc.x += ap.x;
            sc.y += ap.y;
            sc.z += ap.z;
            sc.w += ap.w;
          } else if (j < nh) {
            kv = *reinterpret_cast<const float4*>(&sm.hist_kv[j][c]);
            sc = *reinterpret_cast<const float4*>(&sm.hist_sc[j][c]);
          } else {
            kv = *reinterpret_cast<const float4*>(p.kv_state + sm.src_kv[j] + col);
            sc = *reinterpret_cast<const float4*>(p.score_state + sm.src_sc[j] + col);
          }
          const float kk[4] = {kv.x, kv.y, kv.z, kv.w}, zz[4] = {sc.x, sc.y, sc.z, sc.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float mn = fmaxf(m[i], zz[i]);
            const float f = __expf(m[i] - mn), pz = __expf(zz[i] - mn);
            l[i] = l[i] * f + pz;
            ac[i] = ac[i] * f + pz * kk[i];
            m[i] = mn;
          }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) y[i] = l[i] > 0.f ? ac[i] / l[i] : 0.f;
      }
      finish_row(p, n, c, y, sm.red, sm.zs);
    }
  } else if (ok) {
    // state tails: the other CTAs split (token, 4 columns) groups between them
    const int nb = gridDim.x - n_out;
    const int groups = p.T * (C2 / 4);
    for (int g = (blockIdx.x - n_out) * kThreads + threadIdx.x; g < groups; g += nb * kThreads) {
      const int t = g / (C2 / 4), col = (g % (C2 / 4)) * 4;
      const TokInfo ti = sm.tok[t];
      const bool score = col >= p.C;
      const int64_t so = score ? ti.sc_off : ti.kv_off;
      if (ti.b < 0 || so < 0) continue;
      float4 v = sum_slices(a.part, KS, slice, (int64_t)t * C2 + col);
      const int sc = score ? col - p.C : col;
      if (score) {
        const float4 ap = *reinterpret_cast<const float4*>(p.ape + (int64_t)(ti.pos % p.ratio) * p.C + sc);
        v.x += ap.x;
        v.y += ap.y;
        v.z += ap.z;
        v.w += ap.w;
      }
      *reinterpret_cast<float4*>((score ? p.score_state : p.kv_state) + so + sc) = v;
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, tmem_cols);
  }
  if (threadIdx.x == 0 && sm.abort) atomicOr(p.err, kErrTimeout);
}

// CTAs of one variant that can be resident at once on the current device (cached).
template <int MAXT>
int max_resident() {
  static int cached[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && cached[dev]) return cached[dev];
  const size_t smem = sizeof(Smem<MAXT>) + 1024;
  static int conf[64] = {0};
  int per_sm = 0, sms = 0;
  if (smem_attr_once(decode_fused_kernel<MAXT>, smem, conf) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_fused_kernel<MAXT>, kThreads, smem) !=
          cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    per_sm = 0;
  }
  const int n = per_sm * sms;
  if (dev < 64) cached[dev] = n > 0 ? n : -1;
  return n;
}

int sm_count() {
  int dev = 0, n = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

}  // namespace

// K slices for a call: fill the GPU with one CTA per SM, at least one K block
// per slice, and enough CTAs for every output row.
int decode_fused_kslices(const Params& p) {
  const int tiles = (2 * p.C) / BM;
  const int kb = p.H / BK;
  int ks = sm_count() / tiles;
  if (ks > kb) ks = kb;
  if (ks < 1) ks = 1;
  return ks;
}

bool decode_fused_supported(const Params& p) {
  if (p.T < 1 || p.T > 64 || p.B > kMaxSeqs || p.coff * p.ratio > kMaxRowsPerWindow) return false;
  if (p.H % BK || (2 * p.C) % BM || encode_fn() == nullptr) return false;
  const int grid = ((2 * p.C) / BM) * decode_fused_kslices(p);
  if (grid <= p.n_out) return false;  // one CTA per output row plus at least one for the tails
  const int cap = p.T <= 32 ? max_resident<32>() : max_resident<64>();
  return cap >= grid;
}

size_t decode_fused_workspace(const Params& p) {
  return sizeof(float) * (size_t)decode_fused_kslices(p) * p.T * 2 * p.C;
}

cudaError_t launch_decode_fused(const Params& p, float* part, void* bar, cudaStream_t s) {
  const int NT = (p.T + 15) / 16 * 16;
  CUtensorMap mx, mkv, mg;
  if (!make_tile_map(&mx, p.x, p.T, p.H, (uint32_t)NT) || !make_tile_map(&mkv, p.wkv, p.C, p.H, BM) ||
      !make_tile_map(&mg, p.wgate, p.C, p.H, BM))
    return cudaErrorInvalidValue;
  DecodeArgs a;
  a.part = part;
  a.bar = static_cast<GridBar*>(bar);
  a.ks = decode_fused_kslices(p);
  const int grid = ((2 * p.C) / BM) * a.ks;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (NT <= 32) {
    cfg.dynamicSmemBytes = sizeof(Smem<32>) + 1024;
    static int conf[64] = {0};
    const cudaError_t e = smem_attr_once(decode_fused_kernel<32>, cfg.dynamicSmemBytes, conf);
    if (e != cudaSuccess) return e;
    return cudaLaunchKernelEx(&cfg, decode_fused_kernel<32>, mx, mkv, mg, p, a, NT);
  }
  cfg.dynamicSmemBytes = sizeof(Smem<64>) + 1024;
  static int conf[64] = {0};
  const cudaError_t e = smem_attr_once(decode_fused_kernel<64>, cfg.dynamicSmemBytes, conf);
  if (e != cudaSuccess) return e;
  return cudaLaunchKernelEx(&cfg, decode_fused_kernel<64>, mx, mkv, mg, p, a, NT);
}

}  // namespace cmp
