// Small-T projection (decode, T <= 64 tokens): the cost is reading the two
// weight matrices once, so the kernel is built to stream them at HBM bandwidth
// across the whole GPU.
//
//   proj[t][n] = sum_k W[n][k] * x[t][k]  (raw scores; tail rows, score rows
//   with ape, to the paged state), as in the prefill kernels ("compressor torch_extension
//   API", 计算公式 1-2).
//
// Work split: the weight rows are cut into 128-row tiles (MMA M = 128) and the
// hidden dimension into 8 (or 4) slices; the CTAs that share a row tile form
// one thread-block cluster. Each CTA streams its 128 x (H/8) weight slice and the
// matching x slice with TMA through a 3- or 4-stage ring, accumulates a 128 x N
// partial product in TMEM with tcgen05.mma (N = T rounded up to 16), and parks
// pushes each row of it into the shared memory of the CTA that owns the row
// (CTA j owns rows 16j..16j+15) through distributed shared memory. After one
// cluster barrier every CTA sums its 16 rows over the 8 slices, always in
// slice order (so the result is bitwise reproducible), and writes those rows
// of proj and of the state tail.
// (Splitting the head dimension across more cores to raise the number of
// active cores and the bandwidth in decode is the idea of "NPU DeepSeek-V4
// Ascend C 融合算子优化", Decode; here the split is over K and the reduction
// stays on chip.)
#include <mutex>

#include "cmp_internal.cuh"
#include "cmp_sm100.cuh"

namespace cmp {
namespace {

using namespace sm100;

constexpr int BM = 128;        // weight rows per cluster
constexpr int BK = 64;         // K per stage
constexpr int MAX_T = 64;
constexpr int kThreads = 128;

struct TokMeta {
  int32_t valid;     // token belongs to a sequence
  int32_t ape_row;   // position mod ratio
  int64_t kv_off;    // element offset of its kv_state row if it is a tail row, else -1
  int64_t sc_off;    // same for score_state
};

// Shared memory of one CTA, sized for at most MAXT tokens. Small enough
// (under ~110 KB) that two CTAs fit on one SM, so all 16 clusters of a
// C4A-sized call are resident at once even where a GPC cannot host two
// one-CTA-per-SM clusters.
template <int KSPLIT, int MAXT, int STAGES>
struct Smem {
  __nv_bfloat16 w[STAGES][BM * BK];      // 16 KB per stage, 1024-byte aligned
  __nv_bfloat16 x[STAGES][MAXT * BK];    // MAXT * 128 bytes per stage
  float recv[KSPLIT][MAXT][BM / KSPLIT]; // partials of this CTA's rows, from every K slice
  TokMeta tok[MAXT];
  int32_t cu[MAXT + 1];                  // token offsets of the sequences (B <= MAXT)
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t acc_full;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}

// Store v into the shared memory of cluster CTA `peer`, at the address `local`
// has in this CTA.
__device__ __forceinline__ void st_peer(float* local, uint32_t peer, float v) {
  uint32_t ra;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(smem_u32(local)), "r"(peer));
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(ra), "f"(v) : "memory");
}

template <int KSPLIT, int MAXT, int STAGES>
__global__ void __launch_bounds__(kThreads)
    proj_decode_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_wkv,
                       const __grid_constant__ CUtensorMap map_wg, Params p, int NT) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  using S = Smem<KSPLIT, MAXT, STAGES>;
  constexpr int RPC = BM / KSPLIT;  // weight rows each CTA reduces
  S& sm = *reinterpret_cast<S*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();            // K slice of this CTA
  const int m0 = blockIdx.y * BM;                  // weight row tile (of the 2C rows)
  const bool score = m0 >= p.C;
  const CUtensorMap* wmap = score ? &map_wg : &map_wkv;
  const int wrow = score ? m0 - p.C : m0;
  const int kb_total = p.H / BK;
  const int kb_lo = (int)(rank * kb_total / KSPLIT);
  const int kb_hi = (int)((rank + 1) * kb_total / KSPLIT);
  const uint32_t x_bytes = (uint32_t)NT * BK * 2;
  const uint32_t tmem_cols = NT <= 32 ? 32 : 64;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    mbar_init(&sm.acc_full, 1);
    sm.abort = 0;
    fence_barrier_init();
    prefetch_tmap(wmap);
    prefetch_tmap(&map_x);
  }
  if (warp == 1) tmem_alloc(&sm.tmem_base, tmem_cols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_trigger();  // the pooling kernel may be scheduled now; it waits for this grid
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort = &sm.abort;

  // x and the weights are call inputs: streaming them may start before the
  // scheduler kernel has finished
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
  } else if (warp >= 2) {
    // while the weights stream in: per-token facts for the epilogue, from the
    // scheduler's metadata (so after the grid dependency is met)
    pdl_wait();
    const int et = threadIdx.x - 64;
    const bool staged = p.B <= MAXT;
    if (staged)
      for (int i = et; i <= p.B; i += 64) sm.cu[i] = p.m_cu[i];
    asm volatile("bar.sync 2, 64;" ::: "memory");
    for (int t = et; t < NT; t += 64) {
      TokMeta m{0, 0, -1, -1};
      if (t < p.T) {
        int b;
        if (staged) {
          int lo = 0, hi = p.B;
          while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (sm.cu[mid] <= t) lo = mid; else hi = mid - 1;
          }
          b = lo;
        } else {
          b = upper_index(p.m_cu, p.B, t);
        }
        if (b < p.B) {
          const int s0 = p.m_s[b];
          const int c0 = p.m_cu[b];
          const int pos = s0 + (t - c0);
          const int e = s0 + (p.m_cu[b + 1] - c0);
          m.valid = 1;
          m.ape_row = pos % p.ratio;
          if (pos >= tail_threshold(e, p.ratio, p.coff)) {
            const int rk = table_row(p, p.kv_tbl, b, pos);
            const int rs = table_row(p, p.sc_tbl, b, pos);
            if (rk >= 0) m.kv_off = ((int64_t)rk * p.bs + pos % p.bs) * p.C;
            if (rs >= 0) m.sc_off = ((int64_t)rs * p.bs + pos % p.bs) * p.C;
          }
        }
      }
      sm.tok[t] = m;
    }
  }

  // every warp: its 32 accumulator lanes (weight rows) go to the CTA that owns
  // them (rows 16j..16j+15 -> cluster rank j), into slot [this K slice]
  const bool have = mbar_wait(&sm.acc_full, 0, abort);
  if (__all_sync(0xffffffffu, have)) {
    tc_fence_after();
    const int row = warp * 32 + lane;
    const uint32_t owner = (uint32_t)(row / RPC);
    for (int c0 = 0; c0 < NT; c0 += 32) {
      uint32_t r[32];
      tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + c0, r);
      tmem_ld_wait(r);
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (c0 + j < NT) st_peer(&sm.recv[rank][c0 + j][row % RPC], owner, __uint_as_float(r[j]));
    }
  }
  tc_fence_before();
  cluster_sync();  // every CTA reaches this on every path; the pushes are now visible

  // this CTA's rows RPC*rank .. RPC*rank+RPC-1: sum the K slices in a fixed order
  pdl_wait();
  if (!*abort) {
    for (int i = threadIdx.x; i < RPC * NT; i += kThreads) {
      const int t = i / RPC, r = i % RPC;
      const TokMeta m = sm.tok[t];
      if (t >= p.T || !m.valid) continue;
      float v = 0.f;
#pragma unroll
      for (int q = 0; q < KSPLIT; ++q) v += sm.recv[q][t][r];
      const int col = wrow + (int)rank * RPC + r;
      p.proj[(int64_t)t * (2 * p.C) + (score ? p.C : 0) + col] = v;
      const int64_t so = score ? m.sc_off : m.kv_off;
      if (so >= 0) {
        if (score) v += __ldg(p.ape + (int64_t)m.ape_row * p.C + col);  // state: score + ape
        (score ? p.score_state : p.kv_state)[so + col] = v;
      }
    }
  }

  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, tmem_cols);
  }
  if (threadIdx.x == 0 && sm.abort) atomicOr(p.err, kErrTimeout);
}

}  // namespace

bool proj_decode_supported(const Params& p) {
  return p.T >= 1 && p.T <= MAX_T && (p.H / BK) >= 8 && p.H % BK == 0 && (2 * p.C) % BM == 0 &&
         encode_fn() != nullptr;
}

size_t proj_decode_workspace(const Params&) { return 0; }

template <int KSPLIT, int MAXT, int STAGES>
cudaError_t launch_variant(const Params& p, cudaStream_t s, int NT, const CUtensorMap& mx,
                           const CUtensorMap& mkv, const CUtensorMap& mg) {
  const size_t smem = sizeof(Smem<KSPLIT, MAXT, STAGES>) + 1024;
  static int configured[64] = {0};
  const cudaError_t e = smem_attr_once(proj_decode_kernel<KSPLIT, MAXT, STAGES>, smem, configured);
  if (e != cudaSuccess) return e;
  return launch_chained(proj_decode_kernel<KSPLIT, MAXT, STAGES>, dim3(KSPLIT, (2 * p.C) / BM, 1),
                        dim3(kThreads, 1, 1), smem, s, KSPLIT, mx, mkv, mg, p, NT);
}

// How many clusters of the 8-wide variant the device runs at once (cached
// per device). Where a GPC cannot hold two 8-CTA clusters, fewer than
// (number of SMs / 8) fit, and a call with more weight tiles than that would
// run in two waves; it then uses 4-wide clusters instead.
int max_clusters_8(int NT) {
  static int cached[64][2] = {{0}};
  int dev = 0;
  cudaGetDevice(&dev);
  const int v = NT <= 32 ? 0 : 1;
  if (dev < 64 && cached[dev][v]) return cached[dev][v];
  int n = 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(8, 16, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 8;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  if (v == 0) {
    cfg.dynamicSmemBytes = sizeof(Smem<8, 32, 4>) + 1024;
    static int conf[64] = {0};
    e = smem_attr_once(proj_decode_kernel<8, 32, 4>, cfg.dynamicSmemBytes, conf);
    if (e == cudaSuccess) e = cudaOccupancyMaxActiveClusters(&n, proj_decode_kernel<8, 32, 4>, &cfg);
  } else {
    cfg.dynamicSmemBytes = sizeof(Smem<8, 64, 3>) + 1024;
    static int conf[64] = {0};
    e = smem_attr_once(proj_decode_kernel<8, 64, 3>, cfg.dynamicSmemBytes, conf);
    if (e == cudaSuccess) e = cudaOccupancyMaxActiveClusters(&n, proj_decode_kernel<8, 64, 3>, &cfg);
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  if (dev < 64) cached[dev][v] = n > 0 ? n : -1;
  return n;
}

cudaError_t launch_proj_decode(const Params& p, cudaStream_t s) {
  const int NT = (p.T + 15) / 16 * 16;
  CUtensorMap mx, mkv, mg;
  if (!make_tile_map(&mx, p.x, p.T, p.H, (uint32_t)NT) || !make_tile_map(&mkv, p.wkv, p.C, p.H, BM) ||
      !make_tile_map(&mg, p.wgate, p.C, p.H, BM))
    return cudaErrorInvalidValue;
  const int tiles = (2 * p.C) / BM;
  const bool wide = max_clusters_8(NT) >= tiles;
  if (NT <= 32)
    return wide ? launch_variant<8, 32, 4>(p, s, NT, mx, mkv, mg) : launch_variant<4, 32, 4>(p, s, NT, mx, mkv, mg);
  return wide ? launch_variant<8, 64, 3>(p, s, NT, mx, mkv, mg) : launch_variant<4, 64, 3>(p, s, NT, mx, mkv, mg);
}

}  // namespace cmp
