// Prefill projection on the sm_100a tensor cores: TMA -> shared memory ->
// tcgen05.mma -> TMEM -> epilogue.
//
//   proj[t][n] = sum_k W[n][k] * x[t][k]   (W = wkv for n < C, wgate for n >= C)
// ("compressor torch_extension API", 计算公式 1-2), raw scores (the pooling
// kernel adds ape[p mod ratio]); the state tail rows (positions
// p >= (e/ratio - coff + 1)*ratio of their sequence, score rows with ape) go
// straight into the paged fp32 kv_state / score_state from the epilogue.
//
// Layout of the contraction: the weight rows are the MMA's M side (128 rows of
// wkv or wgate per tile) and the tokens its N side (256 per tile), so an
// accumulator lane is one channel and its columns are tokens: every epilogue
// store of a warp is 32 consecutive channels of one token row (128 bytes).
//
// Warp roles (192 threads, one CTA per SM, persistent over tiles):
//   warp 0     TMA producer: W tile 128x64 and x tile 256x64 per stage (48 KB)
//   warp 1     owns TMEM (512 columns = two 256-column fp32 accumulators) and
//              issues tcgen05.mma (M=128, N=256, K=16) from one thread
//   warps 2-5  epilogue: tcgen05.ld, fp32 stores, tail-state stores (+ ape)
// Four shared-memory stages; the two accumulators let the epilogue of one
// tile overlap the main loop of the next. Every wait is bounded: a role that
// gives up raises the CTA's abort flag and the device error word, and all
// roles then leave their loops, so the kernel always ends.
#include <mutex>

#include "cmp_internal.cuh"
#include "cmp_sm100.cuh"

namespace cmp {
namespace {

using namespace sm100;

constexpr int BM = 128;   // weight rows per tile (MMA M)
constexpr int BN = 256;   // tokens per tile (MMA N)
constexpr int BK = 64;    // K per stage: one 128-byte swizzle row
constexpr int STAGES = 4;
constexpr int kThreads = 192;
constexpr uint32_t kStageBytesA = BM * BK * 2;  // 16 KB
constexpr uint32_t kStageBytesB = BN * BK * 2;  // 32 KB
constexpr uint32_t kIdesc = idesc_bf16_f32(BM, BN);

struct TokInfo {
  int32_t ape_row;   // position mod ratio (used on tail rows only)
  int32_t pad;
  int64_t kv_off;    // element offset of the token's kv_state row, or -1 (not a tail row)
  int64_t sc_off;    // element offset of the token's score_state row, or -1
};

struct Smem {
  // 1024-byte aligned operand stages first
  __nv_bfloat16 a[STAGES][BM * BK];
  __nv_bfloat16 b[STAGES][BN * BK];
  TokInfo tok[2][BN];
  uint32_t tail_mask[2][BN / 32];  // per 32-token chunk: which tokens are state tail rows
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// Per-token facts of one tile, computed by the 128 epilogue threads while the
// tile's main loop runs: which tokens are state tail rows and where they go.
__device__ void fill_tok_info(const Params& p, TokInfo* info, uint32_t* tail_mask, int n0, int e_tid) {
  for (int j = e_tid; j < BN; j += 128) {
    TokInfo ti{0, 0, -1, -1};
    bool tail = false;
    const int t = n0 + j;
    if (t < p.T) {
      const int b = upper_index(p.m_cu, p.B, t);
      if (b < p.B) {
        const int s = p.m_s[b];
        const int c0 = p.m_cu[b];
        const int pos = s + (t - c0);
        const int e = s + (p.m_cu[b + 1] - c0);
        if (pos >= tail_threshold(e, p.ratio, p.coff)) {
          ti.ape_row = pos % p.ratio;
          const int rk = table_row(p, p.kv_tbl, b, pos);
          const int rs = table_row(p, p.sc_tbl, b, pos);
          if (rk >= 0) ti.kv_off = ((int64_t)rk * p.bs + pos % p.bs) * p.C;
          if (rs >= 0) ti.sc_off = ((int64_t)rs * p.bs + pos % p.bs) * p.C;
          tail = true;
        }
      }
    }
    info[j] = ti;
    const unsigned m = __ballot_sync(0xffffffffu, tail);  // j = e_tid + 128 i: one warp = one chunk
    if ((j & 31) == 0) tail_mask[j >> 5] = m;
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    proj_tc_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_wkv,
                   const __grid_constant__ CUtensorMap map_wg, Params p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int n_m = (2 * p.C) / BM;
  const int n_n = (p.T + BN - 1) / BN;
  const int n_tiles = n_m * n_n;
  const int k_blocks = p.H / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&sm.acc_full[a], 1);
      mbar_init(&sm.acc_empty[a], 4);
    }
    sm.abort = 0;
    fence_barrier_init();
    prefetch_tmap(&map_x);
    prefetch_tmap(&map_wkv);
    prefetch_tmap(&map_wg);
  }
  if (warp == 1) tmem_alloc(&sm.tmem_base, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort = &sm.abort;
  pdl_trigger();

  if (warp == 0) {
    // ---------------- TMA producer (x and the weights are call inputs) ----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      for (int tile = blockIdx.x; tile < n_tiles && !*abort; tile += gridDim.x) {
        const int m0 = (tile % n_m) * BM;
        const int n0 = (tile / n_m) * BN;
        const CUtensorMap* wmap = m0 < p.C ? &map_wkv : &map_wg;
        const int wrow = m0 < p.C ? m0 : m0 - p.C;
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (!mbar_wait(&sm.empty[stage], phase ^ 1u, abort)) break;
          mbar_arrive_expect_tx(&sm.full[stage], kStageBytesA + kStageBytesB);
          tma_load_2d(sm.a[stage], wmap, &sm.full[stage], kb * BK, wrow);
          tma_load_2d(sm.b[stage], &map_x, &sm.full[stage], kb * BK, n0);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      for (int tile = blockIdx.x; tile < n_tiles && !*abort; tile += gridDim.x, ++local) {
        const int acc = local & 1;
        const uint32_t acc_phase = (local >> 1) & 1;
        if (!mbar_wait(&sm.acc_empty[acc], acc_phase ^ 1u, abort)) break;
        tc_fence_after();
        const uint32_t d = tmem + acc * BN;
        bool ok = true;
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (!mbar_wait(&sm.full[stage], phase, abort)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sm.a[stage]);
          const uint32_t b0 = smem_u32(sm.b[stage]);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            // advance 16 bf16 = 32 bytes along K inside the 128-byte swizzle row
            mma_bf16(d, sw128_kmajor_desc(a0 + k * 32), sw128_kmajor_desc(b0 + k * 32), kIdesc,
                     (kb > 0 || k > 0) ? 1u : 0u);
          }
          mma_commit(&sm.empty[stage]);  // frees the stage once these MMAs have read it
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        mma_commit(&sm.acc_full[acc]);   // accumulator ready for the epilogue
      }
    }
  } else {
    // ---------------- epilogue (warps 2..5) ----------------
    pdl_wait();  // reads the scheduler's metadata, writes proj and the state
    const int e_tid = threadIdx.x - 64;
    const int quad = warp & 3;            // TMEM lanes this warp may access
    const int row = quad * 32 + lane;     // weight row within the tile = TMEM lane
    int local = 0;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++local) {
      const int m0 = (tile % n_m) * BM;
      const int n0 = (tile / n_m) * BN;
      TokInfo* info = sm.tok[local & 1];
      uint32_t* tmask = sm.tail_mask[local & 1];
      fill_tok_info(p, info, tmask, n0, e_tid);
      epi_bar();
      const int acc = local & 1;
      const uint32_t acc_phase = (local >> 1) & 1;
      const bool ok = mbar_wait(&sm.acc_full[acc], acc_phase, abort);
      if (!bar_and(1, 128, ok)) break;  // all four warps leave together
      tc_fence_after();
      const bool score = m0 >= p.C;
      const int col = (score ? m0 - p.C : m0) + row;  // channel within kv or score
      float* proj_col = p.proj + (score ? p.C : 0) + col;
      float* state = score ? p.score_state : p.kv_state;
      const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16) + acc * BN;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(taddr + c * 32, r);
        tmem_ld_wait(r);
        const int t0 = n0 + c * 32;
        const int jmax = p.T - t0;  // tokens past T are padding
        float* dst = proj_col + (int64_t)t0 * (2 * p.C);
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (j < jmax) dst[(int64_t)j * (2 * p.C)] = __uint_as_float(r[j]);
        const uint32_t m = tmask[c];
        if (m) {  // rare: state tail rows (score rows carry ape in the state)
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            if (m & (1u << j)) {
              const TokInfo ti = info[c * 32 + j];
              const int64_t so = score ? ti.sc_off : ti.kv_off;
              float v = __uint_as_float(r[j]);
              if (score) v += __ldg(p.ape + (int64_t)ti.ape_row * p.C + col);
              if (so >= 0) state[so + col] = v;
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.acc_empty[acc]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (threadIdx.x == 0 && sm.abort) atomicOr(p.err, kErrTimeout);
}

// ---- host side ------------------------------------------------------------------

int sm_count() {
  int dev = 0, n = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

}  // namespace

bool proj_tc_supported(const Params& p) {
  return p.T >= 128 && p.H % BK == 0 && (2 * p.C) % BM == 0 && encode_fn() != nullptr;
}

cudaError_t launch_proj_tc(const Params& p, cudaStream_t s) {
  CUtensorMap mx, mkv, mg;
  if (!make_tile_map(&mx, p.x, p.T, p.H, BN) || !make_tile_map(&mkv, p.wkv, p.C, p.H, BM) ||
      !make_tile_map(&mg, p.wgate, p.C, p.H, BM))
    return cudaErrorInvalidValue;
  const size_t smem = sizeof(Smem) + 1024;
  static int configured[64] = {0};
  const cudaError_t e = smem_attr_once(proj_tc_kernel, smem, configured);
  if (e != cudaSuccess) return e;
  const int n_tiles = ((2 * p.C) / BM) * ((p.T + BN - 1) / BN);
  const int grid = n_tiles < sm_count() ? n_tiles : sm_count();
  return launch_chained(proj_tc_kernel, dim3(grid), dim3(kThreads), smem, s, 1, mx, mkv, mg, p);
}

}  // namespace cmp
