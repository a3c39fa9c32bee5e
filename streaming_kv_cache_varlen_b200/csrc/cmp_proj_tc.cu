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
// wkv or wgate per tile) and the tokens its N side (BN per tile), so an
// accumulator lane is one channel and its columns are tokens: every epilogue
// store of a warp is 32 consecutive channels of one token row (128 bytes).
//
// BN (128 .. 256 tokens, a multiple of 16) is chosen per call so that the
// tiles fill the SMs in whole waves as nearly as possible: with 2C = 512 rows
// and ~10K tokens, 256-token tiles make 160-200 tiles, i.e. a second wave that
// keeps only a few SMs busy; narrower tiles spread the same work over all SMs.
// The stage ring takes as many stages as fit (4 at BN = 256, 5-6 below).
//
// Warp roles (192 threads, one CTA per SM, persistent over tiles):
//   warp 0     TMA producer: W tile 128x64 and x tile BNx64 per stage
//   warp 1     owns TMEM (512 columns = two 256-column fp32 accumulators) and
//              issues tcgen05.mma (M=128, N=BN, K=16) from one thread
//   warps 2-5  epilogue: tcgen05.ld, fp32 stores, tail-state stores (+ ape)
// The two accumulators let the epilogue of one tile overlap the main loop of
// the next. Every wait is bounded: a role that gives up raises the CTA's abort
// flag and the device error word, and all roles then leave their loops, so
// the kernel always ends.
#include <mutex>

#include "cmp_internal.cuh"
#include "cmp_sm100.cuh"

namespace cmp {
namespace {

using namespace sm100;

constexpr int BM = 128;    // weight rows per tile (MMA M)
constexpr int BNMAX = 256; // tokens per tile (MMA N) at most
constexpr int BK = 64;     // K per stage: one 128-byte swizzle row
constexpr int MAXST = 8;
constexpr int kThreads = 192;
constexpr uint32_t kStageBytesA = BM * BK * 2;  // 16 KB
constexpr size_t kSmemLimit = 232448;           // 227 KB of dynamic shared memory

struct TokInfo {
  int32_t ape_row;   // position mod ratio (used on tail rows only)
  int32_t pad;
  int64_t kv_off;    // element offset of the token's kv_state row, or -1 (not a tail row)
  int64_t sc_off;    // element offset of the token's score_state row, or -1
};

// Shared memory: `stages` operand stages of kStageBytesA + BN*128 bytes (W tile,
// then x tile; both 1024-byte aligned), then this.
struct Tail {
  TokInfo tok[2][BNMAX];
  uint32_t tail_mask[2][BNMAX / 32];  // per 32-token chunk: which tokens are state tail rows
  uint64_t full[MAXST];
  uint64_t empty[MAXST];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint32_t tmem_base;
  int abort;
};

__host__ __device__ constexpr uint32_t stage_bytes(int bn) { return kStageBytesA + (uint32_t)bn * BK * 2; }

__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// Per-token facts of one tile, computed by the 128 epilogue threads while the
// tile's main loop runs: which tokens are state tail rows and where they go.
__device__ void fill_tok_info(const Params& p, TokInfo* info, uint32_t* tail_mask, int n0, int e_tid, int bn) {
  const int bn32 = (bn + 31) & ~31;  // whole warps in the ballot (bn may end on half a chunk)
  for (int j = e_tid; j < bn32; j += 128) {
    TokInfo ti{0, 0, -1, -1};
    bool tail = false;
    const int t = n0 + j;
    if (j < bn && t < p.T) {
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
    if (j < bn) info[j] = ti;
    const unsigned m = __ballot_sync(0xffffffffu, tail);  // j = e_tid + 128 i: one warp = one chunk
    if ((j & 31) == 0) tail_mask[j >> 5] = m;
  }
}

// One warp's 32 accumulator lanes (weight row m of 2C, one per lane) over the
// tile's bn tokens from n0: fp32 projection rows, and the state tail rows
// (score rows with ape added) of the tokens the tile info marks.
__device__ __forceinline__ void store_accumulator(const Params& p, uint32_t taddr, int m, int n0, int bn,
                                                  const TokInfo* info, const uint32_t* tmask) {
  const bool score = m >= p.C;
  const int col = score ? m - p.C : m;  // channel within kv or score
  float* proj_col = p.proj + (score ? p.C : 0) + col;
  float* state = score ? p.score_state : p.kv_state;
#pragma unroll 1
  for (int c = 0; c < (bn + 31) / 32; ++c) {
    uint32_t r[32];
    if (c * 32 + 32 <= bn) {
      tmem_ld32(taddr + c * 32, r);
      tmem_ld_wait(r);
    } else {  // a last chunk of 16 columns (bn = 16 mod 32)
      uint32_t h[16];
      tmem_ld16(taddr + c * 32, h);
      tmem_ld_wait16(h);
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        r[j] = h[j];
        r[16 + j] = 0u;
      }
    }
    const int t0 = n0 + c * 32;
    const int jmax = min(p.T - t0, bn - c * 32);  // tokens past T or past the tile are not stored
    float* dst = proj_col + (int64_t)t0 * (2 * p.C);
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (j < jmax) dst[(int64_t)j * (2 * p.C)] = __uint_as_float(r[j]);
    const uint32_t msk = tmask[c];
    if (msk) {  // rare: state tail rows (score rows carry ape in the state)
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        if (msk & (1u << j)) {
          const TokInfo ti = info[c * 32 + j];
          const int64_t so = score ? ti.sc_off : ti.kv_off;
          float v = __uint_as_float(r[j]);
          if (score) v += __ldg(p.ape + (int64_t)ti.ape_row * p.C + col);
          if (so >= 0) state[so + col] = v;
        }
      }
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    proj_tc_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_wkv,
                   const __grid_constant__ CUtensorMap map_wg, Params p, int bn, int stages) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* ring = &smem_align1024<unsigned char>(smem_raw);
  const uint32_t sbytes = stage_bytes(bn);
  Tail& sm = *reinterpret_cast<Tail*>(ring + (size_t)stages * sbytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t idesc = idesc_bf16_f32(BM, bn);

  const int n_m = (2 * p.C) / BM;
  const int n_n = (p.T + bn - 1) / bn;
  const int n_tiles = n_m * n_n;
  const int k_blocks = p.H / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
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
      Armed armed;
      for (int tile = blockIdx.x; tile < n_tiles && !*abort; tile += gridDim.x) {
        const int m0 = (tile % n_m) * BM;
        const int n0 = (tile / n_m) * bn;
        const CUtensorMap* wmap = m0 < p.C ? &map_wkv : &map_wg;
        const int wrow = m0 < p.C ? m0 : m0 - p.C;
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (!mbar_wait(&sm.empty[stage], phase ^ 1u, abort)) break;
          mbar_arrive_expect_tx(&sm.full[stage], sbytes);
          armed.note(stage, phase);
          unsigned char* st = ring + (size_t)stage * sbytes;
          tma_load_2d(st, wmap, &sm.full[stage], kb * BK, wrow);
          tma_load_2d(st + kStageBytesA, &map_x, &sm.full[stage], kb * BK, n0);
          if (++stage == stages) { stage = 0; phase ^= 1u; }
        }
      }
      drain_armed(sm.full, stages, armed);  // no copy still landing when the CTA leaves
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
        const uint32_t d = tmem + acc * BNMAX;
        bool ok = true;
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (!mbar_wait(&sm.full[stage], phase, abort)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(ring + (size_t)stage * sbytes);
          const uint32_t b0 = a0 + kStageBytesA;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            // advance 16 bf16 = 32 bytes along K inside the 128-byte swizzle row
            mma_bf16(d, sw128_kmajor_desc(a0 + k * 32), sw128_kmajor_desc(b0 + k * 32), idesc,
                     (kb > 0 || k > 0) ? 1u : 0u);
          }
          mma_commit(&sm.empty[stage]);  // frees the stage once these MMAs have read it
          if (++stage == stages) { stage = 0; phase ^= 1u; }
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
      const int n0 = (tile / n_m) * bn;
      TokInfo* info = sm.tok[local & 1];
      uint32_t* tmask = sm.tail_mask[local & 1];
      fill_tok_info(p, info, tmask, n0, e_tid, bn);
      epi_bar();
      const int acc = local & 1;
      const uint32_t acc_phase = (local >> 1) & 1;
      const bool ok = mbar_wait(&sm.acc_full[acc], acc_phase, abort);
      if (!bar_and(1, 128, ok)) break;  // all four warps leave together
      tc_fence_after();
      store_accumulator(p, tmem + ((uint32_t)(quad * 32) << 16) + acc * BNMAX, m0 + row, n0, bn, info, tmask);
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

// ---- CTA pairs -------------------------------------------------------------------
//
// The same projection with tcgen05.mma.cta_group::2 on clusters of two CTAs:
// a pair tile is 256 weight rows x BN tokens; each CTA loads its 128 weight
// rows and BN/2 of the tokens (16 + BN/16 KB per k-step instead of 16 + BN/8),
// the even CTA issues M=256 MMAs that read both CTAs' shared memory, and each
// SM's TMEM receives its 128 rows for all BN tokens. Each SM then moves a third
// less data per MMA and holds 6-8 stages, so more of the load latency is hidden.
// Both CTAs' loads count on the even CTA's stage barrier; the MMA commits
// arrive on the stage and accumulator barriers of both CTAs; both epilogues
// report a drained accumulator to the even CTA. Every copy lands in the issuing CTA's own shared memory.
constexpr int BMP = 256;  // weight rows per pair tile (MMA M over the pair)

__host__ __device__ constexpr uint32_t stage_bytes_pair(int bn) {
  return kStageBytesA + (uint32_t)(bn / 2) * BK * 2;
}

__global__ void __launch_bounds__(kThreads, 1)
    proj_tc_pair_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_wkv,
                        const __grid_constant__ CUtensorMap map_wg, Params p, int bn, int stages) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* ring = &smem_align1024<unsigned char>(smem_raw);
  const uint32_t sbytes = stage_bytes_pair(bn);
  Tail& sm = *reinterpret_cast<Tail*>(ring + (size_t)stages * sbytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: the CTA that issues the pair's MMAs
  const uint32_t idesc = idesc_bf16_f32(BMP, bn);
  const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;

  const int n_m = (2 * p.C) / BMP;
  const int n_n = (p.T + bn - 1) / bn;
  const int n_tiles = n_m * n_n;
  const int k_blocks = p.H / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&sm.acc_full[a], 1);
      mbar_init(&sm.acc_empty[a], 8);  // the four epilogue warps of both CTAs
    }
    sm.abort = 0;
    fence_barrier_init();
    prefetch_tmap(&map_x);
    prefetch_tmap(&map_wkv);
    prefetch_tmap(&map_wg);
  }
  if (warp == 1) tmem_alloc_pair(&sm.tmem_base, 512);
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers exist before either signals the other's
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort = &sm.abort;
  const uint32_t full0 = mapa_shared(smem_u32(&sm.full[0]), 0);        // the even CTA's stage barriers
  const uint32_t acc_empty0 = mapa_shared(smem_u32(&sm.acc_empty[0]), 0);
  pdl_trigger();

  if (warp == 0) {
    // ---------------- TMA producer (both CTAs: own weight rows, own half of the tokens) ----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      Armed armed;
      for (int tile = pair; tile < n_tiles && !*abort; tile += n_pairs) {
        const int m0 = (tile % n_m) * BMP + (int)rank * BM;
        const int n0 = (tile / n_m) * bn + (int)rank * (bn / 2);
        const CUtensorMap* wmap = m0 < p.C ? &map_wkv : &map_wg;
        const int wrow = m0 < p.C ? m0 : m0 - p.C;
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (!mbar_wait(&sm.empty[stage], phase ^ 1u, abort)) break;
          if (rank == 0) {
            mbar_arrive_expect_tx(&sm.full[stage], 2 * sbytes);
            armed.note(stage, phase);
          }
          unsigned char* st = ring + (size_t)stage * sbytes;
          tma_load_2d_pair(st, wmap, full0 + 8u * stage, kb * BK, wrow);
          tma_load_2d_pair(st + kStageBytesA, &map_x, full0 + 8u * stage, kb * BK, n0);
          if (++stage == stages) { stage = 0; phase ^= 1u; }
        }
      }
      drain_armed(sm.full, stages, armed);  // the pair's copies (counted here on the even CTA)
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (even CTA) ----------------
    if (rank == 0 && lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      for (int tile = pair; tile < n_tiles && !*abort; tile += n_pairs, ++local) {
        const int acc = local & 1;
        const uint32_t acc_phase = (local >> 1) & 1;
        if (!mbar_wait(&sm.acc_empty[acc], acc_phase ^ 1u, abort)) break;
        tc_fence_after();
        const uint32_t d = tmem + acc * BNMAX;
        bool ok = true;
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (!mbar_wait(&sm.full[stage], phase, abort)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(ring + (size_t)stage * sbytes);
          const uint32_t b0 = a0 + kStageBytesA;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            mma_bf16_pair(d, sw128_kmajor_desc(a0 + k * 32), sw128_kmajor_desc(b0 + k * 32), idesc,
                          (kb > 0 || k > 0) ? 1u : 0u);
          mma_commit_pair(&sm.empty[stage], 0x3);  // frees the stage in both CTAs
          if (++stage == stages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        mma_commit_pair(&sm.acc_full[acc], 0x3);  // both halves of the accumulator ready
      }
    }
  } else {
    // ---------------- epilogue (warps 2..5 of both CTAs: this CTA's 128 rows) ----------------
    pdl_wait();  // reads the scheduler's metadata, writes proj and the state
    const int e_tid = threadIdx.x - 64;
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    int local = 0;
    for (int tile = pair; tile < n_tiles; tile += n_pairs, ++local) {
      const int m0 = (tile % n_m) * BMP + (int)rank * BM;
      const int n0 = (tile / n_m) * bn;
      TokInfo* info = sm.tok[local & 1];
      uint32_t* tmask = sm.tail_mask[local & 1];
      fill_tok_info(p, info, tmask, n0, e_tid, bn);
      epi_bar();
      const int acc = local & 1;
      const uint32_t acc_phase = (local >> 1) & 1;
      const bool ok = mbar_wait(&sm.acc_full[acc], acc_phase, abort);
      if (!bar_and(1, 128, ok)) break;  // all four warps leave together
      tc_fence_after();
      store_accumulator(p, tmem + ((uint32_t)(quad * 32) << 16) + acc * BNMAX, m0 + row, n0, bn, info, tmask);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty0 + 8u * acc);
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // neither CTA leaves while the other may still signal its barriers
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
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

// The tile width for T tokens (128 .. 256, a multiple of 16): the fewest waves
// of tiles over the `slots` concurrent tiles, each wave costing its tile width
// plus ~32 tokens' worth of per-tile overhead (ties go to the wider tile).
int tile_tokens(int64_t n_m, int T, int slots) {
  int best = BNMAX;
  int64_t best_cost = -1;
  for (int bn = BNMAX; bn >= 128; bn -= 16) {
    const int64_t tiles = n_m * ((T + bn - 1) / bn);
    const int64_t cost = ((tiles + slots - 1) / slots) * (bn + 32);
    if (best_cost < 0 || cost < best_cost) {
      best = bn;
      best_cost = cost;
    }
  }
  return best;
}

// Per device: the pair kernel's co-resident clusters (0: not measured yet,
// -1: the device refused the cluster form, use the single-CTA kernel).
int g_pair_slots[64] = {0};

cudaError_t launch_single(const Params& p, cudaStream_t s, int sms) {
  const int bn = tile_tokens((2 * p.C) / BM, p.T, sms);
  const size_t ring_max = kSmemLimit - 1024 - sizeof(Tail);
  int stages = (int)(ring_max / stage_bytes(bn));
  if (stages > MAXST) stages = MAXST;
  CUtensorMap mx, mkv, mg;
  if (!make_tile_map(&mx, p.x, p.T, p.H, bn) || !make_tile_map(&mkv, p.wkv, p.C, p.H, BM) ||
      !make_tile_map(&mg, p.wgate, p.C, p.H, BM))
    return cudaErrorInvalidValue;
  const size_t smem = (size_t)stages * stage_bytes(bn) + sizeof(Tail) + 1024;
  static int configured[64] = {0};
  const cudaError_t e = smem_attr_once(proj_tc_kernel, kSmemLimit, configured);
  if (e != cudaSuccess) return e;
  const int n_tiles = ((2 * p.C) / BM) * ((p.T + bn - 1) / bn);
  const int grid = n_tiles < sms ? n_tiles : sms;
  return launch_chained(proj_tc_kernel, dim3(grid), dim3(kThreads), smem, s, 1, mx, mkv, mg, p, bn, stages);
}

// The pair kernel's launch: returns cudaErrorNotSupported (nothing launched)
// when the device cannot co-schedule its clusters.
cudaError_t launch_pair(const Params& p, cudaStream_t s, int dev) {
  static int configured[64] = {0};
  cudaError_t e = smem_attr_once(proj_tc_pair_kernel, kSmemLimit, configured);
  if (e != cudaSuccess) return e;
  int& slots = g_pair_slots[dev];
  if (slots == 0) {  // how many 2-CTA clusters of the largest footprint fit at once
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemLimit;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 2;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, proj_tc_pair_kernel, &cfg) != cudaSuccess || n < 1) {
      cudaGetLastError();
      slots = -1;
    } else {
      slots = n;
    }
  }
  if (slots < 0) return cudaErrorNotSupported;
  const int bn = tile_tokens((2 * p.C) / BMP, p.T, slots);
  const size_t ring_max = kSmemLimit - 1024 - sizeof(Tail);
  int stages = (int)(ring_max / stage_bytes_pair(bn));
  if (stages > MAXST) stages = MAXST;
  CUtensorMap mx, mkv, mg;
  if (!make_tile_map(&mx, p.x, p.T, p.H, bn / 2) || !make_tile_map(&mkv, p.wkv, p.C, p.H, BM) ||
      !make_tile_map(&mg, p.wgate, p.C, p.H, BM))
    return cudaErrorInvalidValue;
  const size_t smem = (size_t)stages * stage_bytes_pair(bn) + sizeof(Tail) + 1024;
  const int n_tiles = ((2 * p.C) / BMP) * ((p.T + bn - 1) / bn);
  const int pairs = n_tiles < slots ? n_tiles : slots;
  return launch_chained(proj_tc_pair_kernel, dim3(2 * pairs), dim3(kThreads), smem, s, 2, mx, mkv, mg, p, bn,
                        stages);
}

}  // namespace

bool proj_tc_supported(const Params& p) {
  return p.T >= 128 && p.H % BK == 0 && (2 * p.C) % BM == 0 && encode_fn() != nullptr;
}

// CTA pairs when the rows split into 256-row pair tiles (always: 2C is 256,
// 512, 1024 or 2048), unless the call asks for single CTAs or the device
// cannot co-schedule the clusters.
cudaError_t launch_proj_tc(const Params& p, cudaStream_t s) {
  int dev = 0;
  cudaGetDevice(&dev);
  const int sms = sm_count();
  if (p.T >= 256 && (2 * p.C) % BMP == 0 && dev < 64 && g_pair_slots[dev] >= 0 && !p.single_cta) {
    const cudaError_t e = launch_pair(p, s, dev);
    if (e == cudaSuccess || e == cudaErrorInvalidValue) return e;
    // refused before anything ran (a cluster form this device will not
    // schedule): single CTAs from now on
    cudaGetLastError();
    g_pair_slots[dev] = -1;
  }
  return launch_single(p, s, sms);
}

}  // namespace cmp
