// Prefill with the pooling fused into the tensor-core epilogue (sm_100a:
// TMA -> shared memory -> tcgen05.mma -> TMEM -> pooling epilogue).
//
// Work item = one 256-position tile of one sequence, window aligned (it starts
// at position (start_pos/ratio)*ratio + 256k, and ratio divides 256, so no
// window straddles two tiles), times one block of 128 channels of one half of
// the state row (coff = 2: half 0 = columns [0, D) that the *next* window
// uses, half 1 = columns [D, 2D) that this window uses; coff = 1: one half).
// Per k-step two MMAs share the x tile: the 128 wkv rows and the 128 wgate rows
// of the same channels ("compressor torch_extension API", 计算公式 1:
// [kv, score] = X [W^KV, W^Gate]). So TMEM lane i holds channel i's kv
// (columns 0..255) and score (columns 256..511) for all 256 positions, and one
// thread owns one channel of every window in the tile.
//
// The epilogue, per channel and window (计算公式 2-5), adds ape[q mod ratio] to
// the score, takes positions before start_pos from the paged state (only the
// first window of a sequence has any), and runs the per-channel softmax-
// weighted sum over the window's rows. It writes the pooled value y (and, for
// the two halves of a coff = 2 window, the log-sum-exp of its scores so that
// the finish kernel can merge the previous window's half 0 with this window's
// half 1 exactly: the softmax over 8 rows splits into two 4-row softmaxes
// weighted by their exp-sums). The tail rows a later call reads
// (p >= (e/ratio - coff + 1)*ratio) go to the paged fp32 state from here.
//
// Roles (192 threads, one CTA per SM, persistent): warp 0 TMA (3 stages of
// 16 + 16 + 32 KB), warp 1 TMEM owner and MMA issuer (M=128, N=256, K=16, two
// per k-step), warps 2-5 epilogue. All waits are bounded, as in the plain
// projection kernel.
#include <mutex>

#include "cmp_internal.cuh"
#include "cmp_sm100.cuh"

namespace cmp {
namespace {

using namespace sm100;

constexpr int NTOK = 256;   // positions per tile (MMA N)
constexpr int BM = 128;     // channels per item (MMA M)
constexpr int BK = 64;
constexpr int STAGES = 3;
constexpr int kThreads = 192;
constexpr uint32_t kStageBytes = 2 * BM * BK * 2 + NTOK * BK * 2;  // 64 KB
constexpr uint32_t kIdesc = idesc_bf16_f32(BM, NTOK);

struct Smem {
  __nv_bfloat16 a_kv[STAGES][BM * BK];
  __nv_bfloat16 a_g[STAGES][BM * BK];
  __nv_bfloat16 b[STAGES][NTOK * BK];
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t acc_full;
  uint64_t acc_empty;
  uint32_t tmem_base;
  int abort;
};

// What one work item covers.
struct Item {
  int b;      // sequence
  int P0;     // first position of the tile
  int t0;     // x row of position P0 (may lie before the sequence, even < 0)
  int half;   // 0 / 1: which coff half of the state row
  int c0;     // first channel (within the half)
};

__device__ __forceinline__ Item decode_item(const Params& p, int g, int n_cblk) {
  Item it;
  const int tile = g / n_cblk, cb = g % n_cblk;
  const int per_half = p.D / BM;
  it.half = cb / per_half;
  it.c0 = (cb % per_half) * BM;
  it.b = upper_index(p.m_tile, p.B, tile);
  const int k = tile - p.m_tile[it.b];
  const int s = p.m_s[it.b];
  it.P0 = (s / p.ratio) * p.ratio + k * NTOK;
  it.t0 = p.m_cu[it.b] + (it.P0 - s);
  return it;
}

__device__ __forceinline__ int n_items(const Params& p) {
  return p.m_tile[p.B] * (p.coff * p.D / BM);
}

// The epilogue of one item for a compile-time ratio R.
template <int R>
__device__ __forceinline__ void pool_item(const Params& p, const Item& it, uint32_t taddr, int ch) {
  constexpr int COFF = (R == 4) ? 2 : 1;
  const int b = it.b;
  const int s = p.m_s[b];
  const int cu = p.m_cu[b];
  const int e = s + (p.m_cu[b + 1] - cu);
  const int w0 = s / R;        // first window this call completes
  const int w_end = e / R;     // windows below this one complete in this call
  const int off = p.m_off[b];  // output row of window w0
  const int thr = max(s, tail_threshold(e, R, COFF));
  const int col = it.half * p.D + ch;  // column in the coff*D wide state / ape rows
  float* ybase = p.ystat + (int64_t)it.half * p.D + ch;
  float* lbase = p.ylse + (int64_t)it.half * p.D + ch;

  float ap[R <= 32 ? R : 1];
  if constexpr (R <= 32) {
#pragma unroll
    for (int j = 0; j < R; ++j) ap[j] = __ldg(p.ape + (int64_t)j * p.C + col);
  }
  float m = -INFINITY, l = 0.f, acc = 0.f;  // running stats of a window wider than a chunk

#pragma unroll 1
  for (int c = 0; c < NTOK / 32; ++c) {
    const int q0 = it.P0 + c * 32;
    if (q0 >= e) break;  // the rest of the tile lies past the sequence
    uint32_t kr[32], sr[32];
    tmem_ld32(taddr + c * 32, kr);
    tmem_ld32(taddr + NTOK + c * 32, sr);
    tmem_ld_wait(kr);
    tmem_ld_wait(sr);
    float kv[32], z[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      kv[j] = __uint_as_float(kr[j]);
      float a;
      if constexpr (R <= 32) a = ap[j % R];
      else a = __ldg(p.ape + (int64_t)((q0 + j) % R) * p.C + col);
      z[j] = __uint_as_float(sr[j]) + a;
    }
    if (q0 < s) {  // rows written by earlier calls (the first window of the sequence)
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int q = q0 + j;
        if (q < s) {
          const int rk = table_row(p, p.kv_tbl, b, q);
          const int rs = table_row(p, p.sc_tbl, b, q);
          kv[j] = rk >= 0 ? p.kv_state[((int64_t)rk * p.bs + q % p.bs) * p.C + col] : 0.f;
          z[j] = rs >= 0 ? p.score_state[((int64_t)rs * p.bs + q % p.bs) * p.C + col] : -INFINITY;
        }
      }
    }
    if (q0 + 31 >= thr) {  // tail rows: kv and score + ape into the paged state
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int q = q0 + j;
        if (q >= thr && q < e) {
          const int rk = table_row(p, p.kv_tbl, b, q);
          const int rs = table_row(p, p.sc_tbl, b, q);
          if (rk >= 0) p.kv_state[((int64_t)rk * p.bs + q % p.bs) * p.C + col] = kv[j];
          if (rs >= 0) p.score_state[((int64_t)rs * p.bs + q % p.bs) * p.C + col] = z[j];
        }
      }
    }
    if constexpr (R >= 32) {
      // the chunk is one piece of window q0 / R
      const int w = q0 / R;
      if (w < w_end) {
        float mx = z[0];
#pragma unroll
        for (int j = 1; j < 32; ++j) mx = fmaxf(mx, z[j]);
        const float mn = fmaxf(m, mx);
        const float sc = __expf(m - mn);
        l *= sc;
        acc *= sc;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float pz = __expf(z[j] - mn);
          l += pz;
          acc = fmaf(pz, kv[j], acc);
        }
        m = mn;
        if (((c + 1) * 32) % R == 0) {  // last chunk of the window
          const int64_t n = off + (w - w0);
          ybase[n * (COFF * p.D)] = acc / l;
          if (COFF == 2) lbase[n * (COFF * p.D)] = m + __logf(l);
          m = -INFINITY;
          l = 0.f;
          acc = 0.f;
        }
      }
    } else {
#pragma unroll
      for (int k = 0; k < 32 / R; ++k) {  // whole windows inside the chunk
        const int w = (q0 + k * R) / R;
        if (w < w_end) {
          float mx = z[k * R];
#pragma unroll
          for (int j = 1; j < R; ++j) mx = fmaxf(mx, z[k * R + j]);
          float ls = 0.f, as = 0.f;
#pragma unroll
          for (int j = 0; j < R; ++j) {
            const float pz = __expf(z[k * R + j] - mx);
            ls += pz;
            as = fmaf(pz, kv[k * R + j], as);
          }
          const int64_t n = off + (w - w0);
          ybase[n * (COFF * p.D)] = as / ls;
          if (COFF == 2) lbase[n * (COFF * p.D)] = mx + __logf(ls);
        }
      }
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    fused_tc_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_wkv,
                    const __grid_constant__ CUtensorMap map_wg, Params p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_cblk = p.coff * p.D / BM;
  const int k_blocks = p.H / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    mbar_init(&sm.acc_full, 1);
    mbar_init(&sm.acc_empty, 4);
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
  pdl_wait();  // the tile list comes from the scheduler kernel
  const int total = n_items(p);

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      for (int g = blockIdx.x; g < total && !*abort; g += gridDim.x) {
        const Item it = decode_item(p, g, n_cblk);
        const int wrow = it.half * p.D + it.c0;
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (!mbar_wait(&sm.empty[stage], phase ^ 1u, abort)) break;
          mbar_arrive_expect_tx(&sm.full[stage], kStageBytes);
          tma_load_2d(sm.a_kv[stage], &map_wkv, &sm.full[stage], kb * BK, wrow);
          tma_load_2d(sm.a_g[stage], &map_wg, &sm.full[stage], kb * BK, wrow);
          tma_load_2d(sm.b[stage], &map_x, &sm.full[stage], kb * BK, it.t0);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t acc_phase = 0;
      for (int g = blockIdx.x; g < total && !*abort; g += gridDim.x) {
        if (!mbar_wait(&sm.acc_empty, acc_phase ^ 1u, abort)) break;
        tc_fence_after();
        bool ok = true;
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (!mbar_wait(&sm.full[stage], phase, abort)) { ok = false; break; }
          tc_fence_after();
          const uint32_t akv = smem_u32(sm.a_kv[stage]);
          const uint32_t ag = smem_u32(sm.a_g[stage]);
          const uint32_t b0 = smem_u32(sm.b[stage]);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t bd = sw128_kmajor_desc(b0 + k * 32);
            const uint32_t accum = (kb > 0 || k > 0) ? 1u : 0u;
            mma_bf16(tmem, sw128_kmajor_desc(akv + k * 32), bd, kIdesc, accum);
            mma_bf16(tmem + NTOK, sw128_kmajor_desc(ag + k * 32), bd, kIdesc, accum);
          }
          mma_commit(&sm.empty[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        mma_commit(&sm.acc_full);
        acc_phase ^= 1u;
      }
    }
  } else {
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16);
    uint32_t acc_phase = 0;
    for (int g = blockIdx.x; g < total; g += gridDim.x) {
      const Item it = decode_item(p, g, n_cblk);
      const bool ok = mbar_wait(&sm.acc_full, acc_phase, abort);
      if (!bar_and(1, 128, ok)) break;  // all four warps leave together
      tc_fence_after();
      const int ch = it.c0 + row;
      switch (p.ratio) {
        case 1: pool_item<1>(p, it, taddr, ch); break;
        case 2: pool_item<2>(p, it, taddr, ch); break;
        case 4: pool_item<4>(p, it, taddr, ch); break;
        case 8: pool_item<8>(p, it, taddr, ch); break;
        case 16: pool_item<16>(p, it, taddr, ch); break;
        case 32: pool_item<32>(p, it, taddr, ch); break;
        case 64: pool_item<64>(p, it, taddr, ch); break;
        default: pool_item<128>(p, it, taddr, ch); break;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.acc_empty);
      acc_phase ^= 1u;
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

}  // namespace

bool fused_supported(const Params& p) {
  return p.H % BK == 0 && p.D % BM == 0 && NTOK % p.ratio == 0 && encode_fn() != nullptr;
}

// Upper bound of the work items of a call (the exact count is on the device):
// every sequence adds at most one partial tile at each end.
int fused_max_items(const Params& p) {
  const int64_t tiles = ((int64_t)p.T + NTOK - 1) / NTOK + 2LL * p.B;
  return (int)(tiles * (p.coff * p.D / BM));
}

cudaError_t launch_fused(const Params& p, cudaStream_t s, int sm_count) {
  CUtensorMap mx, mkv, mg;
  if (!make_tile_map(&mx, p.x, p.T, p.H, NTOK) || !make_tile_map(&mkv, p.wkv, p.C, p.H, BM) ||
      !make_tile_map(&mg, p.wgate, p.C, p.H, BM))
    return cudaErrorInvalidValue;
  const size_t smem = sizeof(Smem) + 1024;
  static int configured[64] = {0};
  const cudaError_t e = smem_attr_once(fused_tc_kernel, smem, configured);
  if (e != cudaSuccess) return e;
  const int items = fused_max_items(p);
  const int grid = items < sm_count ? items : sm_count;
  return launch_chained(fused_tc_kernel, dim3(grid), dim3(kThreads), smem, s, 1, mx, mkv, mg, p);
}

}  // namespace cmp
