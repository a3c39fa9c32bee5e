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
// thread owns one channel of every window in a 64-position quarter of the tile.
//
// The epilogue, per channel and window (计算公式 2-5), adds ape[q mod ratio] to
// the score, takes positions before start_pos from the paged state (only the
// first window of a sequence has any), and runs the per-channel softmax-
// weighted sum over the window's rows. It writes the pooled value y (and, for
// the two halves of a coff = 2 window, the log-sum-exp of its scores so that
// the row's finish can merge the previous window's half 0 with this window's
// half 1 exactly: the softmax over 8 rows splits into two 4-row softmaxes
// weighted by their exp-sums). The tail rows a later call reads
// (p >= (e/ratio - coff + 1)*ratio) go to the paged fp32 state from here.
//
// Roles (576 threads, one CTA per SM, persistent): warp 0 TMA (3 stages of
// 16 + 16 + 32 KB; CTA pairs: 4 of 16 + 16 + 16 KB), warp 1 TMEM owner and MMA
// issuer (M=128, N=256, K=16, two per k-step; pairs: M=256 over both CTAs),
// warps 2-17 epilogue: four warps per TMEM lane quarter, one for each
// 64-position quarter of the tile (a ratio-128 window spans two quarters, whose
// warps merge their softmax stats through shared memory), so the accumulator —
// all 512 TMEM columns, which the next item's MMAs must wait for — drains with
// four independent chains of TMEM loads per lane quarter. All waits are
// bounded: a role that gives up raises the CTA's abort flag and the device
// error word, and all roles then leave their loops, so the kernel always ends.
//
// Folded mode (no rotation, B <= kMetaSeqs, tile counters available): the call
// is this one kernel.
//  * Every CTA validates cu_seqlens / start_pos and builds the per-sequence
//    metadata (token offsets, start positions, first output rows, first work
//    tiles) in its shared memory, as the scheduler kernel otherwise does.
//  * Each item, once pooled, arrives on its tile's counter (and, for coff = 2,
//    on the next tile's, whose first window needs this tile's half 0). The CTA
//    whose arrival completes a counter finishes that tile's output rows:
//    merge of the halves (coff = 2), RMSNorm, RoPE, bf16 store. Nobody waits:
//    the last arriver does the work, then puts the counter back to zero for the
//    next call (a kernel of the next call touches the counters only after its
//    griddepcontrol.wait, i.e. after this grid has completed).
//  * Rows that hold no window are zeroed by the epilogue warps, spread over
//    the CTAs by sequence.
// Otherwise the scheduler kernel runs before (metadata, hadamard check) and the
// finish kernel after this one.
#include <mutex>

#include "cmp_internal.cuh"
#include "cmp_rowpost.cuh"
#include "cmp_sm100.cuh"

namespace cmp {
namespace {

using namespace sm100;

constexpr int NTOK = 256;   // positions per tile (MMA N)
constexpr int BM = 128;     // channels per item (MMA M per CTA)
constexpr int BK = 64;
constexpr int kThreads = 576;
constexpr int kEpiThreads = 512;  // warps 2-17
constexpr int kMetaSeqs = 512;    // folded mode: sequences whose metadata fits in shared memory

// Single CTAs: 3 stages of 16 + 16 + 32 KB (the whole 256-position x tile).
// CTA pairs: 4 stages of 16 + 16 + 16 KB (each CTA holds half of the x tile).
template <bool PAIR>
struct Cfg {
  static constexpr int ST = PAIR ? 4 : 3;
  static constexpr int NB = PAIR ? NTOK / 2 : NTOK;  // x rows per CTA and stage
  static constexpr uint32_t kStageBytes = 2 * BM * BK * 2 + NB * BK * 2;
  static constexpr uint32_t kIdesc = idesc_bf16_f32(PAIR ? 2 * BM : BM, NTOK);
};

template <bool PAIR>
struct SmemT {
  static constexpr int STAGES = Cfg<PAIR>::ST;
  __nv_bfloat16 a_kv[STAGES][BM * BK];
  __nv_bfloat16 a_g[STAGES][BM * BK];
  __nv_bfloat16 b[STAGES][Cfg<PAIR>::NB * BK];
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t acc_full;
  uint64_t acc_empty;
  uint32_t tmem_base;
  int abort;
  // folded mode: per-sequence metadata, the block scan's scratch, the tiles
  // this CTA finishes after its current item
  int32_t m_cu[kMetaSeqs + 1];
  int32_t m_s[kMetaSeqs];
  int32_t m_off[kMetaSeqs + 1];
  int32_t m_tile[kMetaSeqs + 1];
  int scan_w[32];
  int scan_tot;
  int bad;
  int fin[2];
  int nfin;
  // ratio 128: running softmax stats of the first 64 positions of each window,
  // per TMEM lane quarter and lane, handed to the warp that ends the window
  float part_m[2][4][32];
  float part_l[2][4][32];
  float part_a[2][4][32];
};

// Per-sequence metadata: in shared memory (folded mode) or in the workspace
// (written by the scheduler kernel). Plain loads: the pointers may be either.
struct Meta {
  const int32_t* cu;    // [B+1] validated token offsets
  const int32_t* s;     // [B]   start positions
  const int32_t* off;   // [B+1] first output row of each sequence
  const int32_t* tile;  // [B+1] first work tile of each sequence
};

__device__ __forceinline__ int upper_index_plain(const int32_t* a, int n, int v) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (a[mid] <= v) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 512;" ::: "memory"); }

__device__ __forceinline__ float4 ldcg4(const float* p) { return __ldcg(reinterpret_cast<const float4*>(p)); }

// Exclusive prefix sum over the CTA's threads (every thread calls it); *total
// gets the sum.
__device__ __forceinline__ int cta_exclusive_scan(int v, int* wsum, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int NW = kThreads / 32;
  int inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += n;
  }
  if (lane == 31) wsum[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    const int w = lane < NW ? wsum[lane] : 0;
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += n;
    }
    wsum[lane] = wi - w;
    if (lane == 31) *total = wi;
  }
  __syncthreads();
  const int r = wsum[warp] + inc - v;
  __syncthreads();
  return r;
}

// Folded mode: the scheduler's validation and metadata, in this CTA's shared
// memory (the same rules: cu rises from 0 to T, start_pos >= 0, positions fit in
// int32; a rejected call gets empty sequences, so every output row is 0;
// sequence b reserves min(L, L/ratio + 1) output rows; its work tiles cover
// positions from start_pos rounded down to the ratio to its end).
template <class Smem>
__device__ void build_meta(const Params& p, Smem& sm) {
  const int B = p.B;
  if (threadIdx.x == 0) sm.bad = 0;
  __syncthreads();
  for (int b = threadIdx.x; b <= B; b += kThreads) {
    const int c = __ldg(p.cu_in + b);
    bool ok = c >= 0 && c <= p.T;
    if (b == 0) ok = ok && c == 0;
    if (b == B) ok = ok && c == p.T;
    if (b < B) {
      const int c1 = __ldg(p.cu_in + b + 1);
      const int s = p.start_pos ? __ldg(p.start_pos + b) : 0;
      ok = ok && c1 >= c && s >= 0 && (int64_t)s + (int64_t)(c1 - c) <= (int64_t)INT32_MAX;
    }
    if (!ok) atomicOr(&sm.bad, 1);
  }
  __syncthreads();
  const bool rejected = sm.bad != 0;
  if (rejected && threadIdx.x == 0 && blockIdx.x == 0) atomicOr(p.err, kErrIndex);
  int carry = 0, tcarry = 0;
  for (int base = 0; base < B; base += kThreads) {
    const int b = base + threadIdx.x;
    int c = 0, s = 0, cap = 0, tiles = 0;
    if (b < B && !rejected) {
      c = __ldg(p.cu_in + b);
      const int L = __ldg(p.cu_in + b + 1) - c;
      s = p.start_pos ? __ldg(p.start_pos + b) : 0;
      cap = min(L, L / p.ratio + 1);
      if (L > 0) tiles = (s + L - (s / p.ratio) * p.ratio + NTOK - 1) / NTOK;
    }
    const int ex = cta_exclusive_scan(cap, sm.scan_w, &sm.scan_tot);
    const int cap_total = sm.scan_tot;
    __syncthreads();
    const int tex = cta_exclusive_scan(tiles, sm.scan_w, &sm.scan_tot);
    const int tile_total = sm.scan_tot;
    if (b < B) {
      sm.m_cu[b] = c;
      sm.m_s[b] = s;
      sm.m_off[b] = carry + ex;
      sm.m_tile[b] = tcarry + tex;
    }
    carry += cap_total;
    tcarry += tile_total;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    sm.m_cu[B] = rejected ? 0 : p.T;
    sm.m_off[B] = carry;
    sm.m_tile[B] = tcarry;
  }
}

// What one work item covers.
struct Item {
  int b;      // sequence
  int k;      // tile of the sequence
  int P0;     // first position of the tile
  int t0;     // x row of position P0 (may lie before the sequence, even < 0)
  int half;   // 0 / 1: which coff half of the state row
  int c0;     // first channel (within the half)
};

__device__ __forceinline__ Item decode_item(const Params& p, const Meta& md, int g, int n_cblk) {
  Item it;
  const int tile = g / n_cblk, cb = g % n_cblk;
  const int per_half = p.D / BM;
  it.half = cb / per_half;
  it.c0 = (cb % per_half) * BM;
  it.b = upper_index_plain(md.tile, p.B, tile);
  it.k = tile - md.tile[it.b];
  const int s = md.s[it.b];
  it.P0 = (s / p.ratio) * p.ratio + it.k * NTOK;
  it.t0 = md.cu[it.b] + (it.P0 - s);
  return it;
}

// Where the first 64 positions of a ratio-128 window leave their running
// softmax stats for the warp that ends the window (one slot per window of the
// tile, TMEM lane quarter and lane).
struct Parts {
  float* m;  // [2][4][32]
  float* l;
  float* a;
};

// The epilogue of one item for ratio R in {32, 64, 128} (a window spans 2, 4
// or 8 sub-chunks of 16 positions): the four sub-chunks of one 64-position
// quarter (qt) of the tile, with an online softmax per window; a ratio-128
// window spans two quarters, and the warp of its second quarter merges the
// first quarter's stats (after a barrier of all epilogue warps). The 16 ape
// values a sub-chunk adds to its scores are loaded one sub-chunk ahead (the
// first ones before the accumulator is ready), so their L2 latency overlaps the
// TMEM loads and the previous sub-chunk's math instead of stalling each step
// while the MMA waits for TMEM.
template <int R, int D, class Wait>
__device__ __forceinline__ bool pool_item_wide(const Params& p, const Meta& md, const Item& it, uint32_t taddr,
                                               int ch, int qt, int quad, const Parts& parts, Wait&& wait_acc) {
  static_assert(R == 32 || R == 64 || R == 128, "windows of 2, 4 or 8 sub-chunks");
  constexpr int C = D;  // coff = 1: the state / ape rows are D wide
  const int b = it.b;
  const int s = md.s[b];
  const int cu = md.cu[b];
  const int e = s + (md.cu[b + 1] - cu);
  const int w0 = s / R;
  const int w_end = e / R;
  const int off = md.off[b];
  const int thr = max(s, tail_threshold(e, R, 1));
  const int col = ch;  // coff = 1: one half
  float* ybase = p.ystat + ch;
  // the tile starts on a window boundary: position P0 + 16 u + j has ape row (16 u + j) mod R;
  // the rows of sub-chunk u start at ape + ((16 u) mod R) * C + col (constant offsets j * C)
  const float* ape_col = p.ape + col;
  float apn[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) apn[j] = __ldg(ape_col + ((qt * 64) % R + j) * C);
  if (!wait_acc()) return false;
  float m = -INFINITY, l = 0.f, acc = 0.f;

#pragma unroll 1
  for (int u = qt * 4; u < qt * 4 + 4; ++u) {
    const int q0 = it.P0 + u * 16;
    if (q0 >= e) break;  // the rest of the tile lies past the sequence
    uint32_t kr[16], sr[16];
    tmem_ld16(taddr + u * 16, kr);
    tmem_ld16(taddr + NTOK + u * 16, sr);
    float apc[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) apc[j] = apn[j];
    if (u + 1 < qt * 4 + 4) {
      const float* ap_next = ape_col + ((16 * (u + 1)) % R) * C;
#pragma unroll
      for (int j = 0; j < 16; ++j) apn[j] = __ldg(ap_next + j * C);
    }
    tmem_ld_wait16(kr, sr);
    float kv[16], z[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      kv[j] = __uint_as_float(kr[j]);
      z[j] = __uint_as_float(sr[j]) + apc[j];
    }
    if (q0 < s) {  // rows written by earlier calls (the first window of the sequence)
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int q = q0 + j;
        if (q < s) {
          const int rk = table_row(p, p.kv_tbl, b, q);
          const int rs = table_row(p, p.sc_tbl, b, q);
          kv[j] = rk >= 0 ? p.kv_state[((int64_t)rk * p.bs + q % p.bs) * p.C + col] : 0.f;
          z[j] = rs >= 0 ? p.score_state[((int64_t)rs * p.bs + q % p.bs) * p.C + col] : -INFINITY;
        }
      }
    }
    if (q0 + 15 >= thr) {  // tail rows: kv and score + ape into the paged state
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int q = q0 + j;
        if (q >= thr && q < e) {
          const int rk = table_row(p, p.kv_tbl, b, q);
          const int rs = table_row(p, p.sc_tbl, b, q);
          if (rk >= 0) p.kv_state[((int64_t)rk * p.bs + q % p.bs) * p.C + col] = kv[j];
          if (rs >= 0) p.score_state[((int64_t)rs * p.bs + q % p.bs) * p.C + col] = z[j];
        }
      }
    }
    const int w = q0 / R;  // the sub-chunk is one piece of window w
    if (w < w_end) {
      float mx[8];  // tree maximum (short dependency chains)
#pragma unroll
      for (int j = 0; j < 8; ++j) mx[j] = fmaxf(z[j], z[j + 8]);
#pragma unroll
      for (int j = 0; j < 4; ++j) mx[j] = fmaxf(mx[j], mx[j + 4]);
      const float mn = fmaxf(m, fmaxf(fmaxf(mx[0], mx[2]), fmaxf(mx[1], mx[3])));
      const float sc = __expf(m - mn);
      float l2[2] = {0.f, 0.f}, a2[2] = {0.f, 0.f};  // two independent partial sums
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float pz = __expf(z[j] - mn);
        l2[j & 1] += pz;
        a2[j & 1] = fmaf(pz, kv[j], a2[j & 1]);
      }
      l = fmaf(l, sc, l2[0] + l2[1]);
      acc = fmaf(acc, sc, a2[0] + a2[1]);
      m = mn;
      if (R < 128 && ((u + 1) * 16) % R == 0) {  // last sub-chunk of the window
        const int64_t n = off + (w - w0);
        ybase[n * p.D] = acc / l;
        m = -INFINITY;
        l = 0.f;
        acc = 0.f;
      }
    }
  }
  if constexpr (R == 128) {  // window qt / 2 of the tile: quarters 2 wi and 2 wi + 1
    const int wi = qt >> 1;
    const int slot = (wi * 4 + quad) * 32 + (threadIdx.x & 31);
    if ((qt & 1) == 0) {
      parts.m[slot] = m;
      parts.l[slot] = l;
      parts.a[slot] = acc;
    }
    epi_bar();
    const int w = (it.P0 + wi * 128) / R;
    if ((qt & 1) && w < w_end) {
      const float m1 = parts.m[slot], l1 = parts.l[slot], a1 = parts.a[slot];
      const float mn = fmaxf(m1, m);
      const float f1 = m1 == -INFINITY ? 0.f : __expf(m1 - mn);
      const float f2 = m == -INFINITY ? 0.f : __expf(m - mn);
      const float lt = fmaf(l1, f1, l * f2);
      const float at = fmaf(a1, f1, acc * f2);
      const int64_t n = off + (w - w0);
      ybase[n * p.D] = at / lt;
    }
    epi_bar();  // the slots are free for the next item
  }
  return true;
}

// The epilogue of one item for ratio R <= 16 (whole windows inside a sub-chunk
// of 16 positions): the four sub-chunks of one 64-position quarter (qt) of the tile.
// The R ape rows are loaded before the accumulator is ready. `wait_acc` waits
// for the accumulator (false: give up).
template <int R, class Wait>
__device__ __forceinline__ bool pool_item(const Params& p, const Meta& md, const Item& it, uint32_t taddr,
                                          int ch, int qt, int quad, const Parts& parts, Wait&& wait_acc) {
  if constexpr (R >= 32) {
    if (p.D == 128) return pool_item_wide<R, 128>(p, md, it, taddr, ch, qt, quad, parts, wait_acc);
    return pool_item_wide<R, 512>(p, md, it, taddr, ch, qt, quad, parts, wait_acc);
  } else {
  constexpr int COFF = (R == 4) ? 2 : 1;
  const int b = it.b;
  const int s = md.s[b];
  const int cu = md.cu[b];
  const int e = s + (md.cu[b + 1] - cu);
  const int w0 = s / R;        // first window this call completes
  const int w_end = e / R;     // windows below this one complete in this call
  const int off = md.off[b];   // output row of window w0
  const int thr = max(s, tail_threshold(e, R, COFF));
  const int col = it.half * p.D + ch;  // column in the coff*D wide state / ape rows
  float* ybase = p.ystat + (int64_t)it.half * p.D + ch;
  float* lbase = p.ylse + (int64_t)it.half * p.D + ch;

  float ap[R];
#pragma unroll
  for (int j = 0; j < R; ++j) ap[j] = __ldg(p.ape + (int64_t)j * p.C + col);
  if (!wait_acc()) return false;

#pragma unroll 1
  for (int c = qt * 4; c < qt * 4 + 4; ++c) {
    const int q0 = it.P0 + c * 16;
    if (q0 >= e) break;  // the rest of the tile lies past the sequence
    uint32_t kr[16], sr[16];
    tmem_ld16(taddr + c * 16, kr);
    tmem_ld16(taddr + NTOK + c * 16, sr);
    tmem_ld_wait16(kr, sr);
    float kv[16], z[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      kv[j] = __uint_as_float(kr[j]);
      z[j] = __uint_as_float(sr[j]) + ap[j % R];
    }
    if (q0 < s) {  // rows written by earlier calls (the first window of the sequence)
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int q = q0 + j;
        if (q < s) {
          const int rk = table_row(p, p.kv_tbl, b, q);
          const int rs = table_row(p, p.sc_tbl, b, q);
          kv[j] = rk >= 0 ? p.kv_state[((int64_t)rk * p.bs + q % p.bs) * p.C + col] : 0.f;
          z[j] = rs >= 0 ? p.score_state[((int64_t)rs * p.bs + q % p.bs) * p.C + col] : -INFINITY;
        }
      }
    }
    if (q0 + 15 >= thr) {  // tail rows: kv and score + ape into the paged state
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int q = q0 + j;
        if (q >= thr && q < e) {
          const int rk = table_row(p, p.kv_tbl, b, q);
          const int rs = table_row(p, p.sc_tbl, b, q);
          if (rk >= 0) p.kv_state[((int64_t)rk * p.bs + q % p.bs) * p.C + col] = kv[j];
          if (rs >= 0) p.score_state[((int64_t)rs * p.bs + q % p.bs) * p.C + col] = z[j];
        }
      }
    }
    {
#pragma unroll
      for (int k = 0; k < 16 / R; ++k) {  // whole windows inside the sub-chunk
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
  return true;
  }
}

// Folded mode, one warp: output row n = window w of sequence b (first: w is the
// first window this call completes for b). NG = D / 128; lane l holds channels
// 128 i + 4 l .. +3 of group i. coff = 2 merges half 0 of window w - 1 (the
// previous row, or pooled here from the paged state when that window lies
// wholly before start_pos, or nothing for window 0) with half 1 of window w
// through their log-sum-exps, which is the 2 ratio-row softmax exactly; then
// RMSNorm (eps 1e-6) times norm_weight, interleaved RoPE on the last 64
// channels (pair (2j, 2j+1) takes table columns j and 32 + j) and the bf16
// store ("CANN PyPTO 算子实战", 压缩窗口与状态更新). Every load of the row is
// issued before the first use, so a row costs about one memory round trip.
template <int NG, int COFF>
__device__ __forceinline__ void finish_window(const Params& p, int b, int w, int64_t n, bool first, int lane) {
  constexpr int D = NG * 128;
  constexpr int kRope = 64;  // rope_head_dim (the only value the library accepts)
  const bool rope_lane = lane >= 16;  // group NG-1: channels D-64 .. D-1
  const int j = 2 * (lane - 16);      // its pairs use table columns j, j+1 and 32+j, 33+j
  __nv_bfloat162 c_lo, c_hi, s_lo, s_hi;
  if (rope_lane) {
    const __nv_bfloat16* cs = p.cos + n * kRope;
    const __nv_bfloat16* sn = p.sin + n * kRope;
    c_lo = *reinterpret_cast<const __nv_bfloat162*>(cs + j);
    c_hi = *reinterpret_cast<const __nv_bfloat162*>(cs + 32 + j);
    s_lo = *reinterpret_cast<const __nv_bfloat162*>(sn + j);
    s_hi = *reinterpret_cast<const __nv_bfloat162*>(sn + 32 + j);
  }
  uint2 wraw[NG];  // norm_weight of the lane's channels
#pragma unroll
  for (int i = 0; i < NG; ++i) wraw[i] = *reinterpret_cast<const uint2*>(p.norm_w + i * 128 + lane * 4);
  // per group of 128 channels: the pooled halves (coff = 2: and the previous
  // window's half 0), merged right away so that only one group's loads are
  // live at a time
  const bool prev_row = COFF == 2 && !first;
  float y[NG][4];
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < NG; ++i) {
    const int c = i * 128 + lane * 4;
    float4 yb, lb, ya, la;
    if (COFF == 1) {
      yb = ldcg4(p.ystat + n * D + c);
    } else {
      yb = ldcg4(p.ystat + (n * 2 + 1) * D + c);
      lb = ldcg4(p.ylse + (n * 2 + 1) * D + c);
      if (prev_row) {
        ya = ldcg4(p.ystat + (n - 1) * 2 * D + c);
        la = ldcg4(p.ylse + (n - 1) * 2 * D + c);
      } else {
        ya = make_float4(0.f, 0.f, 0.f, 0.f);
        la = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
      }
      if (first && w > 0) {  // window w - 1 from the paged state (rare: once per sequence)
        float m[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY}, l[4] = {0.f, 0.f, 0.f, 0.f},
              a[4] = {0.f, 0.f, 0.f, 0.f};
        for (int jj = 0; jj < p.ratio; ++jj) {
          const int q = (w - 1) * p.ratio + jj;
          const int rk = table_row(p, p.kv_tbl, b, q);
          const int rs = table_row(p, p.sc_tbl, b, q);
          if (rk < 0 || rs < 0) continue;
          const float4 kv = __ldcg(reinterpret_cast<const float4*>(
              p.kv_state + ((int64_t)rk * p.bs + q % p.bs) * p.C + c));
          const float4 sc = __ldcg(reinterpret_cast<const float4*>(
              p.score_state + ((int64_t)rs * p.bs + q % p.bs) * p.C + c));
          const float kk[4] = {kv.x, kv.y, kv.z, kv.w}, zz[4] = {sc.x, sc.y, sc.z, sc.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float mn = fmaxf(m[u], zz[u]);
            const float f = __expf(m[u] - mn), pz = __expf(zz[u] - mn);
            l[u] = l[u] * f + pz;
            a[u] = a[u] * f + pz * kk[u];
            m[u] = mn;
          }
        }
        float yv[4] = {0.f, 0.f, 0.f, 0.f}, lv[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (l[u] > 0.f) {
            yv[u] = a[u] / l[u];
            lv[u] = m[u] + __logf(l[u]);
          }
        ya = make_float4(yv[0], yv[1], yv[2], yv[3]);
        la = make_float4(lv[0], lv[1], lv[2], lv[3]);
      }
    }
    const float ybv[4] = {yb.x, yb.y, yb.z, yb.w};
    if (COFF == 1) {
#pragma unroll
      for (int u = 0; u < 4; ++u) y[i][u] = ybv[u];
    } else {
      const float lbv[4] = {lb.x, lb.y, lb.z, lb.w};
      const float yav[4] = {ya.x, ya.y, ya.z, ya.w};
      const float lav[4] = {la.x, la.y, la.z, la.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float M = fmaxf(lav[u], lbv[u]);
        const float wa = __expf(lav[u] - M), wb = __expf(lbv[u] - M);
        y[i][u] = (yav[u] * wa + ybv[u] * wb) / (wa + wb);
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) ss = fmaf(y[i][u], y[i][u], ss);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float inv = rsqrtf(ss / (float)D + kRmsEps);
#pragma unroll
  for (int i = 0; i < NG; ++i) {
    const int c = i * 128 + lane * 4;
    const __nv_bfloat162 w01 = *reinterpret_cast<const __nv_bfloat162*>(&wraw[i].x);
    const __nv_bfloat162 w23 = *reinterpret_cast<const __nv_bfloat162*>(&wraw[i].y);
    const float nw[4] = {__low2float(w01), __high2float(w01), __low2float(w23), __high2float(w23)};
    float z[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) z[u] = y[i][u] * inv * nw[u];
    if (i == NG - 1 && rope_lane) {
      const float ce[2] = {__low2float(c_lo), __high2float(c_lo)}, co[2] = {__low2float(c_hi), __high2float(c_hi)};
      const float se[2] = {__low2float(s_lo), __high2float(s_lo)}, so[2] = {__low2float(s_hi), __high2float(s_hi)};
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const float ev = z[2 * u], od = z[2 * u + 1];
        z[2 * u] = ev * ce[u] - od * se[u];
        z[2 * u + 1] = od * co[u] + ev * so[u];
      }
    }
    __nv_bfloat162 o01 = __floats2bfloat162_rn(z[0], z[1]);
    __nv_bfloat162 o23 = __floats2bfloat162_rn(z[2], z[3]);
    uint2 v;
    v.x = *reinterpret_cast<uint32_t*>(&o01);
    v.y = *reinterpret_cast<uint32_t*>(&o23);
    *reinterpret_cast<uint2*>(p.out + n * D + c) = v;
  }
}

// Folded mode: the output rows of work tile t (its windows), one per warp of
// the sixteen epilogue warps at a time.
template <int NG, int COFF>
__device__ void finish_tile_t(const Params& p, const Meta& md, int t, int ew, int lane) {
  const int b = upper_index_plain(md.tile, p.B, t);
  const int k = t - md.tile[b];
  const int s = md.s[b];
  const int e = s + (md.cu[b + 1] - md.cu[b]);
  const int R = p.ratio;
  const int P0 = (s / R) * R + k * NTOK;
  const int w0 = s / R;
  const int wa = P0 / R, wb = min((P0 + NTOK) / R, e / R);
  const int64_t off = md.off[b];
  for (int w = wa + ew; w < wb; w += kEpiThreads / 32)
    finish_window<NG, COFF>(p, b, w, off + (w - w0), w == w0, lane);
}

__device__ void finish_tile(const Params& p, const Meta& md, int t, int ew, int lane) {
  if (p.D == 128) {
    if (p.coff == 2) finish_tile_t<1, 2>(p, md, t, ew, lane);
    else finish_tile_t<1, 1>(p, md, t, ew, lane);
  } else {
    if (p.coff == 2) finish_tile_t<4, 2>(p, md, t, ew, lane);
    else finish_tile_t<4, 1>(p, md, t, ew, lane);
  }
}

// Folded mode: zero the output rows that hold no window (each sequence's
// reserved rows past its completed windows, and the rows after the last
// sequence's), sequences spread over the CTAs; sixteen warps, 16 bytes a lane.
__device__ void zero_rows(const Params& p, const Meta& md, int ew, int lane) {
  const int D = p.D;
  const int per_row = D * 2 / 16;  // uint4 per row
  auto zero = [&](int64_t r0, int64_t r1) {
    const int64_t total = (r1 - r0) * per_row;
    uint4* base = reinterpret_cast<uint4*>(p.out + r0 * D);
    for (int64_t i = ew * 32 + lane; i < total; i += kEpiThreads) base[i] = make_uint4(0u, 0u, 0u, 0u);
  };
  for (int b = blockIdx.x; b < p.B; b += gridDim.x) {
    const int s = md.s[b];
    const int e = s + (md.cu[b + 1] - md.cu[b]);
    const int nw = e / p.ratio - s / p.ratio;
    zero(md.off[b] + nw, md.off[b + 1]);
  }
  if (blockIdx.x == 0) zero(md.off[p.B], p.n_out);
}

template <bool FOLD, bool PAIR>
__global__ void __launch_bounds__(kThreads, 1)
    fused_tc_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_wkv,
                    const __grid_constant__ CUtensorMap map_wg, Params p) {
  using C = Cfg<PAIR>;
  using Smem = SmemT<PAIR>;
  constexpr int STAGES = C::ST;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  Smem& sm = smem_align1024<Smem>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_cblk = p.coff * p.D / BM;
  const int k_blocks = p.H / BK;
  // CTA pairs: rank 0 issues the pair's MMAs; a work unit is two items (channel
  // blocks 2c and 2c + 1 of one tile), the CTA of rank r pooling item 2u + r
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const int unit0 = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int ustep = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    mbar_init(&sm.acc_full, 1);
    mbar_init(&sm.acc_empty, (PAIR ? 2 : 1) * kEpiThreads / 32);  // epilogue warps (of both CTAs)
    sm.abort = 0;
    fence_barrier_init();
    prefetch_tmap(&map_x);
    prefetch_tmap(&map_wkv);
    prefetch_tmap(&map_wg);
  }
  if (warp == 1) {
    if constexpr (PAIR) tmem_alloc_pair(&sm.tmem_base, 512);
    else tmem_alloc(&sm.tmem_base, 512);
  }
  if constexpr (FOLD) build_meta(p, sm);  // reads only this call's inputs
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) cluster_sync_all();  // both CTAs' barriers exist before either signals the other's
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort = &sm.abort;
  const uint32_t full0 = PAIR ? mapa_shared(smem_u32(&sm.full[0]), 0) : 0u;  // the even CTA's barriers
  const uint32_t acc_empty0 = PAIR ? mapa_shared(smem_u32(&sm.acc_empty), 0) : 0u;
  pdl_trigger();
  Meta md;
  if constexpr (FOLD) {
    md = Meta{sm.m_cu, sm.m_s, sm.m_off, sm.m_tile};
  } else {
    pdl_wait();  // the metadata comes from the scheduler kernel
    md = Meta{p.m_cu, p.m_s, p.m_off, p.m_tile};
  }
  const int total = md.tile[p.B] * n_cblk;
  const int n_units = PAIR ? total / 2 : total;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      Armed armed;
      for (int u = unit0; u < n_units && !*abort; u += ustep) {
        const int g = PAIR ? 2 * u + (int)rank : u;
        const Item it = decode_item(p, md, g, n_cblk);
        const int wrow = it.half * p.D + it.c0;
        const int xrow = it.t0 + (int)rank * C::NB;  // pairs: this CTA's half of the positions
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (!mbar_wait(&sm.empty[stage], phase ^ 1u, abort)) break;
          if constexpr (PAIR) {
            if (rank == 0) {
              mbar_arrive_expect_tx(&sm.full[stage], 2 * C::kStageBytes);
              armed.note(stage, phase);
            }
            const uint32_t fb = full0 + 8u * stage;
            tma_load_2d_pair(sm.a_kv[stage], &map_wkv, fb, kb * BK, wrow);
            tma_load_2d_pair(sm.a_g[stage], &map_wg, fb, kb * BK, wrow);
            tma_load_2d_pair(sm.b[stage], &map_x, fb, kb * BK, xrow);
          } else {
            mbar_arrive_expect_tx(&sm.full[stage], C::kStageBytes);
            armed.note(stage, phase);
            tma_load_2d(sm.a_kv[stage], &map_wkv, &sm.full[stage], kb * BK, wrow);
            tma_load_2d(sm.a_g[stage], &map_wg, &sm.full[stage], kb * BK, wrow);
            tma_load_2d(sm.b[stage], &map_x, &sm.full[stage], kb * BK, xrow);
          }
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      drain_armed(sm.full, STAGES, armed);  // no copy still landing when the CTA leaves
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t acc_phase = 0;
      for (int u = unit0; u < n_units && !*abort; u += ustep) {
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
            if constexpr (PAIR) {
              mma_bf16_pair(tmem, sw128_kmajor_desc(akv + k * 32), bd, C::kIdesc, accum);
              mma_bf16_pair(tmem + NTOK, sw128_kmajor_desc(ag + k * 32), bd, C::kIdesc, accum);
            } else {
              mma_bf16(tmem, sw128_kmajor_desc(akv + k * 32), bd, C::kIdesc, accum);
              mma_bf16(tmem + NTOK, sw128_kmajor_desc(ag + k * 32), bd, C::kIdesc, accum);
            }
          }
          if constexpr (PAIR) mma_commit_pair(&sm.empty[stage], 0x3);  // frees the stage in both CTAs
          else mma_commit(&sm.empty[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        if constexpr (PAIR) mma_commit_pair(&sm.acc_full, 0x3);
        else mma_commit(&sm.acc_full);
        acc_phase ^= 1u;
      }
    }
  } else {
    const int ew = warp - 2;                 // 0..15
    const int e_tid = threadIdx.x - 64;      // 0..511
    const int quad = warp & 3;               // TMEM lanes this warp may access
    const int qt = ew >> 2;                  // 64-position quarter of the tile
    const Parts parts{&sm.part_m[0][0][0], &sm.part_l[0][0][0], &sm.part_a[0][0][0]};
    const int row = quad * 32 + lane;
    const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16);
    if constexpr (FOLD) {
      pdl_wait();  // the epilogue writes the state, the pooled halves and out
      zero_rows(p, md, ew, lane);
    }
    uint32_t acc_phase = 0;
    for (int u = unit0; u < n_units; u += ustep) {
      const int g = PAIR ? 2 * u + (int)rank : u;
      const Item it = decode_item(p, md, g, n_cblk);
      auto wait_acc = [&]() {
        const bool ok = mbar_wait(&sm.acc_full, acc_phase, abort);
        if (!bar_and(1, kEpiThreads, ok)) return false;  // all epilogue warps leave together
        tc_fence_after();
        return true;
      };
      const int ch = it.c0 + row;
      bool ok;
      switch (p.ratio) {
        case 1: ok = pool_item<1>(p, md, it, taddr, ch, qt, quad, parts, wait_acc); break;
        case 2: ok = pool_item<2>(p, md, it, taddr, ch, qt, quad, parts, wait_acc); break;
        case 4: ok = pool_item<4>(p, md, it, taddr, ch, qt, quad, parts, wait_acc); break;
        case 8: ok = pool_item<8>(p, md, it, taddr, ch, qt, quad, parts, wait_acc); break;
        case 16: ok = pool_item<16>(p, md, it, taddr, ch, qt, quad, parts, wait_acc); break;
        case 32: ok = pool_item<32>(p, md, it, taddr, ch, qt, quad, parts, wait_acc); break;
        case 64: ok = pool_item<64>(p, md, it, taddr, ch, qt, quad, parts, wait_acc); break;
        default: ok = pool_item<128>(p, md, it, taddr, ch, qt, quad, parts, wait_acc); break;
      }
      if (!ok) break;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if constexpr (PAIR) mbar_arrive_cluster(acc_empty0);
        else mbar_arrive(&sm.acc_empty);
      }
      acc_phase ^= 1u;
      if constexpr (FOLD) {
        // arrive on the tile's counter (coff = 2: also on the next tile's); the
        // barrier orders every epilogue thread's stores before thread 0's
        // release fence and atomic, and the finishing CTA's acquire fence
        // before its loads (the pattern of a cooperative grid barrier)
        epi_bar();
        if (e_tid == 0) {
          const int tile = g / n_cblk;
          const int ntiles_b = md.tile[it.b + 1] - md.tile[it.b];
          int nf = 0;
          __threadfence();
          const unsigned tgt = (unsigned)n_cblk * ((p.coff == 2 && it.k > 0) ? 2u : 1u);
          if (atomicAdd(p.tile_cnt + tile, 1u) + 1u == tgt) {
            atomicExch(p.tile_cnt + tile, 0u);
            sm.fin[nf++] = tile;
          }
          if (p.coff == 2 && it.k + 1 < ntiles_b) {
            if (atomicAdd(p.tile_cnt + tile + 1, 1u) + 1u == 2u * (unsigned)n_cblk) {
              atomicExch(p.tile_cnt + tile + 1, 0u);
              sm.fin[nf++] = tile + 1;
            }
          }
          if (nf) __threadfence();
          sm.nfin = nf;
        }
        epi_bar();
        const int nf = sm.nfin;
        for (int i = 0; i < nf; ++i) finish_tile(p, md, sm.fin[i], ew, lane);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) cluster_sync_all();  // neither CTA leaves while the other may still signal it
  if (warp == 1) {
    tc_fence_after();
    if constexpr (PAIR) tmem_dealloc_pair(tmem, 512);
    else tmem_dealloc(tmem, 512);
  }
  if (threadIdx.x == 0 && sm.abort) atomicOr(p.err, kErrTimeout);
}

}  // namespace

bool fused_supported(const Params& p) {
  return p.H % BK == 0 && p.D % BM == 0 && NTOK % p.ratio == 0 && encode_fn() != nullptr;
}

// Upper bound of the work tiles of a call (the exact count is on the device):
// every sequence adds at most one partial tile at each end.
int64_t fused_max_tiles(const Params& p) { return ((int64_t)p.T + NTOK - 1) / NTOK + 2LL * p.B; }

bool fused_fold_supported(const Params& p) {
  return !p.rotate && p.B <= kMetaSeqs && fused_max_tiles(p) + 1 <= kFusedTileCounters;
}

namespace {

// Per device: co-resident 2-CTA clusters of the pair kernels (0: not measured
// yet, -1: the device refused the cluster form).
int g_fused_pair_slots[64] = {0};

template <bool FOLD, bool PAIR>
cudaError_t launch_form(const Params& p, cudaStream_t s, int units) {
  CUtensorMap mx, mkv, mg;
  if (!make_tile_map(&mx, p.x, p.T, p.H, Cfg<PAIR>::NB) || !make_tile_map(&mkv, p.wkv, p.C, p.H, BM) ||
      !make_tile_map(&mg, p.wgate, p.C, p.H, BM))
    return cudaErrorInvalidValue;
  const size_t smem = sizeof(SmemT<PAIR>) + 1024;
  static int configured[64] = {0};
  const cudaError_t e = smem_attr_once(fused_tc_kernel<FOLD, PAIR>, smem, configured);
  if (e != cudaSuccess) return e;
  const int grid = PAIR ? 2 * units : units;
  return launch_chained(fused_tc_kernel<FOLD, PAIR>, dim3(grid), dim3(kThreads), smem, s, PAIR ? 2 : 1, mx, mkv, mg,
                        p);
}

// How many 2-CTA clusters of the pair kernel fit at once (-1: none).
template <bool FOLD>
int pair_slots(int dev) {
  int& slots = g_fused_pair_slots[dev];
  if (slots != 0) return slots;
  static int configured[64] = {0};
  const size_t smem = sizeof(SmemT<true>) + 1024;
  if (smem_attr_once(fused_tc_kernel<FOLD, true>, smem, configured) != cudaSuccess) {
    cudaGetLastError();
    return slots = -1;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = 2;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, fused_tc_kernel<FOLD, true>, &cfg) != cudaSuccess || n < 1) {
    cudaGetLastError();
    return slots = -1;
  }
  return slots = n;
}

}  // namespace

// CTA pairs (cta_group::2) when the channel blocks pair up (coff * D / 128
// even) and the device co-schedules the clusters, unless the call asks for
// single CTAs; the one-kernel form when p.tile_cnt is set.
cudaError_t launch_fused(const Params& p, cudaStream_t s, int sm_count) {
  const bool fold = p.tile_cnt != nullptr;
  const int n_cblk = p.coff * p.D / BM;
  const int64_t items = fused_max_tiles(p) * n_cblk;
  int dev = 0;
  cudaGetDevice(&dev);
  if (n_cblk % 2 == 0 && !p.single_cta && dev < 64) {
    const int slots = fold ? pair_slots<true>(dev) : pair_slots<false>(dev);
    if (slots > 0) {
      const int64_t units = items / 2;
      const int u = units < slots ? (int)units : slots;
      const cudaError_t e = fold ? launch_form<true, true>(p, s, u) : launch_form<false, true>(p, s, u);
      if (e == cudaSuccess) return e;
      // the launch was refused before anything ran (a cluster form this device
      // will not schedule): single CTAs from now on
      cudaGetLastError();
      g_fused_pair_slots[dev] = -1;
    }
  }
  const int grid = items < sm_count ? (int)items : sm_count;
  return fold ? launch_form<true, false>(p, s, grid) : launch_form<false, false>(p, s, grid);
}

}  // namespace cmp
