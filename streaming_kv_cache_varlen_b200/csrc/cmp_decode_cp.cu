// Decode by channel groups, in one cooperative kernel of 4-CTA clusters
// (T <= 64 tokens, B <= 256 sequences).
//
// The per-channel softmax pooling ("compressor torch_extension API", 计算公式
// 3-5) never mixes channels, so a cluster that holds the complete projections
// of some channels can pool them on its own. Cluster g owns channels
// 16g .. 16g+15 of the D; its four CTAs split the hidden dimension, and after
// an on-chip reduction CTA q holds channels 16g+4q .. 16g+4q+3.
//
// Projection. Per 64-column K block one TMA copy brings the wkv and wgate rows
// of the cluster's channels (both halves for ratio 4, coff 2: 64 rows; else 32;
// one 5-D tensor map spans both matrices) and one brings the x columns; an
// M = 64 tcgen05.mma accumulates the rows x tokens product in TMEM. An M = 64
// accumulator puts rows 16i .. 16i+15 in TMEM lanes 32i .. 32i+15, so each of
// warps 0-3 holds one 16-row block (one half of one matrix). A decode step's
// weight stream is bound by the number of MMA instructions (each costs about
// the same at these sizes), so every MMA carries all the rows it can.
//
// Reduction. Each read-out warp pushes every channel's partial sums to the CTA
// that owns the channel (st.async into its shared memory, completing on its
// mbarrier); each owner adds the four partials in rank order.
//
// Pooling and RMSNorm. Warps 0-3 pool this CTA's 4 channels of every window
// the call completes (the windows' state rows were pre-reduced per channel
// while the weights streamed, so only this call's rows remain). Warp 0 then
// stores the windows' sums of squares over its channels to global memory and
// arrives (release) at a counter, waits (acquire, bounded) until all CTAs have
// arrived and reads every CTA's sums at once, while warps 1-3 write the state
// tails. Warps 0-3 add the sums in a fixed order for the RMSNorm ("CANN PyPTO
// 算子实战", 压缩窗口与状态更新: rms_norm over the D channels), scale their
// channels, apply norm_weight and the interleaved RoPE (a pair never straddles
// two CTAs) and store bf16. With the Hadamard rotation the exchange also
// carries each CTA's u = RoPE(y * norm_weight) for its channels; the RMSNorm
// scale commutes with the product, so every CTA forms its own output columns
// as scale * (u @ hadamard[:, its channels]) from all D values of u ("CANN
// PyPTO 算子实战", kernel 派发逻辑: out @ hadamard).
//
// Warps 4-5 compute the call's metadata (what the varlen scheduler kernel does
// on the other paths) and prefetch what the later steps read: the state rows
// of every window the call completes, ape, norm_weight and the RoPE tables, for
// this CTA's channels. Warp 6 issues the TMA copies, warp 7 the MMAs. Waiting
// warps let one lane poll, so that they do not crowd the shared-memory pipe the
// other warps and the tensor core use. The weights are read once, x once per
// cluster. This call writes state slots of positions >= start_pos only and
// reads those below, so the prefetch and the tail stores never touch the same
// slot.
#include <cstddef>
#include <mutex>

#include "cmp_internal.cuh"
#include "cmp_sm100.cuh"

namespace cmp {
namespace {

using namespace sm100;

// Phase stamps (a measurement build only, compiled with -DCMP_PHASE_STAMPS):
// CTA i writes the global timer at phase k to slot i * kStampSlots + k of a
// device array that cmp_debug_phase_stamps copies out. The normal build has no
// stamps and no array.
#ifdef CMP_PHASE_STAMPS
constexpr int kStampSlots = 32;
constexpr int kStampCtas = 512;
__device__ unsigned long long g_cp_stamps[kStampCtas * kStampSlots];
#define CP_STAMP(cond, k)                                                           \
  do {                                                                              \
    if ((cond) && blockIdx.x < kStampCtas) g_cp_stamps[blockIdx.x * kStampSlots + (k)] = globaltimer(); \
  } while (0)
#else
#define CP_STAMP(cond, k) \
  do {                    \
  } while (0)
#endif

constexpr int KQ = 4;             // CTAs per cluster: they split the hidden dimension
constexpr int GCH = 16;           // channels per cluster
constexpr int OWN = GCH / KQ;     // channels per CTA after the reduction
constexpr int BK = 64;
constexpr int KPS = 2;            // 64-column K blocks per pipeline stage
constexpr int kTileA = 4 * GCH * 128;  // one K block of A: 2 matrices x 2 halves x 16 rows x 128 B
constexpr int kThreads = 256;     // warps 0-3: TMEM read-out (then warp 0: pooling, exchange, stores;
                                  // warps 1-3: state tails, rows without a window); warps 4-5:
                                  // metadata; warp 6 lane 0: TMA; warp 7 lane 0: MMA (warp 7 owns the
                                  // TMEM)
constexpr int kMetaBase = 128;    // first metadata thread
constexpr int kMaxSeqs = 256;
constexpr int kMaxOut = 64;       // n_out <= T <= 64
constexpr int kHistRows = 256;    // prefetched state rows (this CTA's 4 kv + 4 score channels)
constexpr int kMaxWinRows = 128;  // coff * ratio
constexpr int kMaxClusters = 32;  // D / GCH

template <int MAXT>
struct Cfg {
  static constexpr int stages = 4;
};

struct TokInfo {
  int32_t b;        // sequence, or -1
  int32_t pos;      // absolute position
  int64_t kv_off;   // kv_state element offset of its row if it is a tail row, else -1
  int64_t sc_off;   // score_state element offset, else -1
};

struct Win {        // the window of output row n, if the call completes one there
  int32_t w;        // window index, or -1 (the row is stored as zeros)
  int32_t b;        // sequence
  int32_t s;        // its start position
  int32_t cu;       // its first token
  int32_t hrows;    // leading window rows that come from the state (positions < s)
  int32_t hist;     // first prefetched row in hist, or -1 (read from global)
};

template <int MAXT>
struct Smem {
  static constexpr int S = Cfg<MAXT>::stages;
  // stage s: KPS A tiles (coff x 2 x 16 rows each) and KPS x tiles (NT rows
  // each), packed as the TMA boxes land them. An M = 64 MMA reads 64 rows from
  // its A tile on: for coff 1 (32 rows per tile) the last one reads 4 KB past
  // the A ring, into x
  alignas(1024) unsigned char a[S][KPS * kTileA];
  alignas(1024) __nv_bfloat16 x[S][KPS * MAXT * BK];
  alignas(16) float recv[2][KQ][2][OWN][MAXT];  // [half][source rank][kv, score][channel][token]
  alignas(16) float hist[kHistRows][2 * OWN];    // state rows: kv c0..c3, score c0..c3
  alignas(16) float ape[kMaxWinRows][OWN];       // ape of window row j (half * ratio + residue)
  alignas(16) float rope[kMaxOut][8];            // per pair: cos even, cos odd, sin even, sin odd
  alignas(16) float ybuf[kMaxOut][OWN];
  float ss_own[kMaxOut];                         // this CTA's sums of squares per window (list order)
  float ss_tot[kMaxOut];                         // every CTA's, added
  alignas(16) float4 hst[kMaxOut][OWN];          // per window and channel: the state rows' running
                                                 // max, exp-sum and weighted sum
  float norm[OWN];
  alignas(16) float hcolT[OWN][520];  // rotation: this CTA's columns of the hadamard matrix (column-major;
                                      // rows padded by 8 floats onto different banks)
  TokInfo tok[MAXT];
  Win win[kMaxOut];
  int32_t cu[kMaxSeqs + 1];
  int32_t sp[kMaxSeqs];
  int32_t off[kMaxSeqs + 1];
  int32_t hstart[kMaxOut + 1];
  int32_t wlist[kMaxOut];   // the output rows that have a window, in row order
  int32_t n_win;
  uint64_t full[S];
  uint64_t empty[S];
  uint64_t acc_full;        // the accumulator is complete
  uint64_t recv_full;       // the partial blocks of every source rank have landed in recv
  uint32_t tmem_base;
  uint32_t target;          // the arrival count at which this launch's sums are all stored
  int abort;
  int rejected;
  int xch_ok;               // the clusters' sums arrived
};

static_assert(offsetof(Smem<32>, x) % 1024 == 0 && offsetof(Smem<64>, x) % 1024 == 0,
              "TMA swizzled tiles must be 1024-byte aligned");
static_assert(offsetof(Smem<32>, x) == sizeof(Smem<32>::a) && offsetof(Smem<64>, x) == sizeof(Smem<64>::a) &&
                  sizeof(Smem<32>::x) >= 32 * 128,
              "an MMA's 64-row window past the last A tile stays inside x");
static_assert(offsetof(Smem<32>, recv) % 16 == 0 && offsetof(Smem<64>, recv) % 16 == 0 &&
                  offsetof(Smem<32>, hist) % 16 == 0 && offsetof(Smem<64>, hist) % 16 == 0 &&
                  offsetof(Smem<32>, ape) % 16 == 0 && offsetof(Smem<64>, ape) % 16 == 0 &&
                  offsetof(Smem<32>, ybuf) % 16 == 0 && offsetof(Smem<64>, ybuf) % 16 == 0 &&
                  offsetof(Smem<32>, hst) % 16 == 0 && offsetof(Smem<64>, hst) % 16 == 0,
              "float4 shared-memory rows must be 16-byte aligned");
static_assert(sizeof(Smem<32>) + 1024 <= 232448 && sizeof(Smem<64>) + 1024 <= 232448,
              "shared memory per CTA");

// The CTAs' arrivals: a 32-bit counter in the workspace that starts zeroed and
// only grows. Every launch adds exactly kPerLaunch to it (each of its n CTAs
// adds kPerLaunch / n, on every path), so a CTA that reads it at its start,
// before all CTAs of its launch have arrived (which needs this CTA's own
// arrival), sees a value whose multiple of kPerLaunch is the launch's base: the
// launch's sums are all stored once the counter reaches base + kPerLaunch.
// (Measured alternative: every CTA polling all CTAs' epoch-tagged 64-bit words
// instead swamped L2 with polls and took about 10 us.)
constexpr int kMaxCtas = kMaxClusters * KQ;
constexpr uint32_t kPerLaunch = kMaxCtas;

__device__ __forceinline__ uint32_t arrivals_now(const unsigned* counter) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(counter) : "memory");
  return v;
}

__device__ __forceinline__ void arrive_release(unsigned* counter, uint32_t n) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(counter), "r"(n) : "memory");
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}

__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// The shared::cluster address of `local` in cluster CTA `peer`.
__device__ __forceinline__ uint32_t peer_addr(const void* local, uint32_t peer) {
  uint32_t ra;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(smem_u32(local)), "r"(peer));
  return ra;
}

// 16 bytes into a peer's shared memory (addresses from peer_addr), completing
// on the peer's mbarrier.
__device__ __forceinline__ void st_async4(uint32_t dst, uint32_t a, uint32_t b, uint32_t c, uint32_t d,
                                          uint32_t mbar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(
                   dst),
               "r"(a), "r"(b), "r"(c), "r"(d), "r"(mbar)
               : "memory");
}

// TMA copy of a 5-D box into shared memory, completing on an mbarrier.
__device__ __forceinline__ void tma_load_5d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1,
                                            int c2, int c3, int c4) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, "
      "%6, %7}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4)
      : "memory");
}

// Interleaved RoPE on 4 consecutive channels (pairs (2j, 2j+1) of the last
// rope channels; t: per pair cos even, cos odd, sin even, sin odd).
__device__ __forceinline__ void rope4(float (&z)[4], const float* t) {
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const float ev = z[2 * u], od = z[2 * u + 1];
    z[2 * u] = ev * t[4 * u + 0] - od * t[4 * u + 2];
    z[2 * u + 1] = od * t[4 * u + 1] + ev * t[4 * u + 3];
  }
}

__device__ __forceinline__ float4 add4(float4 a, float4 b) {
  return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
}

struct CpArgs {
  unsigned* counter;  // the CTAs' arrivals (zeroed at creation)
  float* sums;        // [window list entry][CTA]: each CTA's sums of squares
  float* u;           // rotation: [window list entry][channel]: RoPE(y * norm_weight) of every channel
  int kv_first;       // the 5-D weight map holds wkv before wgate (else the other way round)
  uint32_t target_extra;  // added to the count the CTAs wait for: kPerLaunch makes it unreachable
                          // (timeout test)
};

// Window row j of window w: its absolute position (rows are in rising order).
__device__ __forceinline__ int window_pos(int w, int j, int r, int coff) {
  return coff == 1 ? w * r + j : (j < r ? (w - 1) * r + j : w * r + (j - r));
}

// Block-table entry of position pos of sequence b, or -1 (and the error bit)
// when the block index or the entry is out of range. The load is issued
// unconditionally (clamped index) so that several of these overlap.
__device__ __forceinline__ int table_entry(const Params& p, const int32_t* __restrict__ tbl, int b, int pos,
                                           bool want) {
  const int blk = pos / p.bs;
  const bool in = want && blk >= 0 && blk < p.stride;
  const int e = __ldg(tbl + (int64_t)b * p.stride + (in ? blk : 0));
  if (!want) return -1;
  if (!in || e < 0 || e >= p.block_num) {
    atomicOr(p.err, kErrIndex);
    return -1;
  }
  return e;
}

// Warps 4-5: validation, output-row offsets, per-token facts, the window of
// every output row, and, for this CTA's channels (columns half * D + ch0 .. +3),
// the state rows of those windows, ape, norm_weight and the RoPE table entries.
// Loads are grouped in three waves: inputs, block-table entries, state rows.
// Also pre-reduces every window's state rows per channel, so that the pooling
// after the stream only adds this call's rows.
template <int MAXT>
__device__ void call_metadata(const Params& p, Smem<MAXT>& sm, int NT, int ch0) {
  const int et = threadIdx.x - kMetaBase;  // 0..63
  const int B = p.B, r = p.ratio;
  const int rows = p.coff * r;
  const int r0 = p.D - p.rope, hr = p.rope / 2;
  const bool roped = ch0 >= r0;

  // ---- first wave of loads: everything that depends on nothing ----
  int cuv[5], spv[4];
#pragma unroll
  for (int u = 0; u < 5; ++u) {
    const int i = et + 64 * u;
    cuv[u] = i <= B ? __ldg(p.cu_in + i) : 0;
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int i = et + 64 * u;
    spv[u] = (i < B && p.start_pos) ? __ldg(p.start_pos + i) : 0;
  }
  float4 apev[2];
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int j = et + 64 * u;
    const int jj = j < rows ? j : 0;
    const int half = (p.coff == 2 && jj >= r) ? 1 : 0;
    apev[u] = __ldg(reinterpret_cast<const float4*>(p.ape + (int64_t)(jj % r) * p.C + half * p.D + ch0));
  }
  const float normv = __bfloat162float(p.norm_w[ch0 + (et & (OWN - 1))]);
  uint32_t rp[4] = {0u, 0u, 0u, 0u};  // cos[j0..j0+1], cos[hr+j0..], sin[j0..], sin[hr+j0..] as bf16 pairs
  const int nr = et < p.n_out ? et : 0;
  if (roped) {
    const int j0 = (ch0 - r0) >> 1;
    const __nv_bfloat16* cs = p.cos + (int64_t)nr * p.rope;
    const __nv_bfloat16* sn = p.sin + (int64_t)nr * p.rope;
    rp[0] = __ldg(reinterpret_cast<const unsigned int*>(cs + j0));
    rp[1] = __ldg(reinterpret_cast<const unsigned int*>(cs + hr + j0));
    rp[2] = __ldg(reinterpret_cast<const unsigned int*>(sn + j0));
    rp[3] = __ldg(reinterpret_cast<const unsigned int*>(sn + hr + j0));
  }
  // rotation: this CTA's 4 columns of the hadamard matrix, rows et, et + 64, ...
  uint2 hv[8];
  if (p.rotate) {
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int k = et + 64 * u;
      hv[u] = k < p.D ? __ldg(reinterpret_cast<const uint2*>(p.had + (int64_t)k * p.D + ch0)) : make_uint2(0u, 0u);
    }
  }
  // these loads are issued: let the weight stream start behind them
  asm volatile("bar.arrive 3, 96;" ::: "memory");
#pragma unroll
  for (int u = 0; u < 5; ++u)
    if (et + 64 * u <= B) sm.cu[et + 64 * u] = cuv[u];
#pragma unroll
  for (int u = 0; u < 4; ++u)
    if (et + 64 * u < B) sm.sp[et + 64 * u] = spv[u];
#pragma unroll
  for (int u = 0; u < 2; ++u)
    if (et + 64 * u < rows) *reinterpret_cast<float4*>(&sm.ape[et + 64 * u][0]) = apev[u];
  if (et < OWN) sm.norm[et] = normv;
  if (p.rotate) {
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int k = et + 64 * u;
      if (k < p.D) {
        const __nv_bfloat162 h01 = *reinterpret_cast<const __nv_bfloat162*>(&hv[u].x);
        const __nv_bfloat162 h23 = *reinterpret_cast<const __nv_bfloat162*>(&hv[u].y);
        sm.hcolT[0][k] = __low2float(h01);
        sm.hcolT[1][k] = __high2float(h01);
        sm.hcolT[2][k] = __low2float(h23);
        sm.hcolT[3][k] = __high2float(h23);
      }
    }
  }
  if (roped && et < p.n_out) {
    float* d = sm.rope[et];
#pragma unroll
    for (int u = 0; u < 2; ++u) {  // pair u: channels ch0 + 2u, ch0 + 2u + 1
      d[4 * u + 0] = __bfloat162float(__ushort_as_bfloat16((unsigned short)(rp[0] >> (16 * u))));
      d[4 * u + 1] = __bfloat162float(__ushort_as_bfloat16((unsigned short)(rp[1] >> (16 * u))));
      d[4 * u + 2] = __bfloat162float(__ushort_as_bfloat16((unsigned short)(rp[2] >> (16 * u))));
      d[4 * u + 3] = __bfloat162float(__ushort_as_bfloat16((unsigned short)(rp[3] >> (16 * u))));
    }
  }
  if (et == 0) sm.rejected = 0;
  for (int n = et; n < kMaxOut; n += 64) sm.win[n].w = -1;
  asm volatile("bar.sync 2, 64;" ::: "memory");
  CP_STAMP(et == 0, 16);  // first wave landed

  // ---- validation, offsets, tokens, windows (shared memory only) ----
  bool bad = false;
  for (int i = et; i <= B; i += 64) {
    const int c = sm.cu[i];
    bool ok = c >= 0 && c <= p.T && (i != 0 || c == 0) && (i != B || c == p.T);
    if (i < B) {
      const int c1 = sm.cu[i + 1], s = sm.sp[i];
      ok = ok && c1 >= c && s >= 0 && (int64_t)s + (c1 - c) <= (int64_t)INT32_MAX;
    }
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
        cap = min(L, L / r + 1);
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
      if (rejected && blockIdx.x == 0) atomicOr(p.err, kErrIndex);
    }
  }
  asm volatile("bar.sync 2, 64;" ::: "memory");
  // this thread's token t = et (T <= 64): sequence, position, tail?
  int tb = -1, tpos = 0;
  bool ttail = false;
  if (et < p.T && !rejected) {
    int lo = 0, hi = B;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (sm.cu[mid] <= et) lo = mid; else hi = mid - 1;
    }
    if (lo < B) {
      const int s = sm.sp[lo];
      tb = lo;
      tpos = s + (et - sm.cu[lo]);
      ttail = tpos >= tail_threshold(s + (sm.cu[lo + 1] - sm.cu[lo]), r, p.coff);
    }
  }
  // the window of output row n = et (n_out <= 64): the sequence b whose rows
  // off[b] .. off[b+1]-1 hold it, its k-th completed window if k < e/r - s/r
  if (et < p.n_out && !rejected) {
    int lo = 0, hi = B;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (sm.off[mid] <= et) lo = mid; else hi = mid - 1;
    }
    if (lo < B) {
      const int b = lo, k = et - sm.off[b];
      const int s = sm.sp[b], cu = sm.cu[b], e = s + (sm.cu[b + 1] - cu);
      if (k < e / r - s / r) {
        const int w = s / r + k;
        Win wi;
        wi.w = w;
        wi.b = b;
        wi.s = s;
        wi.cu = cu;
        wi.hrows = max(0, min(rows, s - window_pos(w, 0, r, p.coff)));
        wi.hist = -1;
        sm.win[et] = wi;
      }
    }
  }
  asm volatile("bar.sync 2, 64;" ::: "memory");
  if (et < 32) {
    // rows 2et, 2et+1 (n_out <= 64): exclusive scans of window count and state
    // rows give the window list and the prefetch ranges; a window whose state
    // rows do not fit in the prefetch buffer (and every later one) reads them
    // from the paged state instead (hist -1, empty range)
    int hw[2], hr[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int n = 2 * et + u;
      hw[u] = n < p.n_out && sm.win[n].w >= 0 ? 1 : 0;
      hr[u] = hw[u] ? sm.win[n].hrows : 0;
    }
    int iw = hw[0] + hw[1], ih = hr[0] + hr[1];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int a1 = __shfl_up_sync(0xffffffffu, iw, o), a2 = __shfl_up_sync(0xffffffffu, ih, o);
      if (et >= o) { iw += a1; ih += a2; }
    }
    const int nw_total = __shfl_sync(0xffffffffu, iw, 31);
    int pw = iw - hw[0] - hw[1], ph = ih - hr[0] - hr[1];  // exclusive prefixes
    int fit_end = 0;
    bool fits[2];
    int start[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      start[u] = ph;
      fits[u] = hr[u] > 0 && ph + hr[u] <= kHistRows;
      if (fits[u]) fit_end = ph + hr[u];
      if (hw[u]) sm.wlist[pw] = 2 * et + u;
      pw += hw[u];
      ph += hr[u];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) fit_end = max(fit_end, __shfl_xor_sync(0xffffffffu, fit_end, o));
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int n = 2 * et + u;
      if (n < p.n_out) {
        sm.hstart[n] = min(start[u], fit_end);  // non-decreasing; empty past the last fitting window
        if (hw[u]) sm.win[n].hist = fits[u] ? start[u] : -1;
      }
    }
    if (et == 0) {
      sm.hstart[p.n_out] = fit_end;
      sm.n_win = nw_total;
    }
  }
  asm volatile("bar.sync 2, 64;" ::: "memory");

  CP_STAMP(et == 0, 17);  // windows and prefetch ranges known
  // ---- second wave of loads: block-table entries (tails, then hist rows i = et + 64u) ----
  const int total = sm.hstart[p.n_out];
  int hb[4], hq[4], hj[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int i = et + 64 * u;
    hb[u] = -1;
    hq[u] = -1;
    hj[u] = 0;
    if (i < total) {
      int lo = 0, hi = p.n_out - 1;  // the last row n with hstart[n] <= i owns hist row i
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (sm.hstart[mid] <= i) lo = mid; else hi = mid - 1;
      }
      const Win& wi = sm.win[lo];
      hj[u] = i - wi.hist;
      hq[u] = window_pos(wi.w, hj[u], r, p.coff);
      hb[u] = wi.b;
    }
  }
  const int tkv = table_entry(p, p.kv_tbl, tb < 0 ? 0 : tb, tpos, ttail);
  const int tsc = table_entry(p, p.sc_tbl, tb < 0 ? 0 : tb, tpos, ttail);
  int hkv[4], hsc[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const bool want = hb[u] >= 0 && hq[u] >= 0;
    hkv[u] = table_entry(p, p.kv_tbl, want ? hb[u] : 0, want ? hq[u] : 0, want);
    hsc[u] = table_entry(p, p.sc_tbl, want ? hb[u] : 0, want ? hq[u] : 0, want);
  }
  if (et < NT) {
    TokInfo ti{tb, tpos, -1, -1};
    if (tkv >= 0) ti.kv_off = ((int64_t)tkv * p.bs + tpos % p.bs) * p.C;
    if (tsc >= 0) ti.sc_off = ((int64_t)tsc * p.bs + tpos % p.bs) * p.C;
    sm.tok[et] = ti;
  }

  CP_STAMP(et == 0, 18);  // second wave landed
  // ---- third wave of loads: the state rows (a row that does not exist: kv 0, score -inf) ----
  float4 v[4][2];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const bool ok = hkv[u] >= 0 && hsc[u] >= 0;
    const int qp = ok ? hq[u] : 0;
    const int col = ((p.coff == 2 && hj[u] >= r) ? p.D : 0) + ch0;
    const float4* kp = reinterpret_cast<const float4*>(
        p.kv_state + ((int64_t)(ok ? hkv[u] : 0) * p.bs + qp % p.bs) * p.C + col);
    const float4* sp = reinterpret_cast<const float4*>(
        p.score_state + ((int64_t)(ok ? hsc[u] : 0) * p.bs + qp % p.bs) * p.C + col);
    v[u][0] = ok ? *kp : make_float4(0.f, 0.f, 0.f, 0.f);
    v[u][1] = ok ? *sp : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int i = et + 64 * u;
    if (i < total) {
      *reinterpret_cast<float4*>(&sm.hist[i][0]) = v[u][0];
      *reinterpret_cast<float4*>(&sm.hist[i][OWN]) = v[u][1];
    }
  }
  asm volatile("bar.sync 2, 64;" ::: "memory");
  CP_STAMP(et == 0, 19);  // third wave landed

  // ---- every window's state rows, pre-reduced per channel (online softmax);
  // two lanes per (window, channel) take alternate rows and merge ----
  for (int base = 0; base < sm.n_win * OWN * 2; base += 64) {
    const int u = (base + et) >> 1, side = et & 1;
    const bool live = u < sm.n_win * OWN;
    const int i = live ? u / OWN : 0, c = u % OWN;
    const Win w = sm.win[sm.wlist[i]];
    float m = -INFINITY, l = 0.f, acc = 0.f;
    for (int j = side; j < w.hrows && live; j += 2) {
      float kv, z;
      if (w.hist >= 0) {
        kv = sm.hist[w.hist + j][c];
        z = sm.hist[w.hist + j][OWN + c];
      } else {  // more state rows than the prefetch holds: from the paged state
        const int qp = window_pos(w.w, j, r, p.coff);
        if (qp < 0) continue;
        const int rk = table_row(p, p.kv_tbl, w.b, qp);
        const int rs = table_row(p, p.sc_tbl, w.b, qp);
        if (rk < 0 || rs < 0) continue;
        const int col = ((p.coff == 2 && j >= r) ? p.D : 0) + ch0 + c;
        kv = p.kv_state[((int64_t)rk * p.bs + qp % p.bs) * p.C + col];
        z = p.score_state[((int64_t)rs * p.bs + qp % p.bs) * p.C + col];
      }
      if (z == -INFINITY) continue;  // a row that does not exist
      const float mn = fmaxf(m, z);
      const float f = __expf(m - mn), e = __expf(z - mn);
      l = l * f + e;
      acc = acc * f + e * kv;
      m = mn;
    }
    {
      const float m2 = __shfl_xor_sync(0xffffffffu, m, 1);
      const float l2 = __shfl_xor_sync(0xffffffffu, l, 1);
      const float a2 = __shfl_xor_sync(0xffffffffu, acc, 1);
      const float mn = fmaxf(m, m2);
      const float f1 = m == -INFINITY ? 0.f : __expf(m - mn);
      const float f2 = m2 == -INFINITY ? 0.f : __expf(m2 - mn);
      l = l * f1 + l2 * f2;
      acc = acc * f1 + a2 * f2;
      m = mn;
    }
    if (live && side == 0) sm.hst[i][c] = make_float4(m, l, acc, 0.f);
  }
}

// The complete projection of kind k (0 kv, 1 score), half h of the state row
// (coff 2: 0 = columns [0, D), 1 = [D, 2D); coff 1: 0), channel c and token t:
// the four received partials added in rank order.
template <int MAXT>
__device__ __forceinline__ float own_value(const Smem<MAXT>& sm, int h, int k, int c, int t) {
  return ((sm.recv[h][0][k][c][t] + sm.recv[h][1][k][c][t]) + sm.recv[h][2][k][c][t]) + sm.recv[h][3][k][c][t];
}

__device__ __forceinline__ void warp_sync_all() { __syncwarp(0xffffffffu); }

// A warp waits for a phase of an mbarrier: lane 0 polls (a whole warp
// spinning would crowd the shared-memory pipe), then the warp synchronises. Bounded (~2 s); with `abort` non-null it also
// gives up when another role aborted, and raises the flag when it times out.
// Returns the same answer in every lane.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) {
    const uint32_t a = smem_u32(bar);
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(a, parity)) {
      if (abort && *abort) { ok = 0; break; }
      if (globaltimer() - t0 > 2000000000ull) {
        ok = 0;
        if (abort) *abort = 1;
        break;
      }
    }
  }
  ok = __shfl_sync(0xffffffffu, ok, 0);
  __syncwarp(0xffffffffu);
  return ok != 0;
}

// A read-out warp w (0..3) holds accumulator rows 16w .. 16w+15 in its TMEM
// lanes 0-15 (an M = 64 accumulator, columns = tokens): for coff 2 the rows of
// matrix w / 2, half w % 2; for coff 1 those of matrix w (warps 0, 1). Each
// lane pushes its row to the CTA that owns the channel, into its
// recv[half][this rank][kind][channel][*]. False if the accumulator never
// completed (nothing is sent).
template <int MAXT>
__device__ bool send_partials(Smem<MAXT>& sm, uint32_t tmem, int w, int coff, int NT, int kv_first, uint32_t q,
                              volatile int* abort) {
  const int lane = threadIdx.x & 31;
  const int matrix = coff == 2 ? w >> 1 : w, half = coff == 2 ? w & 1 : 0;
  if (!warp_wait(&sm.acc_full, 0, abort)) return false;
  tc_fence_after();
  const int kind = ((matrix == 0) == (kv_first != 0)) ? 0 : 1;
  const int cg = lane & 15;
  const uint32_t owner = (uint32_t)(cg / OWN);
  const uint32_t dst = peer_addr(&sm.recv[half][q][kind][cg % OWN][0], owner);
  const uint32_t mbar = peer_addr(&sm.recv_full, owner);
  for (int c0 = 0; c0 < NT; c0 += 32) {
    uint32_t r[32];
    tmem_ld32(tmem + ((uint32_t)(32 * w) << 16) + (uint32_t)c0, r);
    tmem_ld_wait(r);
    if (lane < 16) {
#pragma unroll
      for (int j = 0; j < 32; j += 4)
        if (c0 + j < NT) st_async4(dst + (uint32_t)(c0 + j) * 4u, r[j], r[j + 1], r[j + 2], r[j + 3], mbar);
    }
  }
  return true;
}

// A whole warp waits (bounded, ~2 s, not cut short by the CTA's abort flag:
// pushes into this CTA must land before it goes on) for a phase of pushes.
__device__ __forceinline__ bool wait_pushes(uint64_t* bar) { return warp_wait(bar, 0, nullptr); }

// Warps 1-3: every (half, kind) pair of this CTA's 4 channels goes to the
// state tail rows (score rows with ape); warp 1 + f takes pairs f, f + 3.
template <int MAXT>
__device__ void write_tails(const Params& p, const Smem<MAXT>& sm, int ch0, int f) {
  const int r = p.ratio;
  for (int pair = f; pair < 2 * p.coff; pair += 3) {
    const int half = pair >> 1, k = pair & 1;
    for (int t = threadIdx.x & 31; t < p.T; t += 32) {
      const TokInfo ti = sm.tok[t];
      const int64_t so = k ? ti.sc_off : ti.kv_off;
      if (ti.b < 0 || so < 0) continue;
      float4 v = make_float4(own_value(sm, half, k, 0, t), own_value(sm, half, k, 1, t),
                             own_value(sm, half, k, 2, t), own_value(sm, half, k, 3, t));
      if (k) v = add4(v, *reinterpret_cast<const float4*>(&sm.ape[half * r + ti.pos % r][0]));
      *reinterpret_cast<float4*>((k ? p.score_state : p.kv_state) + so + half * p.D + ch0) = v;
    }
  }
}

__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 7, 128;" ::: "memory"); }

// Warps 0-3 (128 threads), once the partials have landed and the metadata is
// done: pool this CTA's 4 channels of every window the call completes. Two
// threads per (window, channel) take alternate rows of this call (the state
// rows come pre-reduced) and merge; the windows' sums of squares over the 4
// channels go to ss_own, RoPE(y * norm_weight) of a rotating call to ybuf.
template <int MAXT>
__device__ void pool_windows(const Params& p, Smem<MAXT>& sm, int ch0, bool ok) {
  const int tid = threadIdx.x;  // 0..127
  const int r = p.ratio, rows = p.coff * r, nw = sm.n_win;
  for (int base = 0; base < nw * OWN * 2; base += 128) {
    const int u = (base + tid) >> 1, side = tid & 1;
    const int i = u / OWN, c = u % OWN;
    const bool live = i < nw;
    float y = 0.f;
    int n = 0;
    float m = -INFINITY, l = 0.f, acc = 0.f;
    if (live) {
      n = sm.wlist[i];
      const Win w = sm.win[n];
      if (side == 0) {
        const float4 h = sm.hst[i][c];
        m = h.x;
        l = h.y;
        acc = h.z;
      }
      for (int j = w.hrows + side; j < rows && ok; j += 2) {  // this call's rows
        const int h = (p.coff == 2 && j >= r) ? 1 : 0;
        const int t = w.cu + (window_pos(w.w, j, r, p.coff) - w.s);
        const float kv = own_value(sm, h, 0, c, t);
        const float z = own_value(sm, h, 1, c, t) + sm.ape[j][c];
        const float mn = fmaxf(m, z);
        const float f = __expf(m - mn), e = __expf(z - mn);
        l = l * f + e;
        acc = acc * f + e * kv;
        m = mn;
      }
    }
    {  // merge the two sides
      const float m2 = __shfl_xor_sync(0xffffffffu, m, 1);
      const float l2 = __shfl_xor_sync(0xffffffffu, l, 1);
      const float a2 = __shfl_xor_sync(0xffffffffu, acc, 1);
      const float mn = fmaxf(m, m2);
      const float f1 = m == -INFINITY ? 0.f : __expf(m - mn);
      const float f2 = m2 == -INFINITY ? 0.f : __expf(m2 - mn);
      l = l * f1 + l2 * f2;
      acc = acc * f1 + a2 * f2;
    }
    y = (live && ok && l > 0.f) ? __fdividef(acc, l) : 0.f;
    if (live && side == 0) sm.ybuf[n][c] = y;
    // the window's sum of squares over the 4 channels (threads 8i' .. 8i'+7)
    float s = side == 0 ? y * y : 0.f;
    s += __shfl_xor_sync(0xffffffffu, s, 2);
    s += __shfl_xor_sync(0xffffffffu, s, 4);
    if (live && (tid & 7) == 0) sm.ss_own[i] = s;
  }
  epi_sync();
  if (p.rotate) {  // u = RoPE(y * norm_weight) of this CTA's channels, per window
    const bool roped = ch0 >= p.D - p.rope;
    for (int i = tid; i < nw; i += 128) {
      const int n = sm.wlist[i];
      float z[OWN];
#pragma unroll
      for (int c = 0; c < OWN; ++c) z[c] = sm.ybuf[n][c] * sm.norm[c];
      if (roped) rope4(z, sm.rope[n]);
      *reinterpret_cast<float4*>(&sm.ybuf[n][0]) = make_float4(z[0], z[1], z[2], z[3]);
    }
    epi_sync();
  }
}

// Warp 0: exchange the windows' sums of squares (and, rotating, u) with every
// CTA: this CTA's go to global memory, one lane arrives (release) at the
// counter, waits (acquire) for all arrivals, and the warp reads every CTA's sums
// (weak loads that bypass L1, all in flight at once) and adds them in a fixed
// order into ss_tot.
template <int MAXT>
__device__ void exchange_sums(const Params& p, Smem<MAXT>& sm, const CpArgs& a, int ch0) {
  const int lane = threadIdx.x & 31;
  const int nw = sm.n_win;
  if (lane == 0) {
    for (int i = 0; i < nw; ++i) {
      a.sums[(int64_t)i * kMaxCtas + blockIdx.x] = sm.ss_own[i];
      if (p.rotate)
        *reinterpret_cast<float4*>(a.u + (int64_t)i * 512 + ch0) =
            *reinterpret_cast<const float4*>(&sm.ybuf[sm.wlist[i]][0]);
    }
    arrive_release(a.counter, kPerLaunch / gridDim.x);
  }
  CP_STAMP(lane == 0, 7);  // pooled, arrived
  int got = 1;
  if (lane == 0) {
    const uint32_t target = sm.target + a.target_extra;
    const uint64_t t0 = globaltimer();
    while ((int32_t)(arrivals_now(a.counter) - target) < 0) {
      if (globaltimer() - t0 > 1000000000ull) {
        got = 0;
        break;
      }
    }
  }
  CP_STAMP(lane == 0, 11);  // all CTAs arrived
  got = __shfl_sync(0xffffffffu, got, 0);
  if (!got && lane == 0) {
    atomicOr(p.err, kErrTimeout);
    sm.xch_ok = 0;
  }
  warp_sync_all();
  // rotation: warps 1-3 load every window's u while this warp reads the sums
  // (the barrier carries this warp's acquire to them)
  if (p.rotate) asm volatile("bar.arrive 5, 128;" ::: "memory");
  if (got) {
    const int per_lane = (int)gridDim.x / 32;  // 1 or 4 partials per lane and window
    if (per_lane == 1) {  // 32 CTAs: 16 windows' partials in flight per lane at once
      for (int i0 = 0; i0 < nw; i0 += 16) {
        float v[16];
#pragma unroll
        for (int u = 0; u < 16; ++u)
          v[u] = i0 + u < nw ? __ldcg(a.sums + (int64_t)(i0 + u) * kMaxCtas + lane) : 0.f;
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          float t = v[u];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
          if (lane == 0 && i0 + u < nw) sm.ss_tot[i0 + u] = t;
        }
      }
    } else {
      for (int i0 = 0; i0 < nw; i0 += 8) {
        float v[8][4];
#pragma unroll
        for (int u = 0; u < 8; ++u)
#pragma unroll
          for (int k = 0; k < 4; ++k)
            v[u][k] = (i0 + u < nw && k < per_lane) ? __ldcg(a.sums + (int64_t)(i0 + u) * kMaxCtas + lane + 32 * k)
                                                   : 0.f;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          float t = ((v[u][0] + v[u][1]) + v[u][2]) + v[u][3];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
          if (lane == 0 && i0 + u < nw) sm.ss_tot[i0 + u] = t;
        }
      }
    }
  }
  warp_sync_all();
  CP_STAMP(lane == 0, 9);  // exchange complete
}

// Rotation, warps 1-3 (96 threads) once every CTA has arrived: every window's
// u (all D channels, published with the arrivals) into the now idle A ring,
// rows of D + 8 floats (16-byte aligned, rows on different banks), 8 loads in
// flight per thread.
template <int MAXT>
__device__ void load_u_rows(const Params& p, Smem<MAXT>& sm, const CpArgs& a) {
  asm volatile("bar.sync 5, 128;" ::: "memory");
  if (sm.xch_ok == 0) return;
  const int t = threadIdx.x - 32;
  const int nw = sm.n_win;
  const int per_row = p.D / 4;
  const int n4 = nw * per_row;
  float* uall = reinterpret_cast<float*>(&sm.a[0][0]);
  for (int v0 = 0; v0 < n4; v0 += 96 * 8) {
    float4 x4[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int v = v0 + t + 96 * e;
      if (v < n4) x4[e] = __ldcg(reinterpret_cast<const float4*>(a.u + (int64_t)(v / per_row) * 512 + 4 * (v % per_row)));
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int v = v0 + t + 96 * e;
      if (v < n4) *reinterpret_cast<float4*>(uall + (v / per_row) * (p.D + 8) + 4 * (v % per_row)) = x4[e];
    }
  }
}

// Warps 0-3: RMSNorm scale, norm_weight, RoPE and the bf16 store of this CTA's
// channels of every window row; with the rotation, output column ch0 + c of a
// window is scale * sum_k u[k] * hadamard[k][ch0 + c], one thread (two, for up
// to 64 pairs, taking alternate groups of four k) per (window, column), four
// interleaved partial sums from 16-byte shared-memory loads.
template <int MAXT>
__device__ void finish_rows(const Params& p, Smem<MAXT>& sm, const CpArgs& a, int ch0, bool ok) {
  const int tid = threadIdx.x;
  const int nw = sm.n_win;
  const bool fin = ok && sm.xch_ok != 0;
  if (p.rotate) {
    const float* uall = reinterpret_cast<const float*>(&sm.a[0][0]);
    // up to 64 (window, column) pairs: two adjacent lanes per pair, one taking
    // the even and one the odd groups of 4 channels, combined by a shuffle
    const int split = nw * OWN <= 64 ? 2 : 1;
    for (int u = tid; u < nw * OWN * split; u += 128) {
      const int pr = u / split, part = u % split;
      const int i = pr / OWN, c = pr % OWN;
      float o = 0.f;
      if (fin) {
        const float* ui = uall + i * (p.D + 8) + 4 * part;
        const float* hc = sm.hcolT[c] + 4 * part;
        float s4[4] = {0.f, 0.f, 0.f, 0.f};
        for (int k = 0; k < p.D; k += 4 * split) {
          const float4 uv = *reinterpret_cast<const float4*>(ui + k);
          const float4 hv = *reinterpret_cast<const float4*>(hc + k);
          s4[0] = fmaf(uv.x, hv.x, s4[0]);
          s4[1] = fmaf(uv.y, hv.y, s4[1]);
          s4[2] = fmaf(uv.z, hv.z, s4[2]);
          s4[3] = fmaf(uv.w, hv.w, s4[3]);
        }
        o = (s4[0] + s4[1]) + (s4[2] + s4[3]);
      }
      if (split == 2) o += __shfl_xor_sync(__activemask(), o, 1);  // the pair's lanes are both active
      if (part == 0) {
        if (fin) o *= rsqrtf(sm.ss_tot[i] / (float)p.D + 1e-6f);
        p.out[(int64_t)sm.wlist[i] * p.D + ch0 + c] = __float2bfloat16_rn(o);
      }
    }
    CP_STAMP(tid == 0, 10);  // rows stored
    return;
  }
  const bool roped = ch0 >= p.D - p.rope;
  for (int i = tid; i < nw; i += 128) {
    const int n = sm.wlist[i];
    float z[OWN] = {0.f, 0.f, 0.f, 0.f};
    if (fin) {
      const float sc = rsqrtf(sm.ss_tot[i] / (float)p.D + 1e-6f);
#pragma unroll
      for (int c = 0; c < OWN; ++c) z[c] = sm.ybuf[n][c] * sc * sm.norm[c];
      if (roped) rope4(z, sm.rope[n]);
    }
    __nv_bfloat162 o01 = __floats2bfloat162_rn(z[0], z[1]);
    __nv_bfloat162 o23 = __floats2bfloat162_rn(z[2], z[3]);
    uint2 v;
    v.x = *reinterpret_cast<uint32_t*>(&o01);
    v.y = *reinterpret_cast<uint32_t*>(&o23);
    *reinterpret_cast<uint2*>(p.out + (int64_t)n * p.D + ch0) = v;
  }
  CP_STAMP(tid == 0, 10);  // rows stored
}

template <int MAXT>
__global__ void __launch_bounds__(kThreads, 1)
    decode_cp_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w,
                     Params p, CpArgs a, int NT) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  using SM = Smem<MAXT>;
  constexpr int STAGES = SM::S;
  SM& sm = smem_align1024<SM>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t q = cluster_rank();          // this CTA's share of the hidden dimension
  const int g = blockIdx.x / KQ;              // channel group of the cluster
  const int ch0 = g * GCH + (int)q * OWN;     // this CTA's channels after the reduction
  const int nsteps = p.H / (KQ * KPS * BK);   // pipeline steps per CTA
  const uint32_t a_tile = (uint32_t)p.coff * 2 * GCH * 128;  // one K block of A as it lands
  const uint32_t bytes = KPS * (a_tile + (uint32_t)NT * BK * 2);
  const uint32_t tmem_cols = NT <= 32 ? 32 : 64;
  CP_STAMP(threadIdx.x == 0, 0);  // entry

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    mbar_init(&sm.acc_full, 1);
    mbar_init(&sm.recv_full, 1);
    sm.abort = 0;
    sm.xch_ok = 1;
    fence_barrier_init();
    // what lands here from the cluster: every rank's coff halves x 2 kinds x
    // OWN channels x NT tokens
    mbar_arrive_expect_tx(&sm.recv_full, (uint32_t)(KQ * p.coff * 2 * OWN * NT * 4));
    prefetch_tmap(&map_w);
    prefetch_tmap(&map_x);
  }
  if (warp == 7) tmem_alloc(&sm.tmem_base, tmem_cols);
  cluster_arrive_relaxed();  // cluster barrier 0: this CTA runs (its barriers are initialized)
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort = &sm.abort;
  CP_STAMP(threadIdx.x == 0, 1);  // set-up done

  if (warp == 6) {
    // ---- TMA: the metadata's first loads go out before the weight stream (named barrier 3) ----
    asm volatile("bar.sync 3, 96;" ::: "memory");
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      Armed armed;
      for (int st = 0; st < nsteps; ++st) {
        if (!mbar_wait(&sm.empty[stage], phase ^ 1u, abort)) break;
        mbar_arrive_expect_tx(&sm.full[stage], bytes);
        armed.note(stage, phase);
        // K blocks cb, cb+1: clusters start at different steps, the four CTAs of
        // a cluster take adjacent chunks
        const int cb = (((st + g) % nsteps) * KQ + (int)q) * KPS;
        tma_load_5d(sm.a[stage], &map_w, &sm.full[stage], 0, g * GCH, 0, 0, cb);
        tma_load_3d(sm.x[stage], &map_x, &sm.full[stage], 0, 0, cb);
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
      drain_armed(sm.full, STAGES, armed);  // no copy still landing when the CTA leaves
    }
  } else if (warp == 7) {
    // ---- MMA (M = 64): every A row of the stage in one accumulator ----
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      const uint32_t idesc = idesc_bf16_f32(64, NT);
      bool ok = true;
      for (int st = 0; st < nsteps; ++st) {
        if (!mbar_wait(&sm.full[stage], phase, abort)) { ok = false; break; }
        CP_STAMP(st == 0, 2);  // first stage landed
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < KPS; ++kk) {
          // the copies land packed: KPS A tiles of a_tile bytes, KPS x tiles of NT rows
          const uint32_t a0 = smem_u32(sm.a[stage]) + kk * a_tile;
          const uint32_t b0 = smem_u32(sm.x[stage]) + kk * NT * 128;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            mma_bf16(tmem, sw128_kmajor_desc(a0 + k * 32), sw128_kmajor_desc(b0 + k * 32), idesc,
                     (st > 0 || kk > 0 || k > 0) ? 1u : 0u);
        }
        mma_commit(&sm.empty[stage]);
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
      if (ok) mma_commit(&sm.acc_full);
      CP_STAMP(true, 3);  // last MMA issued
    }
  } else if (warp >= 4) {
    // ---- warps 4-5: metadata and prefetch ----
    call_metadata<MAXT>(p, sm, NT, ch0);
    CP_STAMP(threadIdx.x == kMetaBase, 4);  // metadata done
    asm volatile("bar.arrive 4, 192;" ::: "memory");  // to warps 0-3
  } else {
    // ---- warps 0-3: read-out, pooling; then warp 0 exchanges the sums while
    // warps 1-3 write the state tails and the rows without a window; then all
    // four store the rows ----
    uint32_t ctr = 0;
    if (warp == 0) ctr = arrivals_now(a.counter);  // this launch's base (a cold load)
    cluster_wait();  // cluster barrier 0: every CTA of the cluster runs before a push
    bool ok = true;
    if (warp < 2 * p.coff) ok = send_partials(sm, tmem, warp, p.coff, NT, a.kv_first, q, abort);
    CP_STAMP(threadIdx.x == 0, 5);  // partials sent
    ok = wait_pushes(&sm.recv_full) && ok;
    CP_STAMP(threadIdx.x == 0, 6);  // partials received
    if (threadIdx.x == 0) sm.target = ctr - ctr % kPerLaunch + kPerLaunch;
    asm volatile("bar.sync 4, 192;" ::: "memory");  // the metadata is done
    if (!ok && lane == 0) sm.abort = 1;
    epi_sync();
    const bool good = !*abort;
    pool_windows(p, sm, ch0, good);
    if (warp == 0) {
      exchange_sums(p, sm, a, ch0);
    } else {
      if (warp == 1)
        for (int n = lane; n < p.n_out; n += 32)
          if (sm.win[n].w < 0) *reinterpret_cast<uint2*>(p.out + (int64_t)n * p.D + ch0) = make_uint2(0u, 0u);
      if (good) write_tails(p, sm, ch0, warp - 1);
      CP_STAMP(threadIdx.x == 32, 14);  // tails written
      if (p.rotate) load_u_rows(p, sm, a);
    }
    epi_sync();
    finish_rows(p, sm, a, ch0, good);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 7) {
    tc_fence_after();
    tmem_dealloc(tmem, tmem_cols);
  }
  if (threadIdx.x == 0 && sm.abort) atomicOr(p.err, kErrTimeout);
  CP_STAMP(threadIdx.x == 0, 15);  // end
}

// x [T, H] as (column in block, row, 64-column block): a box of 64 columns x
// box_rows rows x kps blocks lands as kps tiles [block][row][128 B].
bool make_x_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows, int kps) {
  EncodeTiledFn f = encode_fn();
  if (!f) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)BK, rows, cols / BK};
  const cuuint64_t strides[2] = {cols * 2, (cuuint64_t)BK * 2};
  const cuuint32_t box[3] = {(cuuint32_t)BK, box_rows, (cuuint32_t)kps};
  const cuuint32_t estr[3] = {1, 1, 1};
  return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Both weight matrices [C, H] as one 5-D tensor: (column in block, row within a
// half, half, matrix, 64-column block), the matrix stride being the distance
// between the two allocations (the lower one first). A box of 64 columns x 16
// rows x coff halves x 2 matrices x kps blocks lands as kps A tiles
// [block][matrix][half][16 rows][128 B].
bool make_w_map(CUtensorMap* m, const Params& p, int* kv_first, int kps) {
  EncodeTiledFn f = encode_fn();
  if (!f) return false;
  const uintptr_t a = reinterpret_cast<uintptr_t>(p.wkv), b = reinterpret_cast<uintptr_t>(p.wgate);
  if (a == b) return false;
  const uintptr_t lo = a < b ? a : b, delta = a < b ? b - a : a - b;
  if (delta % 16 || delta >= (uintptr_t(1) << 40)) return false;
  *kv_first = a < b ? 1 : 0;
  const cuuint64_t dims[5] = {(cuuint64_t)BK, (cuuint64_t)p.D, (cuuint64_t)p.coff, 2, (cuuint64_t)p.H / BK};
  const cuuint64_t strides[4] = {(cuuint64_t)p.H * 2, (cuuint64_t)p.D * p.H * 2, (cuuint64_t)delta,
                                 (cuuint64_t)BK * 2};
  const cuuint32_t box[5] = {(cuuint32_t)BK, (cuuint32_t)GCH, (cuuint32_t)p.coff, 2, (cuuint32_t)kps};
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, reinterpret_cast<void*>(lo), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int MAXT>
size_t smem_bytes() {
  return sizeof(Smem<MAXT>) + 1024;
}

// Cluster shape (4 CTAs along x) and, with cooperative = true, the cooperative
// launch attribute.
template <int MAXT>
cudaLaunchConfig_t launch_config(int grid, cudaStream_t s, cudaLaunchAttribute (&attr)[2], bool cooperative) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem_bytes<MAXT>();
  cfg.stream = s;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = KQ;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeCooperative;
  attr[1].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = cooperative ? 2 : 1;
  return cfg;
}

int g_conf32[64] = {0}, g_conf64[64] = {0};
int g_disabled[64] = {0};  // set when the device refused the launch form

int current_device() {
  int dev = 0;
  cudaGetDevice(&dev);
  return dev;
}

// 4-CTA clusters of one variant that can be resident at once (cached per device).
template <int MAXT>
int max_clusters(int (&conf)[64]) {
  static int cached[64] = {0};
  const int dev = current_device();
  if (dev < 64 && cached[dev]) return cached[dev];
  int n = 0;
  cudaLaunchAttribute attr[2];
  cudaLaunchConfig_t cfg = launch_config<MAXT>(KQ, nullptr, attr, false);
  if (smem_attr_once(decode_cp_kernel<MAXT>, smem_bytes<MAXT>(), conf) != cudaSuccess ||
      cudaOccupancyMaxActiveClusters(&n, decode_cp_kernel<MAXT>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  if (dev < 64) cached[dev] = n > 0 ? n : -1;
  return n;
}

}  // namespace

bool decode_cp_supported(const Params& p) {
  if (p.T < 1 || p.T > 64 || p.B > kMaxSeqs || p.n_out > kMaxOut || p.rope != 64) return false;
  // rotation: every window's u (n_out rows of D + 8 floats) fits in the A ring
  if (p.rotate && (size_t)p.n_out * (p.D + 8) * 4 > sizeof(Smem<32>::a)) return false;
  if (p.coff * p.ratio > kMaxWinRows || p.H % (KQ * KPS * BK) || p.D % GCH || kMaxClusters % (p.D / GCH) ||
      encode_fn() == nullptr)
    return false;
  CUtensorMap w;
  int kv_first = 0;
  if (!make_w_map(&w, p, &kv_first, KPS)) return false;  // e.g. wkv and wgate at the same address
  const int dev = current_device();
  if (dev < 64 && g_disabled[dev]) return false;
  const int clusters = p.D / GCH;
  const int cap = p.T <= 32 ? max_clusters<32>(g_conf32) : max_clusters<64>(g_conf64);
  return cap >= clusters;
}

// Launch. If the device refuses the launch form itself (a cooperative launch of
// clusters), the path is disabled on this device and cudaErrorNotSupported is
// returned before anything ran, so that the caller can take another path.
cudaError_t launch_decode_cp(const Params& p, void* counter, void* xch, void* u, cudaStream_t s,
                             bool unreachable) {
  const int NT = (p.T + 15) / 16 * 16;
  CpArgs a;
  CUtensorMap mx, mw;
  if (!make_x_map(&mx, p.x, p.T, p.H, (uint32_t)NT, KPS) || !make_w_map(&mw, p, &a.kv_first, KPS))
    return cudaErrorInvalidValue;
  a.counter = static_cast<unsigned*>(counter);
  a.sums = static_cast<float*>(xch);
  a.u = static_cast<float*>(u);
  a.target_extra = unreachable ? kPerLaunch : 0u;
  const int grid = (p.D / GCH) * KQ;
  cudaLaunchAttribute attr[2];
  cudaError_t e;
  if (NT <= 32) {
    cudaLaunchConfig_t cfg = launch_config<32>(grid, s, attr, true);
    e = smem_attr_once(decode_cp_kernel<32>, cfg.dynamicSmemBytes, g_conf32);
    if (e == cudaSuccess) e = cudaLaunchKernelEx(&cfg, decode_cp_kernel<32>, mx, mw, p, a, NT);
  } else {
    cudaLaunchConfig_t cfg = launch_config<64>(grid, s, attr, true);
    e = smem_attr_once(decode_cp_kernel<64>, cfg.dynamicSmemBytes, g_conf64);
    if (e == cudaSuccess) e = cudaLaunchKernelEx(&cfg, decode_cp_kernel<64>, mx, mw, p, a, NT);
  }
  if (e == cudaErrorInvalidConfiguration || e == cudaErrorNotSupported ||
      e == cudaErrorCooperativeLaunchTooLarge) {
    cudaGetLastError();
    const int dev = current_device();
    if (dev < 64) g_disabled[dev] = 1;
    return cudaErrorNotSupported;
  }
  return e;
}

}  // namespace cmp

// Measurement hook: the phase stamps of the last channel-group decode launch
// (a -DCMP_PHASE_STAMPS build only; other builds return CMP_ERR_UNSUPPORTED).
extern "C" int cmp_debug_phase_stamps(uint64_t* dst, int64_t n) {
#ifdef CMP_PHASE_STAMPS
  if (!dst || n < 0 || n > (int64_t)cmp::kStampCtas * cmp::kStampSlots) return CMP_ERR_INVALID;
  if (cudaDeviceSynchronize() != cudaSuccess) return CMP_ERR_CUDA;
  return cudaMemcpyFromSymbol(dst, cmp::g_cp_stamps, sizeof(uint64_t) * (size_t)n) == cudaSuccess ? CMP_OK
                                                                                                   : CMP_ERR_CUDA;
#else
  (void)dst;
  (void)n;
  return CMP_ERR_UNSUPPORTED;
#endif
}
