// Decode by channel groups, in one cooperative kernel of 4-CTA clusters
// (T <= 64 tokens, B <= 256 sequences, no Hadamard rotation).
//
// The per-channel softmax pooling ("compressor torch_extension API", 计算公式
// 3-5) never mixes channels, so a cluster that holds the complete projections
// of some channels can pool them on its own:
//
//  1. Cluster g owns channels 16g .. 16g+15 of the D. Its four CTAs split the
//     hidden dimension by 64-column blocks (CTA q takes blocks q, q+4, ...: at
//     any moment the cluster reads 512 contiguous bytes of each weight row).
//     Per block, one TMA copy brings the wkv and wgate rows of those channels
//     (both halves for ratio 4, coff 2: 64 rows, else 32; one 4-D tensor map
//     spans both matrices) and one brings the x columns; tcgen05.mma
//     accumulates the rows x tokens product in TMEM (M = 128: the A rows past
//     the loaded ones are whatever shared memory follows and land in TMEM lanes
//     nobody reads). Clusters start at different blocks so that they spread
//     over the DRAM channels. Meanwhile warps 2-3 compute the call's metadata
//     (what the varlen scheduler kernel does on the other paths) and prefetch
//     what the later steps read: the state rows of every window the call
//     completes, ape, norm_weight and the RoPE tables, for this CTA's channels.
//  2. Each CTA pushes, into the shared memory of CTA q of the cluster, its
//     partial sums of the rows of channels 16g+4q .. 16g+4q+3; after a cluster
//     barrier CTA q adds the four partials (in quarter order) and holds complete
//     kv and score projections of 4 channels for every token of the call.
//  3. It writes those channels of the state tail rows (score + ape), pools the
//     4 channels of every window the call completes (a max pass, then an
//     exp-sum pass, so that the rows' loads and exponentials overlap), and
//     publishes each output row's sum of squares over its channels.
//  4. Grid barrier (bounded); RMSNorm needs the sum over all D channels. Each
//     CTA sums the D/4 partials of each row (fixed order), then scales its
//     channels, applies norm_weight and the interleaved RoPE (a pair never
//     straddles two CTAs) and stores bf16 ("CANN PyPTO 算子实战", 压缩窗口与状态更新).
//
// The weights are read once; x (small) once per cluster. No projection partial
// leaves the cluster: the only global exchange is n_out x D/4 floats.
// This call writes state slots of positions >= start_pos only and reads those
// below, so the prefetch and the tail stores never touch the same slot.
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
constexpr int kStampSlots = 16;
constexpr int kStampCtas = 512;
#ifdef CMP_PHASE_STAMPS
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
constexpr int kThreads = 128;     // warp 0: TMA lane, TMEM rows 0-31; warp 1: MMA lane, rows 32-63;
                                  // warps 2-3: call metadata and prefetch
constexpr int kMaxSeqs = 256;
constexpr int kMaxOut = 64;       // n_out <= T <= 64
constexpr int kHistRows = 256;    // prefetched state rows (this CTA's 4 kv + 4 score channels)
constexpr int kMaxWinRows = 128;  // coff * ratio
constexpr int KPS = 2;            // 64-column K blocks per TMA copy (pipeline stage)
constexpr int kTileA = 8192;      // one K block of A: 2 matrices x 2 halves x 16 rows x 128 B
constexpr int kSlackA = 16384 - kTileA;  // the 128-row window the MMA reads past the last tile
constexpr int kReplicas = 16;     // copies of the sum-of-squares partials (spread the readers)

// Pipeline depth: with 7 stages for T <= 32 each CTA had nearly its whole K
// range in flight at once; 4 measured 2 % faster (13.23 vs 13.5 us, bit-identical
// results), 3 slower.
template <int MAXT>
struct Cfg {
  static constexpr int stages = MAXT <= 32 ? 4 : 5;
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
  // stage s: KPS A tiles (kinds x 16 rows each) and KPS x tiles (NT rows each),
  // packed as the TMA boxes land them; after the MMAs, a[] holds the TMEM copy
  alignas(1024) unsigned char a[S][KPS * kTileA];
  unsigned char a_slack[kSlackA];
  alignas(1024) __nv_bfloat16 x[S][KPS * MAXT * BK];
  alignas(16) float recv[KQ][4 * MAXT * OWN]; // partials from each CTA of the cluster: [kind][token][channel]
  alignas(16) float hist[kHistRows][2 * OWN];  // state rows: kv c0..c3, score c0..c3
  alignas(16) float ape[kMaxWinRows][OWN];     // ape of window row j (half * ratio + residue)
  alignas(16) float rope[kMaxOut][8];          // per pair: cos even, cos odd, sin even, sin odd
  alignas(16) float ybuf[kMaxOut][OWN];
  float norm[OWN];
  float scale[kMaxOut];
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
  uint64_t acc_full;
  uint64_t recv_full;   // the four partial blocks have landed in recv
  uint32_t tmem_base;
  int abort;
  int rejected;
  uint32_t bar_target;
  int grid_ok;
};

static_assert(offsetof(Smem<32>, x) % 1024 == 0 && offsetof(Smem<64>, x) % 1024 == 0,
              "TMA swizzled tiles must be 1024-byte aligned");
static_assert(offsetof(Smem<32>, a_slack) == sizeof(Smem<32>::a) &&
                  offsetof(Smem<64>, a_slack) == sizeof(Smem<64>::a),
              "the MMA's 128-row window past the last stage must stay inside the slack");
static_assert(offsetof(Smem<32>, recv) % 16 == 0 && offsetof(Smem<64>, recv) % 16 == 0 &&
                  offsetof(Smem<32>, hist) % 16 == 0 && offsetof(Smem<64>, hist) % 16 == 0 &&
                  offsetof(Smem<32>, ape) % 16 == 0 && offsetof(Smem<64>, ape) % 16 == 0 &&
                  offsetof(Smem<32>, ybuf) % 16 == 0 && offsetof(Smem<64>, ybuf) % 16 == 0,
              "float4 shared-memory rows must be 16-byte aligned");
static_assert(KQ * 4 * 64 * OWN * 4 <= Cfg<64>::stages * KPS * kTileA &&
                  KQ * 4 * 32 * OWN * 4 <= Cfg<32>::stages * KPS * kTileA,
              "the outgoing partial blocks must fit in the stage buffers");
static_assert(sizeof(Smem<32>) + 1024 <= 232448 && sizeof(Smem<64>) + 1024 <= 232448,
              "shared memory per CTA");

// Grid barrier for a cooperative launch (every CTA is resident), one use per
// launch: a counter in memory that starts zeroed and only grows. Every launch
// adds exactly kQuantum to it (each of its n CTAs adds kQuantum / n), so at
// launch start it is a multiple of kQuantum, and a CTA that reads it before
// arriving rounds down to that multiple: the launch is complete when the
// counter reaches the next one. Arrival is a fire-and-forget release-add
// (publishing the CTA's stores); grid_wait polls with acquire loads, bounded
// (~1 s, then a timeout is recorded and the CTA goes on without the data).
// No reset and no last-arriver step: nothing serializes behind one CTA.
constexpr uint32_t kQuantum = 1024;

__device__ __forceinline__ uint32_t grid_target(const unsigned* counter) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(counter) : "memory");
  return v - v % kQuantum + kQuantum;
}

__device__ __forceinline__ void grid_arrive(unsigned* counter, unsigned nblocks) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(counter), "r"(kQuantum / nblocks) : "memory");
}

__device__ __forceinline__ bool grid_wait(const unsigned* counter, uint32_t target, unsigned* err) {
  const uint64_t t0 = globaltimer();
  for (;;) {
    uint32_t now;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(now) : "l"(counter) : "memory");
    if ((int32_t)(now - target) >= 0) return true;
    if (globaltimer() - t0 > 1000000000ull) {
      atomicOr(err, kErrTimeout);
      return false;
    }
  }
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

// Bulk copy of `bytes` from this CTA's shared memory into a peer's, completing
// on the peer's mbarrier (both addresses from peer_addr); one destination CTA per copy.
__device__ __forceinline__ void bulk_copy_to_peer(uint32_t dst, const void* src, uint32_t bytes, uint32_t mbar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "r"(smem_u32(src)), "r"(bytes), "r"(mbar)
      : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }

// Generic-proxy writes to shared memory before async-proxy reads of it.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
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

__device__ __forceinline__ float4 add4(float4 a, float4 b) {
  return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
}

struct CpArgs {
  float* ss;          // [kReplicas][n_out][D/4] each CTA's sum of squares of its channels, per output row
  unsigned* counter;  // grid-barrier counter (zeroed at creation)
  int kv_first;     // the 4-D weight map holds wkv before wgate (else the other way round)
  uint32_t bar_extra;  // added to the barrier target: kQuantum makes it unreachable (timeout test)
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

// Warps 2-3: validation, output-row offsets, per-token facts, the window of
// every output row, and, for this CTA's channels (columns half * D + ch0 .. +3),
// the state rows of those windows, ape, norm_weight and the RoPE table entries.
// Loads are grouped in three waves: inputs, block-table entries, state rows.
template <int MAXT>
__device__ void call_metadata(const Params& p, Smem<MAXT>& sm, int NT, int ch0) {
  const int et = threadIdx.x - 64;  // 0..63
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
  // these loads are issued: let the weight stream start behind them
  asm volatile("bar.arrive 3, 96;" ::: "memory");
  cluster_wait();  // cluster barrier 0 (every CTA of the cluster runs)
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
  // the windows the call completes: rows off[b] .. off[b] + (e/r - s/r) - 1
  for (int b = et; b < B && !rejected; b += 64) {
    const int s = sm.sp[b], cu = sm.cu[b], e = s + (sm.cu[b + 1] - cu);
    for (int k = 0; k < e / r - s / r; ++k) {
      const int w = s / r + k;
      Win wi;
      wi.w = w;
      wi.b = b;
      wi.s = s;
      wi.cu = cu;
      wi.hrows = max(0, min(rows, s - window_pos(w, 0, r, p.coff)));
      wi.hist = -1;
      sm.win[sm.off[b] + k] = wi;
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
}

// The complete projection of kind k, token t, channel c of this CTA: the four
// received partial blocks added in rank order.
template <int MAXT>
__device__ __forceinline__ float own_value(const Params& p, const Smem<MAXT>& sm, int k, int t, int c) {
  const int i = (k * p.T + t) * OWN + c;
  return ((sm.recv[0][i] + sm.recv[1][i]) + sm.recv[2][i]) + sm.recv[3][i];
}

__device__ __forceinline__ float4 own_value4(const float* r0, const float* r1, const float* r2, const float* r3) {
  const float4 a = *reinterpret_cast<const float4*>(r0), b = *reinterpret_cast<const float4*>(r1);
  const float4 c = *reinterpret_cast<const float4*>(r2), d = *reinterpret_cast<const float4*>(r3);
  return make_float4(((a.x + b.x) + c.x) + d.x, ((a.y + b.y) + c.y) + d.y, ((a.z + b.z) + c.z) + d.z,
                     ((a.w + b.w) + c.w) + d.w);
}

// Window row j's kv and score (score + ape for this call's tokens) for channel c.
template <int MAXT>
__device__ __forceinline__ void window_row(const Params& p, const Smem<MAXT>& sm, const Win& w, int j, int c,
                                           float& kv, float& z) {
  if (j < w.hrows) {
    kv = sm.hist[w.hist + j][c];
    z = sm.hist[w.hist + j][OWN + c];
  } else {
    const int r = p.ratio;
    const int half = (p.coff == 2 && j >= r) ? 1 : 0;
    const int t = w.cu + (window_pos(w.w, j, r, p.coff) - w.s);
    kv = own_value(p, sm, half, t, c);
    z = own_value(p, sm, p.coff + half, t, c) + sm.ape[j][c];
  }
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
  const int kinds = 2 * p.coff;               // kv halves, then score halves
  const int nsteps = p.H / (KQ * KPS * BK);   // pipeline steps per CTA (KPS K blocks each)
  const uint32_t bytes = KPS * ((uint32_t)kinds * GCH * BK * 2 + (uint32_t)NT * BK * 2);
  const uint32_t tmem_cols = NT <= 32 ? 32 : 64;
  // after the MMAs: the outgoing partials, one block per owner CTA [owner][kind][token][channel]
  float* part = reinterpret_cast<float*>(&sm.a[0][0]);
  const int blk_floats = kinds * p.T * OWN;
  CP_STAMP(threadIdx.x == 0, 0);  // entry

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    mbar_init(&sm.acc_full, 1);
    mbar_init(&sm.recv_full, 1);
    sm.abort = 0;
    fence_barrier_init();
    // the four incoming partial blocks (one of them this CTA's own)
    mbar_arrive_expect_tx(&sm.recv_full, (uint32_t)(KQ * kinds * p.T * OWN * 4));
    prefetch_tmap(&map_w);
    prefetch_tmap(&map_x);
  }
  if (warp == 1) tmem_alloc(&sm.tmem_base, tmem_cols);
  cluster_arrive_relaxed();  // cluster barrier 0: this CTA runs (its barriers are initialized)
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort = &sm.abort;
  CP_STAMP(threadIdx.x == 0, 1);  // set-up done

  // ---- 1) stream + MMA (lane 0 of warps 0, 1) / metadata and prefetch (warps 2, 3) ----
  // the metadata's first loads go out before the weight stream (named barrier 3)
  if (warp == 0) asm volatile("bar.sync 3, 96;" ::: "memory");
  if (warp == 0 && lane == 0) {
    int stage = 0;
    uint32_t phase = 0;
    for (int st = 0; st < nsteps; ++st) {
      if (!mbar_wait(&sm.empty[stage], phase ^ 1u, abort)) break;
      mbar_arrive_expect_tx(&sm.full[stage], bytes);
      // K blocks cb .. cb+KPS-1: clusters start at different steps, the four
      // CTAs of a cluster take adjacent chunks
      const int cb = (((st + g) % nsteps) * KQ + (int)q) * KPS;
      tma_load_5d(sm.a[stage], &map_w, &sm.full[stage], 0, g * GCH, 0, 0, cb);
      tma_load_3d(sm.x[stage], &map_x, &sm.full[stage], 0, 0, cb);
      if (++stage == STAGES) { stage = 0; phase ^= 1u; }
    }
  } else if (warp == 1 && lane == 0) {
    int stage = 0;
    uint32_t phase = 0;
    const uint32_t idesc = idesc_bf16_f32(128, NT);
    bool ok = true;
    for (int st = 0; st < nsteps; ++st) {
      if (!mbar_wait(&sm.full[stage], phase, abort)) { ok = false; break; }
      CP_STAMP(st == 0, 2);  // first stage landed
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < KPS; ++kk) {
        // the copies land packed: KPS A tiles of kinds x 16 rows, KPS x tiles of NT rows
        const uint32_t a0 = smem_u32(sm.a[stage]) + kk * kinds * GCH * 128;
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
  } else if (warp >= 2) {
    // the grid barrier's target, read here rather than before the stream starts
    // (a cold global load); any time before this CTA's own arrival is correct:
    // the count cannot reach the next multiple while this CTA's share is missing
    if (threadIdx.x == 64) sm.bar_target = grid_target(a.counter) + a.bar_extra;
    call_metadata<MAXT>(p, sm, NT, ch0);
    CP_STAMP(threadIdx.x == 64, 4);  // metadata and prefetch done
  }

  // ---- 2) warps 0-1: TMEM rows -> the owners' blocks, one bulk copy per owner;
  // every CTA then adds the four blocks it received (in rank order) ----
  if (warp < 2) {
    const bool have = mbar_wait(&sm.acc_full, 0, abort);
    CP_STAMP(threadIdx.x == 0, 5);  // accumulator complete
    __syncwarp();
    if (__all_sync(0xffffffffu, have) && warp * 32 < kinds * GCH) {
      tc_fence_after();
      // TMEM lane = A row: 16-row block of the tile, channel of the cluster's 16
      const int row = warp * 32 + lane, b = row / GCH, cg = row % GCH;
      const int k = a.kv_first ? b : (b + p.coff) % kinds;  // kind of that block
      float* dst = part + (cg / OWN) * blk_floats + k * p.T * OWN + cg % OWN;
      for (int c0 = 0; c0 < NT; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + c0, r);
        tmem_ld_wait(r);
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (c0 + j < p.T) dst[(c0 + j) * OWN] = __uint_as_float(r[j]);
      }
    }
    tc_fence_before();
    fence_proxy_async_smem();  // the blocks are read by the bulk copies
    asm volatile("bar.sync 1, 64;" ::: "memory");
    cluster_wait();  // cluster barrier 0: every CTA of the cluster runs, its barriers initialized
    if (threadIdx.x == 0) {
      const uint32_t bytes = (uint32_t)blk_floats * 4;
      for (int o = 0; o < KQ; ++o)
        bulk_copy_to_peer(peer_addr(&sm.recv[q][0], (uint32_t)o), part + o * blk_floats, bytes,
                          peer_addr(&sm.recv_full, (uint32_t)o));
      bulk_commit();
      CP_STAMP(true, 6);  // partial blocks sent
    }
  }
  if (threadIdx.x == 0) {
    // not cut short by this CTA's abort flag: the peers' copies into this CTA
    // must land before it goes on (and, at the latest, before it exits)
    int never = 0;
    if (!mbar_wait(&sm.recv_full, 0, &never)) atomicOr(p.err, kErrTimeout);
    CP_STAMP(true, 7);  // the four partial blocks landed
  }
  __syncthreads();  // the partials have landed, and the metadata is complete
  const bool mm_ok = !*abort;

  // ---- 3) pooling: 16 threads per window (4 channels x 4 row lanes), 8 windows at a time ----
  const int r = p.ratio, n_out = p.n_out, rows = p.coff * r, nw = sm.n_win;
  {
    const int c = (threadIdx.x >> 2) & 3, rl = threadIdx.x & 3;
    for (int wi = threadIdx.x >> 4; wi < nw + 7 - ((nw + 7) % 8); wi += kThreads / 16) {
      // every lane runs the shuffles; lanes past the last window compute nothing
      const bool live = wi < nw && mm_ok;
      const int n = live ? sm.wlist[wi] : 0;
      Win w = sm.win[n];
      float m = -INFINITY, l = 0.f, acc = 0.f;
      for (int j = rl; j < rows && live; j += 4) {
        float kv, z;
        if (j < w.hrows && w.hist < 0) {  // more state rows than the prefetch holds
          const int qp = window_pos(w.w, j, r, p.coff);
          if (qp < 0) continue;
          const int rk = table_row(p, p.kv_tbl, w.b, qp);
          const int rs = table_row(p, p.sc_tbl, w.b, qp);
          if (rk < 0 || rs < 0) continue;
          const int col = ((p.coff == 2 && j >= r) ? p.D : 0) + ch0 + c;
          kv = p.kv_state[((int64_t)rk * p.bs + qp % p.bs) * p.C + col];
          z = p.score_state[((int64_t)rs * p.bs + qp % p.bs) * p.C + col];
        } else {
          window_row(p, sm, w, j, c, kv, z);
        }
        if (z == -INFINITY) continue;  // a row that does not exist
        const float mn = fmaxf(m, z);
        const float f = __expf(m - mn), e = __expf(z - mn);
        l = l * f + e;
        acc = acc * f + e * kv;
        m = mn;
      }
      // merge the 4 row lanes of each channel (log-sum-exp)
#pragma unroll
      for (int o = 1; o < 4; o <<= 1) {
        const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
        const float l2 = __shfl_xor_sync(0xffffffffu, l, o);
        const float a2 = __shfl_xor_sync(0xffffffffu, acc, o);
        const float mn = fmaxf(m, m2);
        const float f1 = m == -INFINITY ? 0.f : __expf(m - mn);
        const float f2 = m2 == -INFINITY ? 0.f : __expf(m2 - mn);
        l = l * f1 + l2 * f2;
        acc = acc * f1 + a2 * f2;
        m = mn;
      }
      if (live && rl == 0) sm.ybuf[n][c] = l > 0.f ? __fdividef(acc, l) : 0.f;
    }
  }
  __syncthreads();
  CP_STAMP(threadIdx.x == 0, 8);  // pooled
  const int n_cta = gridDim.x;
  const int64_t rep_stride = (int64_t)n_out * n_cta;
  for (int i = threadIdx.x; i < nw * kReplicas; i += kThreads) {
    const int n = sm.wlist[i / kReplicas];
    const float4 y = *reinterpret_cast<const float4*>(&sm.ybuf[n][0]);
    a.ss[(i % kReplicas) * rep_stride + (int64_t)n * n_cta + blockIdx.x] =
        y.x * y.x + y.y * y.y + y.z * y.z + y.w * y.w;
  }
  __syncthreads();
  if (threadIdx.x == 0) grid_arrive(a.counter, n_cta);
  CP_STAMP(threadIdx.x == 0, 9);  // arrived at the grid barrier

  // ---- while the other CTAs arrive: state tails and rows without a window ----
  for (int i = threadIdx.x; i < kinds * p.T && mm_ok; i += kThreads) {
    const int k = i / p.T, t = i % p.T;
    const TokInfo ti = sm.tok[t];
    const bool score = k >= p.coff;
    const int64_t so = score ? ti.sc_off : ti.kv_off;
    if (ti.b < 0 || so < 0) continue;
    const int half = score ? k - p.coff : k;
    const int e = (k * p.T + t) * OWN;
    float4 v = own_value4(&sm.recv[0][e], &sm.recv[1][e], &sm.recv[2][e], &sm.recv[3][e]);
    if (score) v = add4(v, *reinterpret_cast<const float4*>(&sm.ape[half * r + ti.pos % r][0]));
    *reinterpret_cast<float4*>((score ? p.score_state : p.kv_state) + so + half * p.D + ch0) = v;
  }
  for (int n = threadIdx.x; n < n_out; n += kThreads)
    if (sm.win[n].w < 0) *reinterpret_cast<uint2*>(p.out + (int64_t)n * p.D + ch0) = make_uint2(0u, 0u);
  CP_STAMP(threadIdx.x == 0, 10);  // tails written
  if (threadIdx.x == 0) sm.grid_ok = grid_wait(a.counter, sm.bar_target, p.err) ? 1 : 0;
  CP_STAMP(threadIdx.x == 0, 11);  // grid barrier released
  __syncthreads();
  const bool ok = sm.grid_ok != 0 && mm_ok;

  // ---- 4) RMSNorm scale of each window row (its D/4 partials, fixed order), then this CTA's channels ----
  if (ok) {
    const int nq = n_cta / 4;  // float4 per row of partials (<= 32: one per lane)
    const int mine = nw > warp ? (nw - warp + 3) / 4 : 0;  // list entries warp, warp + 4, ...
    for (int u0 = 0; u0 < mine; u0 += 8) {
      float4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int n = sm.wlist[warp + 4 * (u0 + u < mine ? u0 + u : u0)];
        const float* row = a.ss + (int64_t)(blockIdx.x % kReplicas) * rep_stride + (int64_t)n * n_cta;
        v[u] = lane < nq ? __ldcg(reinterpret_cast<const float4*>(row) + lane) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      float t[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) t[u] = (v[u].x + v[u].y) + (v[u].z + v[u].w);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
        for (int u = 0; u < 8; ++u) t[u] += __shfl_xor_sync(0xffffffffu, t[u], o);
      }
      if (lane == 0) {
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (u0 + u < mine) sm.scale[sm.wlist[warp + 4 * (u0 + u)]] = rsqrtf(t[u] / (float)p.D + 1e-6f);
      }
    }
  }
  __syncthreads();
  CP_STAMP(threadIdx.x == 0, 12);  // RMSNorm scales summed
  const bool roped = ch0 >= p.D - p.rope;
  for (int wi = threadIdx.x; wi < nw; wi += kThreads) {
    const int n = sm.wlist[wi];
    float z[OWN] = {0.f, 0.f, 0.f, 0.f};
    if (ok) {
      const float sc = sm.scale[n];
#pragma unroll
      for (int c = 0; c < OWN; ++c) z[c] = sm.ybuf[n][c] * sc * sm.norm[c];
      if (roped) {  // interleaved RoPE: pairs (2j, 2j+1) of the last rope channels
        const float* t = sm.rope[n];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const float ev = z[2 * u], od = z[2 * u + 1];
          z[2 * u] = ev * t[4 * u + 0] - od * t[4 * u + 2];
          z[2 * u + 1] = od * t[4 * u + 1] + ev * t[4 * u + 3];
        }
      }
    }
    __nv_bfloat162 o01 = __floats2bfloat162_rn(z[0], z[1]);
    __nv_bfloat162 o23 = __floats2bfloat162_rn(z[2], z[3]);
    uint2 v;
    v.x = *reinterpret_cast<uint32_t*>(&o01);
    v.y = *reinterpret_cast<uint32_t*>(&o23);
    *reinterpret_cast<uint2*>(p.out + (int64_t)n * p.D + ch0) = v;
  }

  if (threadIdx.x == 0) bulk_wait_read();  // this CTA's outgoing copies have read its blocks
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, tmem_cols);
  }
  if (threadIdx.x == 0 && sm.abort) atomicOr(p.err, kErrTimeout);
  CP_STAMP(threadIdx.x == 0, 13);  // end
}

// x [T, H] as (column in block, row, 64-column block): a box of 64 columns x
// box_rows rows x KPS blocks lands as KPS tiles [block][row][128 B].
bool make_x_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  EncodeTiledFn f = encode_fn();
  if (!f) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)BK, rows, cols / BK};
  const cuuint64_t strides[2] = {cols * 2, (cuuint64_t)BK * 2};
  const cuuint32_t box[3] = {(cuuint32_t)BK, box_rows, (cuuint32_t)KPS};
  const cuuint32_t estr[3] = {1, 1, 1};
  return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Both weight matrices [C, H] as one 5-D tensor: (column in block, row within a
// half, half, matrix, 64-column block), the matrix stride being the distance
// between the two allocations (the lower one first). A box of 64 columns x 16
// rows x coff halves x 2 matrices x KPS blocks lands as KPS A tiles
// [block][matrix][half][16 rows][128 B].
bool make_w_map(CUtensorMap* m, const Params& p, int* kv_first) {
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
  const cuuint32_t box[5] = {(cuuint32_t)BK, (cuuint32_t)GCH, (cuuint32_t)p.coff, 2, (cuuint32_t)KPS};
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
  if (p.T < 1 || p.T > 64 || p.B > kMaxSeqs || p.rotate || p.n_out > kMaxOut || p.rope != 64) return false;
  if (p.coff * p.ratio > kMaxWinRows || p.H % (KQ * KPS * BK) || p.D % GCH || encode_fn() == nullptr)
    return false;
  CUtensorMap w;
  int kv_first = 0;
  if (!make_w_map(&w, p, &kv_first)) return false;  // e.g. wkv and wgate at the same address
  const int dev = current_device();
  if (dev < 64 && g_disabled[dev]) return false;
  const int clusters = p.D / GCH;
  if (kQuantum % (clusters * KQ)) return false;
  const int cap = p.T <= 32 ? max_clusters<32>(g_conf32) : max_clusters<64>(g_conf64);
  return cap >= clusters;
}

size_t decode_cp_workspace(const Params& p) {
  return sizeof(float) * kReplicas * (size_t)(p.n_out > 0 ? p.n_out : 1) * (p.D / OWN);
}

// Launch. If the device refuses the launch form itself (a cooperative launch of
// clusters), the path is disabled on this device and cudaErrorNotSupported is
// returned before anything ran, so that the caller can take another path.
cudaError_t launch_decode_cp(const Params& p, float* ss, void* counter, cudaStream_t s, bool unreachable) {
  const int NT = (p.T + 15) / 16 * 16;
  CUtensorMap mx, mw;
  CpArgs a;
  if (!make_x_map(&mx, p.x, p.T, p.H, (uint32_t)NT) || !make_w_map(&mw, p, &a.kv_first))
    return cudaErrorInvalidValue;
  a.ss = ss;
  a.counter = static_cast<unsigned*>(counter);
  a.bar_extra = unreachable ? kQuantum : 0u;
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
