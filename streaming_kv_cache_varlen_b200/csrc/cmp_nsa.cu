// NsaCompressWithCache: for each batch whose length just reached a compression
// step, the weighted sum of its last compress_block_size cached tokens, written
// to its slot of the output cache ("CANN ops-transformer 算子解析
// NsaCompressWithCache", 计算公式 and 算法流程: trigger s >= compress_block_size
// and (s - compress_block_size) % stride == 0; tokens s - compress_block_size
// .. s - 1 found through the block table (paged) or packed by batch (TND);
// values cast to fp32, multiplied by weight[j, n], summed, cast back to
// fp16 / bf16 with round-to-nearest-even).
//
// HBM bound: every byte of the window's tokens is read once. One CTA per (group
// of nh heads, batch). The window starts at a multiple of 16 tokens and pages
// hold a multiple of 16, so it is cbs / 16 runs of 16 consecutive cache rows,
// each inside one page: each run is ONE TMA box {D, nh heads, 16 rows} of a 3-D
// map over the cache [rows, N, D], a few large copies per CTA instead of one
// per token and chunk (per-copy overhead in the copy engine, not DRAM, limited
// the version with small copies).
//
// A CTA holds its whole window in shared memory (all runs in flight at once)
// unless that would leave part of the grid for a second wave: then it cycles
// its runs through a ring of fewer buffers, so that every CTA is resident from
// the start and the GPU's whole shared memory streams the windows.
#include "cmp_internal.cuh"
#include "cmp_sm100.cuh"

#include <cuda_fp16.h>

namespace cmp {

namespace {

constexpr int kThreads = 128;
constexpr int kRun = 16;                 // cache rows per TMA box
constexpr int kMaxRuns = 64 / kRun;      // compress_block_size <= 64
constexpr int kTargetBytes = 32 << 10;   // window bytes per CTA the head group aims at
constexpr int kCtasPerSm = 16;           // resident CTAs of kThreads (2048 threads; __launch_bounds__)
constexpr int64_t kSmemPerSm = 228 << 10;  // shared memory of one SM
constexpr int64_t kSmemPerCta = 1 << 10;   // reserved by the system for every resident CTA

template <bool BF16>
__device__ __forceinline__ float to_f32(uint16_t v) {
  return BF16 ? __uint_as_float((uint32_t)v << 16) : __half2float(__ushort_as_half(v));
}

template <bool BF16>
__device__ __forceinline__ uint32_t pack(float lo, float hi) {
  if (BF16) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&h);
  }
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Adds tokens [j0, j1) of the window to a thread's 4 sums: element e (of head
// group-relative head hh) of token j is at w[(j - j0) * per_tok + e].
template <bool BF16>
__device__ __forceinline__ void add_tokens(const uint16_t* w, const float* wsm, int j0, int j1, int per_tok,
                                           int nh, int e, int hh, float (&a)[4]) {
  for (int j = j0; j < j1; ++j) {
    const uint2 v = *reinterpret_cast<const uint2*>(w + (size_t)(j - j0) * per_tok + e);
    const float wt = wsm[j * nh + hh];
    a[0] = fmaf(to_f32<BF16>((uint16_t)(v.x & 0xFFFFu)), wt, a[0]);
    a[1] = fmaf(to_f32<BF16>((uint16_t)(v.x >> 16)), wt, a[1]);
    a[2] = fmaf(to_f32<BF16>((uint16_t)(v.y & 0xFFFFu)), wt, a[2]);
    a[3] = fmaf(to_f32<BF16>((uint16_t)(v.y >> 16)), wt, a[3]);
  }
}

template <bool BF16>
__device__ __forceinline__ void store4(uint16_t* dst, const float (&a)[4]) {
  uint2 o;
  o.x = pack<BF16>(a[0], a[1]);
  o.y = pack<BF16>(a[2], a[3]);
  *reinterpret_cast<uint2*>(dst) = o;
}

// Warp 0 validates the batch's slot and the cache rows of its window, then lane
// 0 issues the first nbuf of the window's cbs / 16 boxes (heads h0 .. h0 + nh -
// 1; heads past N read as zeros and are not stored), box k on mbarrier k; the
// other threads stage the weights meanwhile. Then each thread sums 4
// consecutive elements of one head over the window's tokens in order and
// stores them. nbuf = cbs / 16: the whole window is resident. nbuf < cbs / 16
// (the host chooses it only when nh * D <= 4 * kThreads, one element group per
// thread): box r lands in buffer r mod nbuf; once every thread has added it,
// thread 0 issues box r + nbuf into the same buffer. A wait that gives up (2 s)
// raises kErrTimeout, and thread 0 waits at most 20 ms more for the boxes it
// armed, so that no copy is still landing when the CTA leaves.
// Packed layout (a programmatic dependent of nsa_scan_kernel): only lane 0 waits
// for the scan, and every thread's stores come after it through __syncthreads.
template <bool BF16>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    nsa_kernel(const __grid_constant__ CUtensorMap map, NsaParams p, int nh, int page_shift, int nbuf) {
  const int b = blockIdx.y;
  const int h0 = blockIdx.x * nh;
  const int lane = threadIdx.x & 31;
  // paged, table rows of at most 32 pages: warp 0 loads the batch's whole row
  // together with its length and slot, so the entries are at hand when the
  // window is known (one round trip instead of two)
  const bool row_in_warp = !p.packed && p.table_stride <= 32;
  const int32_t* trow = p.table + (int64_t)b * p.table_stride;
  int32_t tpre = -1;
  if (threadIdx.x < 32 && row_in_warp && lane < p.table_stride) tpre = __ldg(trow + lane);
  const int slot = threadIdx.x == 0 ? __ldg(p.slot + b) : 0;
  const int64_t s = __ldg(p.len + b);
  if (s < p.cbs || (s - p.cbs) % p.stride != 0) return;  // not a compression step (whole CTA)
  extern __shared__ __align__(128) unsigned char smem_raw[];
  // TMA destinations start on 128-byte boundaries (the runs are multiples of 512 B)
  uint16_t* buf = reinterpret_cast<uint16_t*>(smem_raw + ((128u - (sm100::smem_u32(smem_raw) & 127u)) & 127u));
  const int per_tok = nh * p.D;
  const int runs = p.cbs / kRun;
  const uint32_t run_bytes = (uint32_t)(kRun * per_tok * 2);
  float* wsm = reinterpret_cast<float*>(buf + (size_t)nbuf * kRun * per_tok);  // [cbs][nh]
  __shared__ __align__(8) uint64_t full[kMaxRuns];
  __shared__ int ok;
  int64_t row[kMaxRuns];  // first cache row of each box (thread 0 issues them all)
  sm100::Armed armed;     // thread 0: the last phase it armed on each buffer
  if (threadIdx.x < 32) {  // warp 0: validation; lane 0 issues the copies
    const int64_t first = s - p.cbs;
    bool good = slot >= 0 && slot < p.result_len;
    if (p.packed) {
      if (lane == 0) {
        pdl_wait();  // the row starts come from nsa_scan_kernel, launched just before
        const int64_t start = p.starts[b];
        good = good && start >= 0 && start + s <= p.tokens;
        for (int k = 0; k < runs; ++k) row[k] = start + first + k * kRun;
      }
    } else {
      const int64_t mask = (int64_t(1) << page_shift) - 1;
      for (int k = 0; k < runs; ++k) {
        const int64_t pos = first + k * kRun;
        const int64_t pg = pos >> page_shift;
        int32_t blk;
        if (row_in_warp) {  // uniform across the warp: every lane shuffles
          const int32_t v = __shfl_sync(0xffffffffu, tpre, (int)(pg & 31));
          blk = pg < p.table_stride ? v : -1;
        } else {
          blk = lane == 0 && pg < p.table_stride ? __ldg(trow + pg) : -1;
        }
        good = good && blk >= 0 && blk < p.tokens;
        row[k] = ((int64_t)blk << page_shift) + (pos & mask);
      }
    }
    if (lane == 0) {
      if (!good) atomicOr(p.err, kErrIndex);
      ok = good ? 1 : 0;
      if (good) {
        sm100::prefetch_tmap(&map);
        for (int k = 0; k < nbuf; ++k) sm100::mbar_init(&full[k], 1);
        sm100::fence_barrier_init();
        for (int k = 0; k < nbuf; ++k) {
          sm100::mbar_arrive_expect_tx(&full[k], run_bytes);
          sm100::tma_load_3d(buf + (size_t)k * kRun * per_tok, &map, &full[k], 0, h0, (int)row[k]);
          armed.note(k, 0);
        }
      }
    }
  }
  for (int i = threadIdx.x; i < p.cbs * nh; i += kThreads) {
    const int j = i / nh, h = h0 + i % nh;
    wsm[i] = h < p.N ? to_f32<BF16>(__ldg(p.weight + j * p.N + h)) : 0.f;
  }
  __syncthreads();
  if (!ok) return;
  int never = 0;
  const int live = (p.N - h0 < nh ? p.N - h0 : nh) * p.D;  // elements of heads < N
  uint16_t* dst = p.out + (int64_t)__ldg(p.slot + b) * p.N * p.D + (int64_t)h0 * p.D;
  if (nbuf == runs) {  // the whole window is resident
    for (int k = 0; k < runs; ++k) {
      if (!sm100::mbar_wait(&full[k], 0, &never)) {
        if (threadIdx.x == 0) {  // no copy may still be landing when the CTA leaves
          atomicOr(p.err, kErrTimeout);
          sm100::drain_armed(full, nbuf, armed);
        }
        return;
      }
    }
    for (int e = threadIdx.x * 4; e < live; e += kThreads * 4) {
      float a[4] = {0.f, 0.f, 0.f, 0.f};
      add_tokens<BF16>(buf, wsm, 0, p.cbs, per_tok, nh, e, e / p.D, a);
      store4<BF16>(dst + e, a);
    }
    return;
  }
  const int e = threadIdx.x * 4;  // live <= 4 * kThreads here
  const bool mine = e < live;
  float a[4] = {0.f, 0.f, 0.f, 0.f};
  for (int r = 0; r < runs; ++r) {
    const int k = r % nbuf;
    const bool landed = sm100::mbar_wait(&full[k], (uint32_t)(r / nbuf) & 1u, &never);
    if (landed && mine) add_tokens<BF16>(buf + (size_t)k * kRun * per_tok, wsm, r * kRun, r * kRun + kRun, per_tok,
                                         nh, e, e / p.D, a);
    if (__syncthreads_or(!landed)) {  // buffer k is free again, unless a wait gave up
      if (threadIdx.x == 0) {  // no copy may still be landing when the CTA leaves
        atomicOr(p.err, kErrTimeout);
        sm100::drain_armed(full, nbuf, armed);
      }
      return;
    }
    if (threadIdx.x == 0 && r + nbuf < runs) {
      sm100::mbar_arrive_expect_tx(&full[k], run_bytes);
      sm100::tma_load_3d(buf + (size_t)k * kRun * per_tok, &map, &full[k], 0, h0, (int)row[r + nbuf]);
      armed.note(k, (uint32_t)((r + nbuf) / nbuf));
    }
  }
  if (mine) store4<BF16>(dst + e, a);
}

// Packed layout: the first row of every batch, starts[b] = sum of the lengths of
// batches before b (-1 if one of them is negative), by one CTA: each thread sums
// a contiguous chunk of up to 64 lengths, the chunk totals are scanned across
// the block, and each thread then writes its chunk's starts.
constexpr int kScanThreads = 1024;

__global__ void __launch_bounds__(kScanThreads) nsa_scan_kernel(const int64_t* len, int B, int64_t* starts) {
  pdl_trigger();  // the main kernel may be scheduled now; it waits for this grid to finish
  __shared__ int64_t w_sum[kScanThreads / 32];
  __shared__ int w_neg[kScanThreads / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int per = (B + kScanThreads - 1) / kScanThreads;
  const int i0 = threadIdx.x * per, i1 = i0 + per < B ? i0 + per : B;
  int64_t sum = 0;
  int neg = 0;
  for (int i = i0; i < i1; ++i) {
    const int64_t li = __ldg(len + i);
    sum += li > 0 ? li : 0;
    neg |= li < 0;
  }
  int64_t inc = sum;  // inclusive scan over the warp
  int ineg = neg;
  for (int o = 1; o < 32; o <<= 1) {
    const int64_t t = __shfl_up_sync(0xffffffffu, inc, o);
    const int n = __shfl_up_sync(0xffffffffu, ineg, o);
    if (lane >= o) {
      inc += t;
      ineg |= n;
    }
  }
  if (lane == 31) {
    w_sum[warp] = inc;
    w_neg[warp] = ineg;
  }
  __syncthreads();
  if (warp == 0) {  // inclusive scan of the warp totals
    int64_t v = w_sum[lane];
    int n = w_neg[lane];
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t t = __shfl_up_sync(0xffffffffu, v, o);
      const int m = __shfl_up_sync(0xffffffffu, n, o);
      if (lane >= o) {
        v += t;
        n |= m;
      }
    }
    w_sum[lane] = v;
    w_neg[lane] = n;
  }
  __syncthreads();
  int64_t run = __shfl_up_sync(0xffffffffu, inc, 1);  // exclusive within the warp
  int nrun = __shfl_up_sync(0xffffffffu, ineg, 1);
  if (lane == 0) {
    run = 0;
    nrun = 0;
  }
  if (warp > 0) {
    run += w_sum[warp - 1];
    nrun |= w_neg[warp - 1];
  }
  for (int i = i0; i < i1; ++i) {
    starts[i] = nrun ? -1 : run;
    const int64_t li = __ldg(len + i);
    run += li > 0 ? li : 0;
    nrun |= li < 0;
  }
}

// The cache as a 3-D tensor (d, head, row) with a box of {D, nh, 16}.
bool make_cache_map(CUtensorMap* m, const NsaParams& p, int64_t rows, int nh) {
  sm100::EncodeTiledFn f = sm100::encode_fn();
  if (!f) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)p.D, (cuuint64_t)p.N, (cuuint64_t)rows};
  const cuuint64_t strides[2] = {(cuuint64_t)p.D * 2, (cuuint64_t)p.N * p.D * 2};
  const cuuint32_t box[3] = {(cuuint32_t)p.D, (cuuint32_t)nh, (cuuint32_t)kRun};
  const cuuint32_t estr[3] = {1, 1, 1};
  return f(m, p.bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
           const_cast<uint16_t*>(p.input), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
           CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int g_nsa_conf[2][64] = {{0}, {0}};
int g_nsa_carve[2][64] = {{0}, {0}};

}  // namespace

cudaError_t launch_nsa(const NsaParams& p, cudaStream_t s, int sm_count) {
  const int head_bytes = p.cbs * p.D * 2;  // one head of the window
  int nh = kTargetBytes / head_bytes;
  nh = nh < 1 ? 1 : (nh > p.N ? p.N : nh);
  CUtensorMap map;
  if (!make_cache_map(&map, p, p.packed ? p.tokens : p.tokens * p.pbs, nh)) return cudaErrorNotSupported;
  const int page_shift = p.packed ? 0 : (p.pbs == 64 ? 6 : 7);
  const dim3 grid((unsigned)((p.N + nh - 1) / nh), (unsigned)p.B);
  // Buffers of 16 cache rows per CTA: all cbs / 16 of them, unless the grid's
  // whole windows do not fit on the GPU at once while a ring of fewer would
  // (then the largest such ring: one wave, every CTA resident from the start).
  const int runs = p.cbs / kRun;
  const int64_t run_smem = (int64_t)kRun * nh * p.D * 2;
  auto cta_smem = [&](int nb) { return 128 + nb * run_smem + (int64_t)p.cbs * nh * 4; };  // + alignment slack
  const int64_t sms = sm_count > 0 ? sm_count : 1;
  const int64_t per_sm = ((int64_t)grid.x * grid.y + sms - 1) / sms;
  auto one_wave = [&](int nb) { return per_sm * (cta_smem(nb) + kSmemPerCta) <= kSmemPerSm; };
  int nbuf = runs;
  if (runs > 1 && nh * p.D <= 4 * kThreads && per_sm <= kCtasPerSm && !one_wave(runs)) {
    int nb = runs - 1;
    while (nb >= 1 && !one_wave(nb)) --nb;
    if (nb >= 1) nbuf = nb;
  }
  const size_t smem = (size_t)cta_smem(nbuf);
  // the attribute is raised once per device, to the largest size a call can
  // ask for (window bytes <= kTargetBytes unless one head is larger: cbs <= 64,
  // D <= 256 gives 32 KB)
  constexpr size_t kMaxSmem = (size_t)kTargetBytes + kTargetBytes / 2 + 64 * 64 * 4;
  auto* kernel = p.bf16 ? nsa_kernel<true> : nsa_kernel<false>;
  cudaError_t e = smem_attr_once(kernel, kMaxSmem, g_nsa_conf[p.bf16 ? 1 : 0]);
  int dev = 0;
  if (e == cudaSuccess) e = cudaGetDevice(&dev);
  if (e == cudaSuccess && dev < 64 && !g_nsa_carve[p.bf16 ? 1 : 0][dev]) {
    // the most shared memory per SM: the residency counted above relies on it
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             (int)cudaSharedmemCarveoutMaxShared);
    g_nsa_carve[p.bf16 ? 1 : 0][dev] = e == cudaSuccess;
  }
  if (e != cudaSuccess) return e;
  if (p.packed)  // a programmatic dependent of nsa_scan_kernel
    return launch_chained(kernel, grid, dim3(kThreads), smem, s, 1, map, p, nh, page_shift, nbuf);
  kernel<<<grid, kThreads, smem, s>>>(map, p, nh, page_shift, nbuf);
  return cudaGetLastError();
}

cudaError_t launch_nsa_scan(const NsaParams& p, cudaStream_t s) {
  nsa_scan_kernel<<<1, kScanThreads, 0, s>>>(p.len, p.B, p.starts);
  return cudaGetLastError();
}

}  // namespace cmp
