// cmp_compressor_noalloc: the decode-sized Compressor call (T <= 64 tokens)
// with no device allocation at all.
//
// Who needs it: callers that must not allocate device memory while they run.
// A serving engine that reserves all of its device memory at start-up and
// treats any later cudaMalloc as a bug, a caller that already holds the GPU
// close to full and cannot risk an allocation failing mid-step, or code on a
// latency-critical path where cudaMalloc / cudaFree may synchronise the device.
// The regular cmp_compressor allocates a per-(device, stream) workspace on its
// first call; this variant keeps its scratch (the error word, the per-sequence
// metadata and the fp32 projection rows) in one fixed 1 MiB array in device
// memory that is part of the library image, so the loader reserves it when the
// library is loaded and every GPU that loads the library holds it until exit.
//
// The host cannot pass the array's name to a kernel: in host code it is a
// host-side stand-in, not a device address. So on the first call on each
// device (with that device current) the address is looked up once with
// cudaGetSymbolAddress and cached; make that first call before any stream
// capture. Every call on a device shares the array: calls that overlap on the
// GPU (two streams at once) race on it and must be ordered by the caller. The
// array keeps the last call's contents. The only part that must start at zero
// is the error word at its start: it is zero when the library is loaded, the
// kernels only ever set bits in it, and cmp_get_error reads and clears it, so
// device-side errors of these calls are reported like those of cmp_compressor.
// A device reset (cudaDeviceReset) unloads the library image from the device and
// may move the array when it is loaded again: cmp_release_workspaces forgets
// the cached addresses, so the next call looks the address up afresh.
#include <mutex>

#include "cmp_internal.cuh"

namespace cmp {
cudaError_t launch_proj_decode(const Params& p, cudaStream_t s);
bool proj_decode_supported(const Params& p);
int noalloc_take_error(int dev, unsigned* word);
void noalloc_forget_addresses();
}  // namespace cmp

namespace {

constexpr size_t kScratchBytes = size_t(1) << 20;
constexpr int kMaxTokens = 64;  // the decode projection kernel's limit

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

struct ScratchLayout {
  size_t err, m_cu, m_s, m_off, had, proj, total;
};

ScratchLayout scratch_layout(int64_t B, int64_t T, int64_t C) {
  ScratchLayout L{};
  size_t o = 0;
  auto take = [&](size_t n) {
    const size_t r = o;
    o += (n + 255) & ~size_t(255);
    return r;
  };
  L.err = take(16);  // offset 0: the error word (cmp::noalloc_take_error reads it there)
  L.m_cu = take(sizeof(int32_t) * (B + 1));
  L.m_s = take(sizeof(int32_t) * (B > 0 ? B : 1));
  L.m_off = take(sizeof(int32_t) * (B + 1));
  L.had = take(sizeof(int32_t) * 16);  // the scheduler's verdicts on the hadamard matrix
  L.proj = take(sizeof(float) * (size_t)T * 2 * C);
  L.total = o;
  return L;
}

std::mutex g_mu;
unsigned char* g_addr[64] = {nullptr};  // device address of the array, per device

// Set-up, once per device, with that device current.
int scratch_address(unsigned char** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return CMP_ERR_CUDA;
  if (dev < 0 || dev >= 64) return CMP_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return CMP_ERR_CUDA;
    g_addr[dev] = static_cast<unsigned char*>(p);
  }
  *out = g_addr[dev];
  return CMP_OK;
}

bool ratio_ok(int r) { return r == 1 || r == 2 || r == 4 || r == 8 || r == 16 || r == 32 || r == 64 || r == 128; }

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

namespace cmp {

// The error word of this entry point's calls on device `dev` (current), read
// and cleared; 0 if no call has run on that device. The caller has synchronised
// the stream the calls ran on.
int noalloc_take_error(int dev, unsigned* word) {
  *word = 0;
  if (dev < 0 || dev >= 64) return CMP_OK;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_addr[dev]) return CMP_OK;
  unsigned v = 0;
  if (cudaMemcpy(&v, g_addr[dev], sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return CMP_ERR_CUDA;
  if (v && cudaMemset(g_addr[dev], 0, sizeof(v)) != cudaSuccess) return CMP_ERR_CUDA;
  *word = v;
  return CMP_OK;
}

void noalloc_forget_addresses() {
  std::lock_guard<std::mutex> lk(g_mu);
  for (auto& a : g_addr) a = nullptr;
}

}  // namespace cmp

extern "C" int cmp_compressor_noalloc(const cmp_bf16* x, float* kv_state, float* score_state,
                                      const int32_t* kv_block_table, const int32_t* state_block_table,
                                      const cmp_bf16* sin, const cmp_bf16* cos, const cmp_bf16* wkv,
                                      const cmp_bf16* wgate, const float* ape, const cmp_bf16* norm_weight,
                                      const cmp_bf16* hadamard, const int32_t* start_pos,
                                      const int32_t* cu_seqlens, int32_t ratio, int32_t rope_head_dim,
                                      bool rotate, cmp_bf16* out, void* stream, const cmp_dims* dims) {
  if (!dims) return CMP_ERR_NULLPTR;
  if (!ratio_ok(ratio)) return CMP_ERR_UNSUPPORTED;
  const cmp_dims& d = *dims;
  if (d.B < 0 || d.T < 0 || (d.D != 128 && d.D != 512) || d.H < 512 || d.H > 16384 || d.H % 512 ||
      d.block_size < 1 || d.block_size > 1024 || d.block_num < 1 || d.table_stride < 1 ||
      rope_head_dim != 64)
    return CMP_ERR_INVALID;
  if (d.B == 0 && d.T != 0) return CMP_ERR_INVALID;
  if (d.B == 0 || d.T == 0) return CMP_OK;
  if (d.T > kMaxTokens) return CMP_ERR_INVALID;  // beyond what the fixed scratch serves
  const int coff = ratio == 4 ? 2 : 1;
  const ScratchLayout L = scratch_layout(d.B, d.T, (int64_t)coff * d.D);
  if (L.total > kScratchBytes) return CMP_ERR_INVALID;  // too many sequences for the scratch
  if (!x || !kv_state || !score_state || !kv_block_table || !state_block_table || !sin || !cos ||
      !wkv || !wgate || !ape || !norm_weight || !cu_seqlens || !out || (rotate && !hadamard))
    return CMP_ERR_NULLPTR;
  if (!aligned(x, 16) || !aligned(wkv, 16) || !aligned(wgate, 16) || !aligned(kv_state, 16) ||
      !aligned(score_state, 16) || !aligned(ape, 16) || !aligned(out, 8) || !aligned(norm_weight, 8) ||
      !aligned(sin, 4) || !aligned(cos, 4) || (rotate && !aligned(hadamard, 8)) ||
      !aligned(kv_block_table, 4) || !aligned(state_block_table, 4) || !aligned(cu_seqlens, 4) ||
      (start_pos && !aligned(start_pos, 4)))
    return CMP_ERR_INVALID;

  cmp::Params p{};
  p.x = reinterpret_cast<const __nv_bfloat16*>(x);
  p.kv_state = kv_state;
  p.score_state = score_state;
  p.kv_tbl = kv_block_table;
  p.sc_tbl = state_block_table;
  p.sin = reinterpret_cast<const __nv_bfloat16*>(sin);
  p.cos = reinterpret_cast<const __nv_bfloat16*>(cos);
  p.wkv = reinterpret_cast<const __nv_bfloat16*>(wkv);
  p.wgate = reinterpret_cast<const __nv_bfloat16*>(wgate);
  p.ape = ape;
  p.norm_w = reinterpret_cast<const __nv_bfloat16*>(norm_weight);
  p.had = rotate ? reinterpret_cast<const __nv_bfloat16*>(hadamard) : nullptr;
  p.start_pos = start_pos;
  p.cu_in = cu_seqlens;
  p.out = reinterpret_cast<__nv_bfloat16*>(out);
  p.B = d.B;
  p.T = d.T;
  p.H = d.H;
  p.D = d.D;
  p.C = coff * d.D;
  p.coff = coff;
  p.ratio = ratio;
  p.rope = rope_head_dim;
  p.rotate = rotate ? 1 : 0;
  p.block_num = d.block_num;
  p.bs = d.block_size;
  p.stride = d.table_stride;
  p.n_out = d.T < d.T / ratio + d.B ? d.T : d.T / ratio + d.B;
  if (!cmp::proj_decode_supported(p)) return CMP_ERR_UNSUPPORTED;

  unsigned char* ws = nullptr;
  const int rc = scratch_address(&ws);
  if (rc != CMP_OK) return rc;
  p.err = reinterpret_cast<unsigned*>(ws + L.err);
  p.m_cu = reinterpret_cast<int32_t*>(ws + L.m_cu);
  p.m_s = reinterpret_cast<int32_t*>(ws + L.m_s);
  p.m_off = reinterpret_cast<int32_t*>(ws + L.m_off);
  p.proj = reinterpret_cast<float*>(ws + L.proj);
  p.had_sylv = p.rotate ? reinterpret_cast<int32_t*>(ws + L.had) : nullptr;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cmp::launch_sched(p, s) != cudaSuccess) return CMP_ERR_CUDA;
  if (cmp::launch_proj_decode(p, s) != cudaSuccess) return CMP_ERR_CUDA;
  if (cmp::launch_pool(p, s) != cudaSuccess) return CMP_ERR_CUDA;
  return CMP_OK;
}
