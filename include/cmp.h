/*
 * cmp.h — C ABI of the B200 streaming KV-cache Compressor.
 *
 * One call compresses every ratio-token window that the call completes into
 * one bf16 row of D channels (DeepSeek-V4 C4A / C4Li / C128A attention):
 *
 *   1. dual projection   kv = x·Wkvᵀ,  score = x·Wgateᵀ + ape[p mod ratio]
 *      ("compressor torch_extension API", 计算公式 1-2; "CANN PyPTO 算子实战:
 *      Compressor", 主要计算过程);
 *   2. per-window pooling: a per-channel softmax over the window's rows weights
 *      a sum of its kv rows; for ratio 4 (coff 2) a window pairs columns [0, D)
 *      of the previous window's 4 rows with columns [D, 2D) of its own 4 rows,
 *      and the first window of a sequence has no previous rows
 *      ("compressor torch_extension API", 计算公式 2-5; "NPU DeepSeek-V4 Ascend C
 *      融合算子优化", Compressor 计算公式; "CANN PyPTO 算子实战", 压缩窗口与状态更新);
 *   3. RMSNorm (eps 1e-6) with norm_weight, interleaved RoPE on the last
 *      rope_head_dim channels, and, if rotate, a product with the D×D hadamard
 *      matrix ("CANN PyPTO 算子实战", 压缩窗口与状态更新, kernel 派发逻辑).
 *
 * Streaming: kv_state / score_state keep, in fp32, the projected rows of
 * windows a later call still has to pool. They are paged: position p of
 * sequence b lives in slot (table[b][p / block_size], p % block_size) of its
 * pool, with kv_block_table for kv_state and state_block_table for
 * score_state ("CANN PyPTO 算子实战", 参数说明; "Triton-Ascend Compressor",
 * state_block_table example). A call reads slots of positions before
 * start_pos[b] and writes slots of positions from start_pos[b] on, so the
 * slots it reads and the slots it writes are disjoint and an identical call
 * repeated gives identical results.
 *
 * Conventions for every entry point below:
 *  - bf16 tensors are passed as cmp_bf16 (their 16-bit patterns);
 *  - all tensors are dense, row-major and contiguous;
 *  - "device" pointers are CUDA device memory of the current device, owned by
 *    the caller (the library never frees or keeps them past the call);
 *  - "host" pointers are ordinary host memory;
 *  - entry points returning int return a cmp_status.
 */
#ifndef CMP_H_
#define CMP_H_

#include <stdbool.h>
#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define CMP_API __attribute__((visibility("default")))
#else
#define CMP_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t cmp_bf16;

typedef enum cmp_status {
  CMP_OK = 0,
  CMP_ERR_NULLPTR = 1,      /* a required pointer is NULL */
  CMP_ERR_INVALID = 2,      /* a size or argument outside the supported range */
  CMP_ERR_UNSUPPORTED = 3,  /* a ratio the library does not implement */
  CMP_ERR_CUDA = 4,         /* a CUDA runtime call or kernel launch failed */
  CMP_ERR_DEVICE_INDEX = 5, /* a kernel met a bad index (see cmp_get_error) */
  CMP_ERR_TIMEOUT = 6       /* a kernel gave up waiting on its own pipeline */
} cmp_status;

/* Shape scalars of one call; the pages' operator reads them from tensor shapes.
 *   B            sequences (requests) in the call, >= 0
 *   T            total tokens = rows of x = cu_seqlens[B], >= 0
 *   H            hidden size: a multiple of 512 in [512, 16384]
 *   D            compressed row width: 128 or 512
 *   block_num    pool rows of kv_state and of score_state, >= 1
 *   block_size   positions per pool row, in [1, 1024]
 *   table_stride columns of kv_block_table and state_block_table, >= 1
 * ("compressor torch_extension API", 约束说明: D in {128, 512}; H a multiple of
 * 512; block_size 1..1024. H down to 512 is accepted for small tests.) */
typedef struct cmp_dims {
  int32_t B;
  int32_t T;
  int32_t H;
  int32_t D;
  int32_t block_num;
  int32_t block_size;
  int32_t table_stride;
} cmp_dims;

/* Rows of out, sin and cos: min(T, T / ratio + B)
 * ("CANN PyPTO 算子实战", 返回值说明: out is [min(T, T//ratio + B), D]).
 * Returns -1 if ratio < 1, B < 0 or T < 0. Host only. */
CMP_API int64_t cmp_out_rows(int64_t B, int64_t T, int32_t ratio);

/* Host-side output-row layout, for callers that build sin/cos per row.
 * Window w of sequence b completes when the token at position (w+1)*ratio - 1
 * arrives ("CANN PyPTO 算子实战", 数值精度与验证要点: (start_pos + i + 1) % ratio == 0).
 * Sequence b reserves cap_b = min(L_b, L_b / ratio + 1) consecutive rows after
 * those of sequences 0..b-1; its k-th completed window goes to the k-th of
 * them. For every row n < n_out: row_seq[n] = b and row_window[n] = w if the
 * row holds window w of sequence b, else row_seq[n] = row_window[n] = -1.
 * cu_seqlens [B+1], start_pos [B] (NULL: all 0), row_seq / row_window
 * [n_out]: host memory. n_out must equal cmp_out_rows(B, cu_seqlens[B], ratio).
 * Errors: CMP_ERR_NULLPTR, CMP_ERR_INVALID (cu_seqlens not rising from 0,
 * start_pos < 0, n_out mismatch, positions past INT32_MAX). */
CMP_API int cmp_out_row_layout(const int32_t* cu_seqlens, const int32_t* start_pos, int32_t B,
                       int32_t ratio, int64_t n_out, int32_t* row_seq, int32_t* row_window);

/* The Compressor ("CANN PyPTO 算子实战", 函数原型 and 参数说明, plus cu_seqlens
 * for packed variable-length input from "compressor torch_extension API").
 *
 *  x                  device bf16 [T, H]; sequence b owns rows
 *                     cu_seqlens[b] .. cu_seqlens[b+1]-1, at absolute positions
 *                     start_pos[b], start_pos[b]+1, ...
 *  kv_state           device fp32 [block_num, block_size, coff*D], updated in place
 *  score_state        device fp32 [block_num, block_size, coff*D], updated in place
 *                     (holds x·Wgateᵀ + ape, as the pooling reads it)
 *  kv_block_table     device int32 [B, table_stride]: pool row of kv_state per block
 *  state_block_table  device int32 [B, table_stride]: pool row of score_state per block
 *                     Entries a call does not need are never read (may be -1).
 *  sin, cos           device bf16 [n_out, rope_head_dim]: RoPE tables of output
 *                     row n; element 2j of a pair uses column j, element 2j+1
 *                     column rope_head_dim/2 + j
 *  wkv, wgate         device bf16 [coff*D, H]
 *  ape                device fp32 [ratio, coff*D]: added to the score of the
 *                     token at position p from row p mod ratio
 *  norm_weight        device bf16 [D]
 *  hadamard           device bf16 [D, D] (out = out @ hadamard); NULL iff !rotate
 *  start_pos          device int32 [B]; NULL means every sequence starts at 0
 *  cu_seqlens         device int32 [B+1], rising from 0 to T
 *  ratio              tokens per window: 1, 2, 4, 8, 16, 32, 64 or 128;
 *                     coff = 2 for ratio 4, else 1 (ratio 1: every token is
 *                     its own window, so only projection and normalisation
 *                     remain, as the Triton-Ascend Compressor article notes)
 *  rope_head_dim      64 (the only value the pages support)
 *  rotate             apply the hadamard product
 *  out                device bf16 [n_out, D], n_out = cmp_out_rows(B, T, ratio);
 *                     every row is written (rows with no window: 0)
 *  stream             cudaStream_t to run on (NULL: the legacy default stream)
 *  dims               host pointer to the shape scalars
 *
 * State update: for sequence b with e = start_pos[b] + L_b, the rows of
 * positions p in [start_pos[b], e) with p >= (e/ratio - coff + 1)*ratio are
 * written to both states — exactly the rows a later call can still read. No
 * other state byte changes.
 *
 * Asynchronous on stream; no host synchronisation. The first call on a
 * (device, stream) pair allocates a workspace that later calls reuse (it grows
 * if a later call needs more); see cmp_workspace_size / cmp_release_workspaces.
 * Results are bitwise reproducible run to run (no floating-point atomics).
 * Requirements the library does not check: the pool rows used by different
 * sequences are disjoint, and the tables map the blocks a call needs (the Python
 * binding's debug_check_tables checks both on the host, for tests and debugging).
 *
 * Returns CMP_OK, CMP_ERR_NULLPTR, CMP_ERR_INVALID, CMP_ERR_UNSUPPORTED or
 * CMP_ERR_CUDA, all decided on the host before anything is launched, except
 * CMP_ERR_CUDA for a failed launch. B == 0 or T == 0 is a successful no-op.
 * Faults found inside kernels (a needed table entry outside [0, block_num) or
 * a block index past table_stride; cu_seqlens not rising from 0 to T;
 * start_pos < 0; positions past INT32_MAX) never trap: the access is skipped,
 * an error word on the device is set, and cmp_get_error reports it. */
CMP_API int cmp_compressor(const cmp_bf16* x, float* kv_state, float* score_state,
                   const int32_t* kv_block_table, const int32_t* state_block_table,
                   const cmp_bf16* sin, const cmp_bf16* cos, const cmp_bf16* wkv,
                   const cmp_bf16* wgate, const float* ape, const cmp_bf16* norm_weight,
                   const cmp_bf16* hadamard, const int32_t* start_pos, const int32_t* cu_seqlens,
                   int32_t ratio, int32_t rope_head_dim, bool rotate, cmp_bf16* out,
                   void* stream, const cmp_dims* dims);

/* No counterpart on the pages: an entry point for callers that must not
 * allocate device memory at call time (for example a serving engine that
 * reserves all device memory at start-up, or a caller running with the GPU
 * nearly full, where a cudaMalloc could fail or synchronise the device).
 *
 * Same arguments and results as cmp_compressor, for decode-sized calls:
 * T <= 64 tokens, and the call's scratch (error word, per-sequence metadata,
 * fp32 projection rows: about 12*B + 8*T*coff*D bytes) must fit a fixed
 * 1 MiB array in device memory that the library image carries; larger calls
 * return CMP_ERR_INVALID before launching anything. It never calls cudaMalloc,
 * cudaFree or any allocating routine.
 *
 * The first call on each device (with that device current) looks up the
 * array's device address once (cudaGetSymbolAddress); make that first call
 * before any stream capture. All calls on a device share the array, so calls
 * that overlap on the GPU race and must be ordered by the caller (one stream,
 * or events). The array keeps the last call's contents. Its error word starts
 * at zero when the library is loaded, kernels only set bits in it, and
 * cmp_get_error reads and clears it: device-side errors (a bad needed table
 * entry, cu_seqlens or start_pos) are reported by cmp_get_error(stream) on the
 * same device, once the calls' stream is synchronised (pass that stream).
 * After a device reset (cudaDeviceReset), call cmp_release_workspaces before
 * the next call: the array may move when the library image is loaded again,
 * and that call makes the next one look its address up afresh. */
CMP_API int cmp_compressor_noalloc(const cmp_bf16* x, float* kv_state, float* score_state,
                                   const int32_t* kv_block_table, const int32_t* state_block_table,
                                   const cmp_bf16* sin, const cmp_bf16* cos, const cmp_bf16* wkv,
                                   const cmp_bf16* wgate, const float* ape, const cmp_bf16* norm_weight,
                                   const cmp_bf16* hadamard, const int32_t* start_pos,
                                   const int32_t* cu_seqlens, int32_t ratio, int32_t rope_head_dim,
                                   bool rotate, cmp_bf16* out, void* stream, const cmp_dims* dims);

/* Synchronises stream, then returns and clears the error word the kernels of
 * the current device set: CMP_OK, CMP_ERR_DEVICE_INDEX or CMP_ERR_TIMEOUT
 * (CMP_ERR_CUDA if the synchronisation itself fails). Covers the calls made on
 * `stream` and every cmp_compressor_noalloc call on the current device. */
CMP_API int cmp_get_error(void* stream);

/* Bytes of device workspace a call with these shapes uses (the two-phase
 * "query the workspace, then run" pattern of the aclnn API on "NsaCompressWithCache").
 * Returns 0 for invalid dims. Host only. */
CMP_API size_t cmp_workspace_size(const cmp_dims* dims, int32_t ratio);

/* Frees every workspace the library holds (synchronises the devices first) and
 * forgets the cached device addresses of cmp_compressor_noalloc's array.
 * Returns CMP_OK or CMP_ERR_CUDA. */
CMP_API int cmp_release_workspaces(void);

/* Static text for a status code. */
CMP_API const char* cmp_status_string(int status);

/* ---- NsaCompressWithCache (a second workload) ------------------------------
 * "CANN ops-transformer 算子解析 NsaCompressWithCache" — 计算公式, 算法流程,
 * 参数说明, 约束说明. For each batch b with s = act_seq_len[b] (per-batch
 * lengths): if s >= compress_block_size and (s - compress_block_size) %
 * compress_stride == 0, then for every head n and channel d
 *   output_cache[slot_mapping[b], n, d] =
 *     round(sum_{j < compress_block_size} input[token s - compress_block_size + j of b, n, d] * weight[j, n])
 * with the products and the sum in fp32 and one round-to-nearest-even cast to
 * the cache dtype. Other slots are not touched. */
typedef struct {
  int64_t B;             /* batches: entries of slot_mapping and act_seq_len, at most 65535 */
  int64_t N;             /* heads, 1..64 (even when above 50) */
  int64_t D;             /* channels per head, a multiple of 16, at most 256 */
  int64_t tokens;        /* paged: block_num (input rows / page_block_size); packed: T, the input rows;
                            input rows at most INT32_MAX */
  int64_t table_stride;  /* paged: columns of block_table (pages per batch); packed: ignored */
  int64_t result_len;    /* rows of output_cache */
} cmp_nsa_dims;

enum { CMP_NSA_FP16 = 0, CMP_NSA_BF16 = 1 };
enum { CMP_NSA_PAGED = 0, CMP_NSA_PACKED = 1 };

/* input: device, dtype elements, paged [block_num, page_block_size, N, D]
 *   (a token at position p of batch b is at block block_table[b][p /
 *   page_block_size], row p % page_block_size) or packed [T, N, D] (batch b's
 *   tokens follow those of batches < b, in order); 16-byte aligned.
 * weight: device [compress_block_size, N], same dtype. slot_mapping: device
 * int32 [B], distinct values in [0, result_len). act_seq_len: device int64 [B].
 * block_table: device int32 [B, table_stride] (paged; NULL allowed when packed).
 * output_cache: device [result_len, N, D], same dtype, updated in place;
 * 16-byte aligned. The call is asynchronous on `stream` (a cudaStream_t, NULL =
 * default stream). It keeps its error word, and for the packed layout the B
 * batches' first rows (8 * B bytes), in the library's workspace for this device
 * and stream. Growing that workspace synchronises the device, so make the
 * largest call once before capturing calls into a CUDA graph, as for
 * cmp_compressor. All other memory is the caller's.
 * compress_block_size: a multiple of 16 in [16, 64], >= compress_stride;
 * compress_stride: 16, 32, 48 or 64; page_block_size: 64 or 128 (paged).
 * Returns CMP_OK, CMP_ERR_NULLPTR (a required pointer or dims is NULL),
 * CMP_ERR_INVALID (a size or alignment outside the ranges above),
 * CMP_ERR_UNSUPPORTED (dtype or layout value), CMP_ERR_CUDA (launch, or the driver
 * cannot describe the cache as a TMA tensor). B == 0
 * is a no-op. A slot outside [0, result_len), a needed table entry outside
 * [0, block_num) or packed rows past T set the device error word (the batch is
 * skipped; cmp_get_error reports CMP_ERR_DEVICE_INDEX). */
CMP_API int cmp_nsa_compress(const void* input, const void* weight, const int32_t* slot_mapping,
                             const int64_t* act_seq_len, const int32_t* block_table, int32_t layout,
                             int32_t dtype, int64_t compress_block_size, int64_t compress_stride,
                             int64_t page_block_size, void* output_cache, void* stream,
                             const cmp_nsa_dims* dims);

/* ---- measurement --------------------------------------------------------
 * Kernels of the library, by id: */
enum {
  CMP_KERNEL_SCHED = 0,        /* varlen scheduler */
  CMP_KERNEL_PROJ_TC = 1,      /* prefill projection, tcgen05 / TMEM / TMA */
  CMP_KERNEL_PROJ_MMA = 2,     /* projection, warp-level mma.sync */
  CMP_KERNEL_PROJ_DECODE = 3,  /* small-T projection streaming the weights */
  CMP_KERNEL_POOL = 4,         /* pooling + RMSNorm + RoPE + Hadamard + store */
  CMP_KERNEL_FUSED = 5,        /* prefill projection with the pooling in its epilogue */
  CMP_KERNEL_FINISH = 6,       /* fused path: merge halves + RMSNorm + RoPE + Hadamard */
  CMP_KERNEL_DECODE_FUSED = 7, /* decode (T <= 64) in one cooperative kernel, K-split grid */
  CMP_KERNEL_DECODE_CP = 8,    /* decode (T <= 64) in one cooperative kernel of 4-CTA clusters
                                  that each own 16 channels */
  CMP_KERNEL_NSA = 9,          /* NsaCompressWithCache */
  CMP_KERNEL_NSA_SCAN = 10,    /* NsaCompressWithCache, packed layout: each batch's first row */
  CMP_KERNEL_COUNT = 11
};

/* Name of a kernel id (NULL if out of range). */
CMP_API const char* cmp_kernel_name(int kernel);

/* Total kernels this library has launched in this process (all devices). */
CMP_API int64_t cmp_launch_count(void);

/* Start per-kernel timing: every launch from now on is bracketed by CUDA
 * events on its stream. Clears earlier totals. Returns CMP_OK or CMP_ERR_CUDA. */
CMP_API int cmp_profile_start(void);

/* Stop timing; synchronise the recorded events and write, per kernel id, the
 * summed milliseconds and launch count into ms[CMP_KERNEL_COUNT] and
 * launches[CMP_KERNEL_COUNT] (host arrays; either may be NULL). */
CMP_API int cmp_profile_stop(double* ms, int64_t* launches);

/* Measurement hook of a library built with -DCMP_PHASE_STAMPS (bench.py
 * --only decode-phases builds one beside the normal library and runs it): the
 * channel-group decode kernel writes the global timer (ns) at up to 32 points
 * of its timeline; this copies those of its last launch, CTA i's phase k at
 * dst[i * 32 + k] for the first n entries (host array, n <= 512 * 32), after
 * synchronising the device. Phases: 0 entry, 1 set-up done, 2 first weight
 * stage landed, 3 last MMA issued, 4 metadata done, 5 partials sent,
 * 6 partials received, 7 pooled and arrived, 9 exchange complete, 10 rows
 * stored, 11 all CTAs arrived, 14 tails written, 15 end; 16-19 the metadata's
 * first wave, window list, second and third wave. Other builds return
 * CMP_ERR_UNSUPPORTED. */
CMP_API int cmp_debug_phase_stamps(uint64_t* dst, int64_t n);

/* Testing knob: which path calls take. 0 = automatic (for T <= 64 the
 * channel-group decode kernel, or without it (rotate, or a device that cannot
 * hold its clusters) the weight-streaming projection + pooling kernels, else
 * the K-split one-kernel decode; the fused tcgen05 pooling kernel for long
 * sequences, T >= 1024 and T >= 256*B, when its (T/256)*(C/128) work items
 * fill the SMs twice; else the tcgen05 projection + pooling kernel), 1 = force the mma.sync projection, 2 = the tcgen05 projection
 * (on CTA pairs, cta_group::2, where the device can co-schedule them),
 * 3 = weight streaming, 4 = the fused path, 5 = the K-split one-kernel decode,
 * 6 = the channel-group decode, 7 = the tcgen05 projection on single CTAs,
 * 8 = the fused path on single CTAs (4 runs on CTA pairs, cta_group::2, when
 * coff * D / 128 is even and the device co-schedules them).
 * A forced path a call cannot take falls back to 1.
 * Returns the previous value, or -1 if out of range. */
CMP_API int cmp_set_proj_kernel(int which);

/* Testing knob for failure detection: the next `launches` launches of the
 * channel-group decode kernel (CMP_KERNEL_DECODE_CP) wait for the other
 * clusters' exchange words of an epoch that no cluster publishes. Each CTA's
 * bounded wait gives up after about one second, the rows of the call come out
 * as zeros, the CTAs free their tensor memory and return, and cmp_get_error
 * then reports CMP_ERR_TIMEOUT and resets the exchange words, so the next call
 * runs normally. Nothing faults or hangs. Returns the previous count, or -1 if
 * launches < 0. */
CMP_API int cmp_debug_unreachable_barrier(int launches);

#ifdef __cplusplus
}
#endif

#endif /* CMP_H_ */
