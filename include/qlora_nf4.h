/*
 * qlora_nf4.h -- C ABI of the B200 (sm_100a) QLoRA NF4 library.
 *
 * The library implements one data path from the QLoRA pages: blockwise NF4 quantization of a frozen
 * weight with double quantization of its block constants, dequantization, and the QLoRA linear layer
 * (forward and backward) that consumes the quantized weight.
 *
 * Sources (pages by title and section):
 *   [PEFT]  PEFT page, zerotofrontier.app/sft/peft:
 *           "Block-wise quantization in one page", "NF4, derived from normal quantiles",
 *           "Double quantization", "Paged optimizers, and QLoRA end to end", "The real way".
 *   [EXPL]  QLoRA explainer, prism.theerrors.in ("QLoRA: Efficient Finetuning of Quantized LLMs"):
 *           "For the curious", "Putting it together".
 *
 * Conventions for every call:
 *   - All tensor pointers are DEVICE pointers unless a parameter says "host". The caller owns and
 *     allocates every buffer; the library never allocates device memory and keeps no per-call state
 *     (the one exception is qlora_paged_alloc, which allocates managed memory on request).
 *     Its only state is a constant-memory codebook and one status word per device.
 *   - Every device pointer must be 16-byte aligned (QLORA_ERR_ALIGNMENT otherwise).
 *   - Layouts are row-major and dense. bf16 tensors are passed as `const void*`/`void*`.
 *   - Calls are asynchronous on `stream` (NULL = legacy default stream) and return after enqueueing.
 *     Argument checks happen on the host before anything is enqueued; a failed check enqueues nothing.
 *   - Return value: QLORA_OK (0) or a negative QLORA_ERR_* code. Device-side conditions (non-finite
 *     input, a bounded wait that gave up) are recorded in the device status word and reported by
 *     qlora_get_status().
 *   - Calls are reentrant and may run concurrently on different streams when their buffers
 *     (including workspaces) do not overlap.
 */
#ifndef QLORA_NF4_H
#define QLORA_NF4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
typedef struct CUstream_st* qlora_stream_t;   /* a cudaStream_t */

enum qlora_status_code {
  QLORA_OK = 0,
  QLORA_ERR_INVALID_ARG = -1,  /* null pointer, bad dtype, bad rank r or alpha                     */
  QLORA_ERR_SHAPE = -2,        /* a size that is <= 0, too large, or breaks a divisibility rule    */
  QLORA_ERR_ALIGNMENT = -3,    /* a device pointer that is not 16-byte aligned                     */
  QLORA_ERR_WORKSPACE = -4,    /* workspace missing or smaller than the matching *_workspace query  */
  QLORA_ERR_CUDA = -5,         /* a CUDA runtime/driver call or kernel launch failed               */
  QLORA_ERR_NONFINITE = -6,    /* (status) a quantized input held Inf or NaN                        */
  QLORA_ERR_TIMEOUT = -7,      /* (status) a kernel's bounded wait gave up; its outputs are invalid */
  QLORA_ERR_UNSUPPORTED = -8,  /* the current device is not an sm_100 (B200-class) GPU             */
  QLORA_ERR_TOO_LARGE = -9,    /* input larger than the fixed scratch of qlora_nf4_quantize_noalloc */
  QLORA_ERR_CODEBOOK = -10     /* codebook not 2..16 ascending levels in [-1, 1], or too dense      */
};

/* Bits of the device status word (qlora_get_status). */
enum { QLORA_STATUS_NONFINITE = 1, QLORA_STATUS_TIMEOUT = 2 };

/* Element types of quantize inputs and dequantize outputs. */
enum { QLORA_F32 = 0, QLORA_BF16 = 1 };

/*
 * An NF4 tensor with double-quantized constants [PEFT "Double quantization"; EXPL "For the curious"].
 * numel = rows * cols, flattened row-major; nb = ceil(numel/64) blocks; ng = ceil(nb/256) groups.
 *   codes        ceil(numel/2) bytes; byte i = code(2i) << 4 | code(2i+1); for odd numel the last
 *                low nibble is 0. Codes index the 16-level NF4 codebook [PEFT "NF4, ..."].
 *   absmax_e4m3  nb bytes; E4M3 (OCP FP8) code of each block's mean-subtracted absmax constant.
 *   scale2       ng floats; the fp32 second-level constant of each group of 256 blocks.
 *   offset       1 float; the mean that was subtracted from the block constants.
 * All four are device pointers owned by the caller; sizes come from qlora_nf4_storage_bytes().
 */
typedef struct qlora_nf4_tensor {
  uint8_t* codes;
  uint8_t* absmax_e4m3;
  float* scale2;
  float* offset;
  int64_t rows;
  int64_t cols;
} qlora_nf4_tensor;

/*
 * The NF4 codebook [PEFT "NF4, derived from normal quantiles"]: 16 levels, 7 negative, an exact 0 at
 * index 7, 8 positive, normal quantiles of evenly spaced probabilities from 0.9677 down to 0.5, rescaled
 * so the ends are exactly -1 and +1; and the 15 decision thresholds (fp32-rounded midpoints of adjacent
 * levels). An element w of a block with absmax a > 0 gets code #{j : w > thresholds[j] * a} in exact
 * arithmetic (ties to the lower index); a block with a = 0 codes as 7.
 * `levels` (16 floats) and `thresholds` (15 floats) are HOST arrays written by the call. Needs no GPU.
 */
int qlora_nf4_codebook(float* levels, float* thresholds);

/*
 * Exact byte sizes of the four arrays of an n-element NF4 tensor (host outputs; any may be NULL).
 * Overhead of the constants: 8/64 + 32/(64*256) = 0.12695 bits per weight [PEFT "Double quantization"].
 * Needs no GPU. QLORA_ERR_SHAPE if n <= 0 or n > 2^40.
 */
int qlora_nf4_storage_bytes(int64_t n, size_t* codes_bytes, size_t* absmax_bytes,
                            size_t* scale2_bytes, size_t* offset_bytes);

/* Device workspace bytes qlora_nf4_quantize needs for an n-element input (host output). No GPU. */
int qlora_nf4_quantize_workspace(int64_t n, size_t* bytes);

/*
 * Quantize w (rows x cols, dtype QLORA_F32 or QLORA_BF16) into `out`, whose four pointers the caller
 * has allocated with qlora_nf4_storage_bytes(rows*cols) and whose rows/cols must match
 * [PEFT "Block-wise quantization in one page", "Double quantization"; EXPL "For the curious"]:
 *   1. per block of 64 consecutive elements: absmax c1 (fp32), codes, two per byte;
 *   2. mu = mean of all c1 (fp64 balanced pairwise tree over c1 zero-padded to max(256, 2^ceil(log2 nb))
 *      leaves, divided by nb in fp64, rounded to fp32);
 *   3. per group of 256 blocks: d = c1 - mu (fp32), s2 = max|d| / 448 (fp32), e = E4M3 round-to-nearest-
 *      even, saturating, of d / s2 (e = 0 when s2 = 0).
 * Any numel >= 1 is accepted; the last block and group may be partial. `workspace` (device, >=
 * qlora_nf4_quantize_workspace bytes) holds the fp32 c1, fp64 partial sums of the mean's tree and an
 * arrival counter between passes; its contents need no initialisation and are not kept between calls.
 * A non-finite input sets QLORA_STATUS_NONFINITE; the outputs of that call are then unspecified.
 * Results are deterministic and bit-identical run to run.
 */
int qlora_nf4_quantize(const void* w, int w_dtype, int64_t rows, int64_t cols,
                       const qlora_nf4_tensor* out, void* workspace, size_t workspace_bytes,
                       qlora_stream_t stream);

/*
 * qlora_nf4_quantize without a caller-provided workspace. (The QLoRA pages have no counterpart; this is
 * an interface variant of qlora_nf4_quantize, with identical results.)
 *
 * For callers that cannot allocate device memory at the point of the call: code running under a
 * framework's caching allocator, where a cudaMalloc behind the framework's back can synchronize the
 * device and fragment memory the framework manages; plugin or callback interfaces that hand over only
 * the input and output buffers; and loops that forbid allocation after start-up. The caller still
 * allocates `out` (qlora_nf4_storage_bytes); the intermediate per-block constants and partial sums live
 * in one fixed scratch array inside the library, QLORA_NOALLOC_SCRATCH_BYTES (about 4 MiB) of device
 * memory that every GPU which loads the library holds until the process exits.
 *   - rows * cols must not exceed QLORA_NOALLOC_MAX_NUMEL (2^26); larger inputs return
 *     QLORA_ERR_TOO_LARGE and enqueue nothing.
 *   - The first call on a device looks up that device's scratch address (host-side set-up, done once
 *     per device); make that first call before any stream capture.
 *   - Every call on a device shares the same scratch and nothing in it is cleared or kept between calls
 *     (each call writes every scratch element it reads). Calls that can overlap on the GPU -- on
 *     different streams without ordering between them -- race on the scratch and must not be issued.
 *   - The call allocates nothing: no cudaMalloc/cudaFree and no allocating library routine.
 * Other arguments, checks, status reporting and results are those of qlora_nf4_quantize.
 */
#define QLORA_NOALLOC_MAX_NUMEL (((int64_t)1) << 26)
#define QLORA_NOALLOC_SCRATCH_BYTES ((size_t)4 * 1024 * 1024 + (size_t)128 * 1024 + (size_t)512)
int qlora_nf4_quantize_noalloc(const void* w, int w_dtype, int64_t rows, int64_t cols,
                               const qlora_nf4_tensor* out, qlora_stream_t stream);

/*
 * Dequantize q into out (rows x cols, dtype QLORA_BF16 or QLORA_F32) [PEFT "Block-wise quantization in
 * one page": look up the level and multiply back; "Double quantization"; EXPL "Putting it together":
 * dequantized to bf16]:  c1_hat = fma(decode(e), s2, mu) (one fp32 rounding),
 * w_hat = fp32(level[code] * c1_hat), then round-to-nearest-even bf16 for QLORA_BF16.
 */
int qlora_nf4_dequantize(const qlora_nf4_tensor* q, void* out, int out_dtype, qlora_stream_t stream);

/*
 * NF4 without double quantization: the same 4-bit codes (two per byte, even element in the high
 * nibble) with the fp32 block constants kept as they are [PEFT "Double quantization": the constants
 * before the second level, 32/64 = 0.5 bits per weight; "The real way": double quantization is one of
 * the listed savings]. For an n-element tensor the caller allocates `codes` (ceil(n/2) bytes) and
 * `absmax` (ceil(n/64) fp32), both device pointers, 16-byte aligned.
 *   qlora_nf4_quantize_single writes both from w (rows x cols, QLORA_F32 or QLORA_BF16); codes are
 *     identical to qlora_nf4_quantize's. A non-finite input sets QLORA_STATUS_NONFINITE. No workspace.
 *   qlora_nf4_dequantize_single writes w_hat = fp32(level[code] * absmax[block]), rounded to bf16 (RNE)
 *     for QLORA_BF16 output.
 */
int qlora_nf4_quantize_single(const void* w, int w_dtype, int64_t rows, int64_t cols, void* codes,
                              float* absmax, qlora_stream_t stream);
int qlora_nf4_dequantize_single(const void* codes, const float* absmax, int64_t rows, int64_t cols,
                                void* out, int out_dtype, qlora_stream_t stream);

/*
 * Codebook comparison [PEFT "NF4, derived from normal quantiles": a Gaussian matrix quantized in blocks
 * of 64 with the symmetric int4 grid {-7..7}/7, the grid {-8..7}/8, NF4 and Lloyd's least-squares
 * codebook, compared by code entropy and RMS error; "Block-wise quantization in one page"]. The same
 * quantizer and dequantizer as the NF4 calls, with fp32 block constants and the caller's codebook.
 *
 * levels (host, nlevels fp32 values): 2 <= nlevels <= 16, strictly ascending, every |level| <= 1.
 * Thresholds are T_j = fp32((level_j + level_{j+1}) / 2), the sum formed in fp64; the code of w in a
 * block with absmax a > 0 is #{j : w > T_j * a} evaluated exactly (at most nlevels - 1), and an all-zero
 * block codes as the index of the level of least magnitude (the lower one on a tie). The quantizer looks
 * thresholds up by buckets of width 1/15 in w / a, so every bucket (widened by 2^-18) may hold at most
 * one threshold: any two thresholds more than 1/15 + 2^-17 apart always pass (the NF4, int4, {-8..7}/8
 * and Lloyd codebooks do). A codebook that breaks a rule returns QLORA_ERR_CODEBOOK, before any device
 * call. n is the element count of a dense tensor (1 <= n <= 2^40); the caller allocates `codes`
 * (ceil(n/2) bytes, two codes per byte, even element in the high nibble) and `absmax` (ceil(n/64) fp32).
 *   qlora_codebook_quantize    w (QLORA_F32 or QLORA_BF16) -> codes, absmax. A non-finite input sets
 *                              QLORA_STATUS_NONFINITE. With the NF4 levels the output equals
 *                              qlora_nf4_quantize_single's.
 *   qlora_codebook_dequantize  w_hat = fp32(level[code] * absmax[block]), bf16 (RNE) for QLORA_BF16.
 *   qlora_codebook_stats       what the codebook did to w (w, codes and absmax as written by
 *                              qlora_codebook_quantize with the same levels; w finite). `stats` is a
 *                              device array of QLORA_CODEBOOK_STATS_LEN doubles:
 *       [0..15]   count_j, the number of elements with code j
 *       [16..31]  sum_j, the sum of u = w / a over them in fp64 (u formed as w * fp64(1/a), within one
 *                 fp64 ulp of the quotient; 0 in an all-zero block)
 *       [32]      sum over all elements of (w_hat - w)^2 in fp64, w_hat as qlora_codebook_dequantize's fp32
 *       [33]      code entropy in bits, -sum_j p_j log2 p_j with p_j = count_j / n
 *       [34]      RMS error, sqrt([32] / n)
 *       [35..50]  one step of Lloyd's algorithm: fp32(sum_j / count_j), or level_j where count_j = 0
 *                 (entries past nlevels hold 0)
 *     Sums run in a fixed order for a given n and device, so the result is deterministic.
 *     `workspace` >= qlora_codebook_stats_workspace(n) bytes (device).
 */
#define QLORA_CODEBOOK_STATS_LEN 51
int qlora_codebook_quantize(const void* w, int w_dtype, int64_t n, const float* levels, int nlevels,
                            void* codes, float* absmax, qlora_stream_t stream);
int qlora_codebook_dequantize(const void* codes, const float* absmax, int64_t n, const float* levels,
                              int nlevels, void* out, int out_dtype, qlora_stream_t stream);
int qlora_codebook_stats_workspace(int64_t n, size_t* bytes);
int qlora_codebook_stats(const void* w, int w_dtype, const void* codes, const float* absmax, int64_t n,
                         const float* levels, int nlevels, double* stats, void* workspace,
                         size_t workspace_bytes, qlora_stream_t stream);

/*
 * Paged optimizer [PEFT "Paged optimizers, and QLoRA end to end": the optimizer states are allocated in
 * NVIDIA unified memory, which the driver pages between GPU and CPU RAM when the GPU runs short, and paged
 * back when the optimizer step needs them; EXPL "The three innovations": paged optimizers absorb memory
 * spikes]. The update is not written on the pages; it is the standard AdamW (Adam with decoupled weight
 * decay, Loshchilov & Hutter 2019) in fp32:
 *     p <- p (1 - lr wd);  m <- b1 m + (1 - b1) g;  v <- b2 v + (1 - b2) g^2;
 *     p <- p - [lr / (1 - b1^t)] m / (sqrt(v) / sqrt(1 - b2^t) + eps)
 * with the two bias corrections formed in fp64 on the host for step t >= 1.
 *
 * qlora_adamw_step   one fused pass over n fp32 elements: p (read, written), g (read), m and v (read,
 *                    written); p_bf16 (n bf16, or NULL) receives bf16(p) after the update. The pointers may
 *                    be device memory or managed memory from qlora_paged_alloc, resident or not (pages move
 *                    to the GPU as the kernel touches them). QLORA_ERR_INVALID_ARG unless t >= 1,
 *                    0 <= b1, b2 < 1, eps > 0, lr >= 0 and wd >= 0 (all finite).
 * qlora_paged_alloc  *ptr = `bytes` of managed (unified) memory, accessible from the host and every GPU;
 *                    contents uninitialised. The one call that allocates: the caller frees with
 *                    qlora_paged_free.
 * qlora_paged_prefetch  enqueue on `stream` a migration of [ptr, ptr + bytes) to the current GPU
 *                    (to_device != 0) or to host memory (to_device == 0, as the driver does when it evicts
 *                    under memory pressure). QLORA_ERR_UNSUPPORTED if the GPU cannot access managed memory
 *                    concurrently with the host.
 */
int qlora_adamw_step(float* p, const float* g, float* m, float* v, void* p_bf16, int64_t n, int64_t step,
                     float lr, float beta1, float beta2, float eps, float weight_decay, qlora_stream_t stream);
int qlora_paged_alloc(size_t bytes, void** ptr);
int qlora_paged_free(void* ptr);
int qlora_paged_prefetch(const void* ptr, size_t bytes, int to_device, qlora_stream_t stream);

/*
 * Device workspace bytes for qlora_linear_fwd / qlora_linear_bwd with T tokens, weight N x K (out x in)
 * and LoRA rank r (host output). One buffer of this size serves both calls.
 */
int qlora_linear_workspace(int64_t T, int64_t N, int64_t K, int r, size_t* bytes);

/*
 * QLoRA linear forward [EXPL "Putting it together": Y = X dequant(W) + X L1 L2; PEFT "Paged optimizers,
 * and QLoRA end to end": the frozen NF4 weight is dequantized to bf16 block by block, multiplied in
 * 16-bit precision, and a bf16 LoRA adapter is added to the output]:
 *     Y = X W~^T + s (X A^T) B^T,   s = alpha / r,   W~ = dequant(W) in bf16 (as qlora_nf4_dequantize).
 *   X      T x K bf16          W  NF4 tensor, rows = N (out), cols = K (in)
 *   A      r x K bf16          B  N x r bf16          Y  T x N bf16 (written)
 *   U_out  T x r bf16 or NULL: if given, receives s * (X A^T) rounded to bf16, the scaled adapter
 *          activation, in the form qlora_linear_bwd takes as U (saves recomputing it there).
 * fp32 accumulation on the tensor cores. Rules: T >= 1; K % 64 == 0; N % 8 == 0; r % 8 == 0 and
 * 8 <= r <= 256; alpha finite. `workspace` >= qlora_linear_workspace(T, N, K, r).
 */
int qlora_linear_fwd(const void* X, int64_t T, const qlora_nf4_tensor* W, const void* A,
                     const void* B, int r, float alpha, void* Y, void* U_out, void* workspace,
                     size_t workspace_bytes, qlora_stream_t stream);

/*
 * QLoRA linear backward [EXPL "Putting it together": gradients flow only into the adapters, never into
 * the 4-bit weights; PEFT "Paged optimizers, and QLoRA end to end": gradients flow back through the
 * dequantized weights to earlier layers]:
 *     dX = dY W~ + s (dY B) A,   dA = s (dY B)^T X,   dB = s dY^T (X A^T);   no gradient for W.
 *   dY  T x N bf16;  X, W, A, B, r, alpha as in qlora_linear_fwd;
 *   U   T x r bf16 from qlora_linear_fwd's U_out with the same X, A, alpha, or NULL to recompute it;
 *   dX  T x K bf16 or NULL (skip the input gradient, e.g. for the first layer);
 *   dA  r x K fp32, dB  N x r fp32 (written, not accumulated; the adapters' gradients stay fp32).
 * Same shape rules and workspace as qlora_linear_fwd.
 */
int qlora_linear_bwd(const void* dY, const void* X, int64_t T, const qlora_nf4_tensor* W,
                     const void* A, const void* B, int r, float alpha, const void* U, void* dX,
                     float* dA, float* dB, void* workspace, size_t workspace_bytes,
                     qlora_stream_t stream);

/*
 * Synchronize `stream`, then read and clear the current device's status word into *device_status
 * (host; a bitwise OR of QLORA_STATUS_* set by kernels since the last call). Returns QLORA_OK, or
 * QLORA_ERR_NONFINITE / QLORA_ERR_TIMEOUT when the corresponding bit was set (TIMEOUT wins).
 */
int qlora_get_status(int* device_status, qlora_stream_t stream);

/*
 * Failure-path controls for tests (the pages have no counterpart; the bounded waits and the status word
 * are this library's own error handling).
 *
 * qlora_set_wait_limit sets, for the current device, how long (ns, device time) any bounded wait in the
 * library's kernels -- on a shared-memory barrier, or on a device word written by another CTA of the
 * same grid -- waits before it gives up, records QLORA_STATUS_TIMEOUT and lets its kernel unwind. 0
 * restores the default of 2 s; other values must lie in [1000, 2e9]. Every later launch on the device
 * uses the new limit, so a short limit can make long legitimate waits fail: it is meant for tests.
 * Synchronous (a copy to device memory). QLORA_ERR_INVALID_ARG for a value out of range.
 *
 * qlora_selftest_wait launches, on `stream`, a one-warp kernel that waits on something that never
 * happens: kind QLORA_SELFTEST_MBARRIER waits on a shared-memory barrier that no thread arrives on,
 * QLORA_SELFTEST_DEVICE_WORD on a device word that nothing writes. The wait gives up after the limit in
 * force and the kernel returns; qlora_get_status then reports QLORA_ERR_TIMEOUT and the context stays
 * usable. Nothing faults, traps or spins without a bound.
 *
 * Host-side fault injection: with the environment variable QLORA_FAULT_INJECT set to "<entry point>"
 * or "<entry point>:<k>" (e.g. "qlora_linear_fwd:2"), the k-th call (default: the first) of that entry
 * point since the variable took its current value returns QLORA_ERR_CUDA, as a failed launch would,
 * after its argument checks and before it enqueues anything. With QLORA_DEBUG set, each injected failure
 * is reported on stderr. Applies to the entry points that launch kernels.
 */
enum { QLORA_SELFTEST_MBARRIER = 0, QLORA_SELFTEST_DEVICE_WORD = 1 };
int qlora_set_wait_limit(uint64_t ns);
int qlora_selftest_wait(int kind, qlora_stream_t stream);

/* Static English text for a QLORA_* code (never NULL). */
const char* qlora_error_string(int code);

/*
 * Kernel timing for benchmarks. While enabled, the library records a CUDA event pair on the launch
 * stream around every launch of its main matrix kernels and its codec kernels. qlora_profile_read
 * synchronizes the recorded events and returns, per kernel class (QLORA_PROF_*), the number of launches
 * and their summed device time in milliseconds (host arrays of QLORA_PROF_COUNT entries), then clears
 * the record. Enabling does not change any result.
 */
enum {
  QLORA_PROF_QUANTIZE = 0,    /* the three quantize kernels of one call, as one interval   */
  QLORA_PROF_DEQUANTIZE = 1,
  QLORA_PROF_FWD_GEMM = 2,    /* fused dequant + tensor-core forward (Y)                    */
  QLORA_PROF_BWD_GEMM = 3,    /* fused dequant + tensor-core backward (dX)                  */
  QLORA_PROF_LORA = 4,        /* the adapter kernels (U, V, dA, dB and their reductions)    */
  QLORA_PROF_COUNT = 5
};
int qlora_profile_enable(int on);
int qlora_profile_read(int64_t* launches, double* total_ms);

/* Number of kernels the library has launched in this process (all devices, all streams). */
int64_t qlora_kernel_launches(void);

#ifdef __cplusplus
}
#endif
#endif /* QLORA_NF4_H */
