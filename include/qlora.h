/*
 * libqlora — the QLoRA linear layer on NVIDIA B200 (sm_100a).
 *
 * C ABI.  Every pointer argument is a plain pointer; unless stated otherwise
 * it is a DEVICE pointer to memory owned by the caller (for example a PyTorch
 * tensor's data pointer).  The library never allocates or frees device
 * memory: scratch space is passed in as a workspace whose size the matching
 * *_workspace_bytes() query returns.  Every compute call is asynchronous on
 * the given stream and returns a qlora_status_t after validating its
 * arguments on the host (nothing is launched when validation fails).
 *
 * Layouts: row-major and contiguous.  bf16 tensors are passed as uint16_t
 * bit patterns.  Notation follows the layer h = W0 x + (alpha/r) B A x with
 * W0 d x k (frozen), A r x k, B d x r, tokens as rows: X is T x k, Y is T x d.
 * s = alpha / r.
 *
 * Sources, cited by page title and section:
 *   [P1] "LoRA and QLoRA fine-tuning: mechanics, and when not to fine-tune"
 *   [P2] "Fine-Tuning on a Budget: LoRA and QLoRA"
 *
 * Inputs must be finite; results for NaN/Inf inputs are unspecified.
 */
#ifndef QLORA_H_
#define QLORA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define QLORA_API __attribute__((visibility("default")))
#else
#define QLORA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  QLORA_OK = 0,
  QLORA_ERR_INVALID_ARG = 1,       /* null pointer, negative size, bad alpha */
  QLORA_ERR_UNSUPPORTED_SHAPE = 2, /* k % 64 != 0, r outside [1, 256], too large */
  QLORA_ERR_MISALIGNED = 3,        /* a pointer is not 16-byte aligned */
  QLORA_ERR_WORKSPACE_TOO_SMALL = 4,
  QLORA_ERR_CUDA = 5,              /* a CUDA runtime/driver call or launch failed */
  QLORA_ERR_TIMEOUT = 6,           /* a device-side wait gave up (device status) */
  QLORA_ERR_NO_DEVICE = 7,         /* no sm_100 device is current */
  QLORA_ERR_EXCEEDS_STATIC_SCRATCH = 8, /* too large for qlora_nf4_quantize_noalloc */
  QLORA_ERR_NCCL = 9               /* NCCL could not be loaded, or an NCCL call failed */
} qlora_status_t;

/* A cudaStream_t passed as an opaque pointer (NULL = legacy default stream). */
typedef void* qlora_stream_t;

/*
 * NF4 storage of a frozen d x k weight with double-quantised block constants
 * ([P1] "What QLoRA freezes, and in how many bits": NF4, first-level block
 * 64, second-level FP8 constants in blocks of 256 after subtracting their
 * mean; [P1] "What to choose and why": keep NF4/64/256 with the bundle).
 * All buffers are device memory owned by the caller:
 *   codes     d*k/2 bytes; byte m holds element 2m (row-major order) in bits
 *             0-3 and element 2m+1 in bits 4-7
 *   absmax_q  n_b = d*k/64 bytes: E4M3 code of (absmax_b - mean)/scale2_j
 *   scale2    n_g = ceil(n_b/256) floats: second-level scale of group j
 *   mean      1 float: mean of the first-level absmax constants
 * block and block2 must be 64 and 256.
 */
typedef struct {
  uint8_t* codes;
  uint8_t* absmax_q;
  float* scale2;
  float* mean;
  int64_t d;
  int64_t k;
  int32_t block;
  int32_t block2;
} qlora_nf4_t;

/* Per-kernel timing collected while profiling is on (see qlora_profile_*). */
typedef struct {
  char name[48];
  int64_t launches;
  double total_ms;       /* sum of CUDA-event durations on the launch stream */
  double flops;          /* algorithmic flops of all launches (0 if not a GEMM) */
  double bytes;          /* algorithmic DRAM bytes of all launches */
} qlora_kernel_stat_t;

/* Human-readable text for a status code (static storage, never NULL). */
QLORA_API const char* qlora_strerror(int status);

/* Library version as 10000*major + 100*minor + patch. */
QLORA_API int qlora_version(void);

/*
 * The library's own NF4 table (host call, no GPU needed): the 16 fp32 levels
 * in ascending order and the 15 encoder thresholds t_i = the smallest fp32
 * strictly above the exact midpoint of levels i and i+1, so that
 * code(x) = #{i : x >= t_i} is the nearest level with ties to the lower code.
 * Either pointer may be NULL.  Always returns QLORA_OK.
 */
QLORA_API int qlora_nf4_levels(float* levels16, float* thresholds15);

/* ---------------------------------------------------------------- quantise */

/* Workspace for qlora_nf4_quantize: fp32 absmax per block, fp64 sum per
 * group and a 4-byte completion counter (each part 256-byte aligned). */
QLORA_API size_t qlora_quantize_workspace_bytes(int64_t d, int64_t k);

/*
 * nf4_quantize(W0, block=64) ([P1] 4-bit NormalFloat and Double
 * quantisation paragraphs).  W0: fp32 d x k, device.  `out` is a HOST struct
 * whose four device pointers the caller has set; the call writes d, k, block
 * and block2 into it and fills the device buffers:
 *   a_b  = max |w| over each 64-block,
 *   code = nearest NF4 level of fp32(w / a_b) (ties to the lower code; an
 *          all-zero block gives the zero level),
 *   mean = fp32(S / n_b), S the float64 pairwise sum of all a_b,
 *   scale2_j = fp32(max_b |fp32(a_b - mean)| / 448) per group of 256,
 *   absmax_q_b = E4M3_RN_satfinite(fp32(fp32(a_b - mean) / scale2_j))
 *               (0 when scale2_j == 0).
 * Requires block == 64, k % 64 == 0, d >= 1, d*k < 2^34.  W0 and the output
 * buffers must be 16-byte aligned.  Every weight must be finite: a NaN or
 * infinity makes the results unspecified (the call still completes and
 * returns QLORA_OK; nothing is read or written out of bounds).  Subnormal
 * weights and block maxima are handled exactly.
 */
QLORA_API int qlora_nf4_quantize(const float* W0, int64_t d, int64_t k, int block, qlora_nf4_t* out,
                       void* workspace, size_t workspace_bytes, qlora_stream_t stream);

/*
 * doubleDequant ([P1] forward equation): W' (bf16, d x k, device) with
 *   a'_b = fp32(fp32(E4M3(absmax_q_b) * scale2_j) + mean),
 *   w'   = bf16_RN(fp32(level[code] * a'_b)).
 * This is the exact bf16 weight every GEMM of this library multiplies by.
 */
QLORA_API int qlora_nf4_dequantize(const qlora_nf4_t* q, uint16_t* W_out, qlora_stream_t stream);

/*
 * Quantise without any allocation and without a caller workspace.
 *
 * (This entry point has no counterpart on the source pages; it exists for
 * callers that cannot allocate device memory at all.)  Some callers hold only
 * the device buffers they were handed: a plugin whose host framework owns
 * every byte of device memory through its own pool and forbids allocations
 * outside it, or a recovery path that re-quantises weights after the device
 * has run out of memory, where any new cudaMalloc would fail.  They can call
 * this instead of qlora_nf4_quantize.
 *
 * Same arguments and results as qlora_nf4_quantize, minus the workspace.  The
 * scratch space (fp32 block constants and fp64 group sums) lives in a
 * file-scope __device__ array of QLORA_NOALLOC_MAX_WEIGHTS/16 +
 * QLORA_NOALLOC_MAX_WEIGHTS/2048 + 256 bytes (16.1 MiB) that every GPU which loads
 * this library holds until the process exits.  d*k above
 * QLORA_NOALLOC_MAX_WEIGHTS (2^28 weights) is rejected with
 * QLORA_ERR_EXCEEDS_STATIC_SCRATCH before anything is launched.
 *
 * The first call on a device looks up the array's device address (with that
 * device current) and caches it with the id of the current CUDA context; make
 * that first call before any stream capture begins.  After a device reset the
 * next call runs in a new context and looks the address up again (the array's
 * contents start over then).  All calls share the one array, which keeps the contents
 * of the last call; every byte a call reads from it is first written by the
 * same call, so nothing needs clearing.  Calls that overlap on the GPU (on
 * different streams, or from different threads) race on the array and must
 * be serialised by the caller.  No cudaMalloc, cudaFree or allocating library
 * routine is called.
 */
#define QLORA_NOALLOC_MAX_WEIGHTS ((int64_t)1 << 28)
QLORA_API int qlora_nf4_quantize_noalloc(const float* W0, int64_t d, int64_t k, int block,
                                         qlora_nf4_t* out, qlora_stream_t stream);

/* ---------------------------------------------------------------- forward */

QLORA_API size_t qlora_fwd_workspace_bytes(int64_t d, int64_t k, int r, int64_t T);

/*
 * Forward ([P1] forward equation; [P2] "The LoRA hypothesis" figure):
 *   U = X A^T                  (fp32, T x r, written to U_save for backward)
 *   Y = X W'^T + s U B^T       (bf16, T x d)
 * W' is doubleDequant(q) in bf16; the rank-r term is accumulated in the same
 * fp32 tile as the base product (its operand s*U is rounded to bf16).
 * X: bf16 T x k; A: bf16 r x k; B: bf16 d x r; alpha > 0 (s = alpha / r).
 * T may be 0 (no work).  Requires 1 <= r <= 256.
 */
QLORA_API int qlora_fwd(const qlora_nf4_t* q, const uint16_t* A, const uint16_t* B, int r, float alpha,
              const uint16_t* X, int64_t T, uint16_t* Y, float* U_save, void* workspace,
              size_t workspace_bytes, qlora_stream_t stream);

/* ---------------------------------------------------------------- backward */

QLORA_API size_t qlora_bwd_workspace_bytes(int64_t d, int64_t k, int r, int64_t T);

/*
 * Backward of L with dL/dY = dY ([P1] "The update LoRA is allowed to learn":
 * only the adapter factors are trained; [P1] "What QLoRA freezes": the
 * activation gradient is formed through W dequantised to bf16):
 *   G  = dY B                  (fp32 accumulate, used as bf16 s*G)
 *   dX = dY W' + s G A         (bf16, T x k)
 *   dA = s G^T X               (fp32, r x k, overwritten)
 *   dB = s dY^T U              (fp32, d x r, overwritten; U = U_saved)
 * Requires d % 8 == 0 (rows of dY 16-byte aligned).  No weight gradient is
 * formed.  dA and dB are reduced in a fixed order, so
 * repeated calls give identical bits.
 */
QLORA_API int qlora_bwd(const qlora_nf4_t* q, const uint16_t* A, const uint16_t* B, int r, float alpha,
              const uint16_t* X, const float* U_saved, const uint16_t* dY, int64_t T,
              uint16_t* dX, float* dA, float* dB, void* workspace, size_t workspace_bytes,
              qlora_stream_t stream);

/* ------------------------------------------------ LoRA dropout (next row) */

/*
 * The layer with LoRA dropout on the adapter input ([P5] "LoRA vs QLoRA:
 * Parameter-Efficient Fine-Tuning Explained", run configuration: a LoRA
 * dropout of 0.05-0.1).  The pages give no formula; this library applies
 * inverted dropout to the input of the adapter path only:
 *   D(X) = X * keep / (1 - p),   U = D(X) A^T,   Y = X W'^T + s U B^T
 * and the matching gradients
 *   G = dY B,  dX = dY W' + D(s G A),  dA = s G^T D(X),  dB = s dY^T U.
 * keep: device, bit-packed T x k mask drawn by the caller (bit j % 8 of byte
 * (t*k + j) / 8 is 1 where element (t, j) is kept), 16-byte aligned; the
 * forward and the backward of one step must get the same mask.  0 <= p < 1;
 * p == 0 ignores `keep` and is exactly qlora_fwd / qlora_bwd.  U_save holds
 * the dropped-out U for the backward.  Otherwise the arguments, results and
 * errors are those of qlora_fwd / qlora_bwd; the workspaces also hold the
 * masked input (T x k bf16).
 */
QLORA_API size_t qlora_fwd_dropout_workspace_bytes(int64_t d, int64_t k, int r, int64_t T);
QLORA_API int qlora_fwd_dropout(const qlora_nf4_t* q, const uint16_t* A, const uint16_t* B, int r, float alpha,
                                const uint16_t* X, const uint8_t* keep, float p, int64_t T, uint16_t* Y,
                                float* U_save, void* workspace, size_t workspace_bytes, qlora_stream_t stream);
QLORA_API size_t qlora_bwd_dropout_workspace_bytes(int64_t d, int64_t k, int r, int64_t T);
QLORA_API int qlora_bwd_dropout(const qlora_nf4_t* q, const uint16_t* A, const uint16_t* B, int r, float alpha,
                                const uint16_t* X, const uint8_t* keep, float p, const float* U_saved,
                                const uint16_t* dY, int64_t T, uint16_t* dX, float* dA, float* dB,
                                void* workspace, size_t workspace_bytes, qlora_stream_t stream);

/* ------------------------------------- several unmerged adapters (next row) */

/*
 * One frozen base with a stack of unmerged adapters, each token using its own
 * ([P2] "The LoRA hypothesis": serving many tasks keeps the adapters unmerged,
 * one base in memory and a few-MB adapter chosen per request; [P1] "What to
 * choose and why": one deployed base, a small B A per task).  The pages give
 * no batching rule; here token t uses adapter idx[t] of the stack:
 *   U[t] = X[t] A_i^T,   Y[t] = X[t] W'^T + s_i U[t] B_i^T,   i = idx[t], s_i = alphas[i] / r
 * and the backward gives dX and, per adapter, dA_i = s_i sum_{t: idx[t]=i} G[t]^T X[t],
 * dB_i = s_i sum_{t: idx[t]=i} dY[t]^T U[t] with G[t] = dY[t] B_i (an adapter
 * no token uses gets dA_i = dB_i = 0 exactly).
 * As: device, n x r x k bf16 (adapter i's A at As + i r k); Bs: device,
 * n x d x r bf16; alphas: HOST array of n floats (> 0); idx: device int32[T]
 * (a token whose index is outside [0, n) gets no adapter term and a zero U
 * row); U_save: T x r fp32, the token's own U.  dAs (n x r x k) and dBs
 * (n x d x r) are fp32 and overwritten.  1 <= n <= 64 and n r <= 256.  With
 * n = 1 and every idx 0 the results are bit-identical to qlora_fwd /
 * qlora_bwd.  Other arguments and errors as for qlora_fwd / qlora_bwd.
 */
QLORA_API size_t qlora_fwd_multi_workspace_bytes(int64_t d, int64_t k, int n, int r, int64_t T);
QLORA_API int qlora_fwd_multi(const qlora_nf4_t* q, int n, const uint16_t* As, const uint16_t* Bs, int r,
                              const float* alphas, const int32_t* idx, const uint16_t* X, int64_t T, uint16_t* Y,
                              float* U_save, void* workspace, size_t workspace_bytes, qlora_stream_t stream);
QLORA_API size_t qlora_bwd_multi_workspace_bytes(int64_t d, int64_t k, int n, int r, int64_t T);
QLORA_API int qlora_bwd_multi(const qlora_nf4_t* q, int n, const uint16_t* As, const uint16_t* Bs, int r,
                              const float* alphas, const int32_t* idx, const uint16_t* X, const float* U_saved,
                              const uint16_t* dY, int64_t T, uint16_t* dX, float* dAs, float* dBs,
                              void* workspace, size_t workspace_bytes, qlora_stream_t stream);

/* ------------------------------------------- plain LoRA on a bf16 base */

/*
 * The same layer on an unquantised bf16 base W ([P2] "The LoRA hypothesis":
 * h = W0 x + (alpha/r) B A x with W0 frozen; [P2] "QLoRA: shrink the frozen
 * part too": QLoRA buys its memory saving with a dequantisation of the base
 * in every step, which LoRA on a 16-bit base does not pay).  Same arguments,
 * results and errors as qlora_fwd / qlora_bwd with W in place of W' and its
 * shape passed as d, k.  W: bf16 d x k, device, 16-byte aligned, k % 8 == 0
 * (rows 16-byte aligned for TMA), caller-owned and only read.  The workspace
 * holds no copy of the weight, so it is smaller than the QLoRA one.
 */
QLORA_API size_t lora_fwd_workspace_bytes(int64_t d, int64_t k, int r, int64_t T);
QLORA_API int lora_fwd(const uint16_t* W, int64_t d, int64_t k, const uint16_t* A, const uint16_t* B, int r,
             float alpha, const uint16_t* X, int64_t T, uint16_t* Y, float* U_save, void* workspace,
             size_t workspace_bytes, qlora_stream_t stream);

QLORA_API size_t lora_bwd_workspace_bytes(int64_t d, int64_t k, int r, int64_t T);
QLORA_API int lora_bwd(const uint16_t* W, int64_t d, int64_t k, const uint16_t* A, const uint16_t* B, int r,
             float alpha, const uint16_t* X, const float* U_saved, const uint16_t* dY, int64_t T,
             uint16_t* dX, float* dA, float* dB, void* workspace, size_t workspace_bytes,
             qlora_stream_t stream);

/* ------------------------------------------------- optimiser (next row) */

/*
 * One Adam step on a trainable fp32 tensor, e.g. A (n = r*k) or B (n = d*r)
 * with their gradients dA, dB ([P1] "The update LoRA is allowed to learn":
 * only A and B carry optimiser state; [P2] "Why full fine-tuning costs so
 * much": a 16-bit forward copy, an fp32 master copy and fp32 moments m, v per
 * parameter).  The pages print no update rule; this is bias-corrected Adam
 * (Kingma and Ba 2015) with decoupled weight decay (Loshchilov and Hutter
 * 2019), computed in fp32:
 *   m = beta1 m + (1 - beta1) g;   v = beta2 v + (1 - beta2) g^2;
 *   master -= lr (m / (1 - beta1^step) / (sqrt(v / (1 - beta2^step)) + eps)
 *                 + weight_decay master);
 *   weight_bf16 = bf16_RN(master)   (the copy the forward and backward read).
 * All five arrays are device, n elements, 16-byte aligned and updated in
 * place (grad is only read).  step counts from 1; lr, eps, weight_decay >= 0;
 * 0 <= beta1, beta2 < 1.  Returns QLORA_ERR_INVALID_ARG otherwise.
 */
QLORA_API int lora_adam_step(float* master, uint16_t* weight_bf16, float* m, float* v, const float* grad,
                             int64_t n, int64_t step, float lr, float beta1, float beta2, float eps,
                             float weight_decay, qlora_stream_t stream);

/* ---------------------------------------------------------------- deploy */

QLORA_API size_t lora_merge_workspace_bytes(int64_t d, int64_t k, int r);

/*
 * Merge ([P1] deploy paragraph; [P2] "The LoRA hypothesis": the scaled
 * product is added to the base weight; [P2] "What actually goes wrong": the
 * merge goes into a 16-bit base while the adapter is kept separately):
 *   W = bf16_RN(fp32(w' + s (B A)_fp32))   (bf16 d x k, out of place)
 * The NF4 storage is left untouched so the merge can be undone.
 */
QLORA_API int lora_merge(const qlora_nf4_t* q, const uint16_t* A, const uint16_t* B, int r, float alpha,
               uint16_t* W_out, void* workspace, size_t workspace_bytes, qlora_stream_t stream);

/*
 * Unmerge / task switch ([P1] deploy paragraph: a task is removed by
 * subtracting its scaled product again):
 *   W0'' = bf16_RN(fp32(W - s (B A)_fp32))   (bf16 d x k, out of place)
 */
QLORA_API int lora_unmerge(const uint16_t* W, const uint16_t* A, const uint16_t* B, int r, float alpha,
                 int64_t d, int64_t k, uint16_t* W0_out, void* workspace,
                 size_t workspace_bytes, qlora_stream_t stream);

/* ---------------------------------------------------------------- status */

/*
 * Synchronises `stream`, then returns (in *status) and clears the device
 * status word of the current device: QLORA_OK, or the first error a kernel
 * recorded (QLORA_ERR_TIMEOUT when a bounded device wait gave up).  The
 * return value reports failures of this call itself.
 */
QLORA_API int qlora_get_device_status(qlora_stream_t stream, int* status);

/*
 * Self-test of the bounded wait: launches one block that waits on a barrier
 * nothing will complete, with a limit of `limit_us` microseconds (1..2e6).
 * The kernel gives up, records QLORA_ERR_TIMEOUT and exits; read it with
 * qlora_get_device_status.  The wait limit of other kernels is unchanged.
 */
QLORA_API int qlora_selftest_wait_timeout(int limit_us, qlora_stream_t stream);

/* ------------------------------------------------------------ data parallel */

/*
 * The layer is data-parallel over tokens ([P1] "The update LoRA is allowed to
 * learn": only A and B get gradients, the frozen weight needs no exchange).
 * Each GPU keeps a replica of the NF4 weight, A and B, runs forward and
 * backward on its own tokens, and the one exchange is the sum of dA and dB
 * over the ranks.  The library makes that call through NCCL; the caller owns
 * the communicator.  NCCL (libnccl.so.2) is loaded at the first of these
 * calls, so the library itself loads without it; QLORA_ERR_NCCL when it is
 * missing or a call fails.
 */
#define QLORA_NCCL_ID_BYTES 128

/* Writes a new NCCL unique id (QLORA_NCCL_ID_BYTES bytes, host memory) for
 * the caller to share with every rank before qlora_comm_init. */
QLORA_API int qlora_comm_unique_id(uint8_t* id);

/* Creates this rank's communicator on the current device (collective: every
 * rank calls it with the same id and nranks, each with its own rank in
 * [0, nranks)).  *comm receives an opaque handle. */
QLORA_API int qlora_comm_init(const uint8_t* id, int nranks, int rank, void** comm);

/* Releases a communicator made by qlora_comm_init (call it on every rank,
 * after the last collective using it has completed). */
QLORA_API int qlora_comm_destroy(void* comm);

/*
 * In place, on `stream`: dA (nA fp32) and dB (nB fp32, device memory) become
 * their sums over the ranks of `comm`, as one group of two NCCL all-reduces.
 * Either count may be 0.  Every rank must make the same call with the same
 * counts.  Returns at once (stream-ordered); QLORA_ERR_INVALID_ARG for a null
 * communicator, a negative count or a null pointer with a positive count.
 */
QLORA_API int qlora_grad_allreduce(void* comm, float* dA, int64_t nA, float* dB, int64_t nB,
                                   qlora_stream_t stream);

/* ---------------------------------------------------------------- profiling */

/*
 * Profiling: while on, every kernel launch of this library is bracketed by
 * CUDA events recorded on its launch stream.  qlora_profile_begin clears the
 * counters; qlora_profile_end synchronises the recorded events, writes up to
 * `capacity` per-kernel-class sums to `out` (host array) and the number of
 * classes to *n_out, and turns profiling off.
 */
QLORA_API int qlora_profile_begin(void);
QLORA_API int qlora_profile_end(qlora_kernel_stat_t* out, int capacity, int* n_out);

/* Number of kernels this library has launched in this process (all devices). */
QLORA_API int64_t qlora_launch_count(void);

/*
 * Selects the build of the NF4 base GEMM used above 64 tokens, for every
 * later call in this process: 0 = default (CTA pairs where the device can
 * hold clusters of two, else one CTA per tile), 1 = one CTA per 256 x 256
 * tile, 2 = CTA pairs (two CTAs of a cluster run 256-row tensor-core MMAs
 * over both SMs, each decoding half of every weight tile).  Both builds give
 * bit-identical results; the choice only changes speed.  Returns
 * QLORA_ERR_INVALID_ARG for any other mode.
 */
QLORA_API int qlora_set_nf4_gemm_mode(int mode);

#ifdef __cplusplus
}
#endif

#endif /* QLORA_H_ */
