/*
 * qlora.h - C ABI of libqlora.so: NF4 blockwise quantization with double-
 * quantized constants, dequantization, and the QLoRA frozen-base linear
 * layer (forward and backward) on NVIDIA B200 (sm_100a).
 *
 * Method: QLoRA (Dettmers et al., "QLoRA: Efficient Finetuning of Quantized
 * LLMs", NeurIPS 2023), as restated on the diycv.top QLoRA walkthrough:
 *   - "方法总览" §1 blockwise quantization (absmax per contiguous block of 64),
 *   - §2 NF4 (16 normal-quantile code values with an exact zero),
 *   - §3 double quantization (block constants, mean subtracted, to 8-bit
 *     floats in groups of 256),
 *   - "关键公式" the QLoRA linear layer Y = X doubleDequant(c1, c2, W)
 *     + s X L1 L2, and the data-type table (NF4 weights, FP8 first-level and
 *     FP32 second-level constants, BF16 matmuls),
 *   - "训练" step 5: the backward pass goes through the frozen weight, only
 *     the LoRA factors L1, L2 receive gradients.
 *
 * Conventions shared by every entry point
 *   - Pointers are DEVICE pointers unless marked "host".  The caller owns and
 *     allocates every buffer; the library allocates no device memory.  Where
 *     an operation needs scratch space, a *_workspace_size() function returns
 *     the byte count and the caller passes a buffer at least that large.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  All work is enqueued on it; no call synchronizes the host.
 *     Inputs are never modified.
 *   - bf16 is IEEE bfloat16 stored as uint16_t; fp32 is IEEE binary32.
 *   - Every function validates its arguments before it launches anything and
 *     returns a status code (QLORA_OK = 0).  An invalid argument launches
 *     nothing.  Faults inside kernels surface asynchronously, as in CUDA;
 *     qlora_check_status() reports a pipeline wait that gave up.
 *   - Weight layout: W is logically h x o (in x out); it is stored as its
 *     transpose W^T[o][h], row-major, so every block of 64 consecutive
 *     elements lies in one output row along the reduction axis (h % 64 == 0).
 *   - No CPU fallback: without a CUDA device every compute call returns
 *     QLORA_ERR_CUDA.
 */
#ifndef QLORA_H
#define QLORA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes. */
#define QLORA_OK              0
#define QLORA_ERR_NULL        1  /* a required pointer is NULL */
#define QLORA_ERR_SHAPE       2  /* sizes violate a divisibility or range rule */
#define QLORA_ERR_ALIGN       3  /* a pointer is not 16-byte aligned */
#define QLORA_ERR_UNSUPPORTED 4  /* block != 64, dq_block != 256, bad r or dtype */
#define QLORA_ERR_CODEBOOK    5  /* codebook not 16 finite increasing values with one 0.0 */
#define QLORA_ERR_CUDA        6  /* a CUDA call or launch failed */
#define QLORA_ERR_TIMEOUT     7  /* a kernel pipeline wait gave up (see qlora_check_status) */
#define QLORA_ERR_WORKSPACE   8  /* workspace missing or smaller than *_workspace_size() */
#define QLORA_ERR_SCRATCH_LIMIT 9 /* problem needs more than the built-in scratch of the no-allocation call */

/* Output dtypes of the linear layer. */
#define QLORA_DTYPE_F32  0
#define QLORA_DTYPE_BF16 1

#define QLORA_BLOCK     64   /* first-level block (NF4 absmax), walkthrough §1 */
#define QLORA_DQ_BLOCK  256  /* second-level block (FP8 constants), walkthrough §3 */
#define QLORA_MAX_RANK  256

/* A blockwise-quantized NF4 weight, W^T[o][h] (all pointers device,
 * read-only).
 *   codes      : uint8 [o*h/2]; element 2k in the high nibble of byte k.
 *   Double-quantized constants (walkthrough §3; absmax == NULL):
 *   absmax_fp8 : uint8 [o*h/64]; FP8 E4M3 code of each block's centred,
 *                scaled absmax.
 *   dq_scale   : fp32 [o*h/64/256]; absmax of the centred constants of each
 *                group of 256 blocks.
 *   dq_mean    : fp32 [1]; mean of all first-level constants.
 *   codebook   : the 16 code values (host copy, by value).
 *   block must be 64; dq_block must be 256 when the constants are
 *   double-quantized (o*h then a multiple of 64 * 256).
 *   absmax     : single-level constants instead (the scheme §3 compares
 *                double quantization with: one fp32 constant per block of 64,
 *                32/64 = 0.5 bit per parameter): fp32 [o*h/64], the block
 *                absmax as qlora_quantize_nf4 writes it.  When non-NULL the
 *                block constant is absmax[b] itself, absmax_fp8 / dq_scale /
 *                dq_mean / dq_block are ignored (may be NULL / 0) and o*h need
 *                only be a multiple of 64.  Appended last, so the layout of
 *                the fields before it is unchanged.                         */
typedef struct qlora_nf4_t {
    const uint8_t* codes;
    const uint8_t* absmax_fp8;
    const float*   dq_scale;
    const float*   dq_mean;
    int64_t        o;
    int64_t        h;
    float          codebook[16];
    int32_t        block;
    int32_t        dq_block;
    const float*   absmax;
} qlora_nf4_t;

/* Human-readable name of a status code (static string). */
const char* qlora_status_string(int status);

/* Library version, as major*10000 + minor*100 + patch. */
int qlora_version(void);

/* qlora_nf4_codebook - host-only: the 16 NF4 code values (walkthrough §2,
 * NF4; neura.market "How It Works"): standard-normal quantiles at evenly
 * spaced probabilities between delta = ((1 - 1/30) + (1 - 1/32)) / 2 and 1/2,
 * 8 for the positive half and 7 for the negative half, plus an exact zero,
 * divided by the largest so that they span [-1, 1]; fp32, increasing.
 *   out : host fp32[16].  Needs no GPU.                                     */
int qlora_nf4_codebook(float* out);

/* qlora_quantize_nf4 - blockwise absmax NF4 quantization
 * (walkthrough §1 Int8 absmax equation with the NF4 codebook of §2).
 *   W        : bf16 [n], finite values (not checked), any 16-byte-aligned
 *              flat tensor (the weight in W^T[o][h] order).
 *   n        : element count, n > 0, n % 64 == 0.
 *   codebook : host fp32[16], strictly increasing, finite, exactly one 0.0.
 *   block    : must be 64.
 *   codes    : out uint8 [n/2], code of element 2k in the high nibble.
 *   absmax   : out fp32 [n/64], c[b] = max |W| over block b.
 * Per element x = fp32(w / c) (IEEE round-to-nearest division) and the code is
 * the number of thresholds t_j = fp32((q_j + q_{j+1}) / 2) strictly below x:
 * the nearest code value, ties to the lower code.  An all-zero block has
 * c = 0 and every code equal to the index of 0.0.                          */
int qlora_quantize_nf4(const void* W, int64_t n, const float* codebook, int block,
                       uint8_t* codes, float* absmax, void* stream);

/* qlora_double_quant - double quantization of the block constants (§3).
 *   absmax     : fp32 [nblocks] from qlora_quantize_nf4.
 *   nblocks    : > 0, nblocks % 256 == 0.
 *   dq_block   : must be 256.
 *   absmax_fp8 : out uint8 [nblocks]; E4M3, round-to-nearest-even, saturating.
 *   dq_scale   : out fp32 [nblocks/256].
 *   dq_mean    : out fp32 [1].
 *   ws         : device workspace of qlora_double_quant_workspace_size() bytes.
 * mu = fp32(fp64(sum c) / nblocks); d = fp32(c - mu); dq_scale = max |d| per
 * group; code = E4M3(fp32(d * fp32(448 / dq_scale))), zeros for a group whose
 * dq_scale is 0.  The fp64 sum is exact (so independent of summation order)
 * when the constants span fewer than 45 - log2(nblocks) binades, which holds
 * for any realistic weight tensor; outside that range the last bit of mu may
 * depend on the order of summation.                                         */
size_t qlora_double_quant_workspace_size(int64_t nblocks, int dq_block);
int qlora_double_quant(const float* absmax, int64_t nblocks, int dq_block,
                       uint8_t* absmax_fp8, float* dq_scale, float* dq_mean,
                       void* ws, size_t ws_bytes, void* stream);

/* qlora_dequant - doubleDequant (key-formula section):
 *   c'   = fp32(fp32(E4M3(e) * fp32(dq_scale / 448)) + mu)
 *          (c' = absmax[b] for single-level constants)
 *   W'_i = bf16_rn(fp32(q[code_i] * c'))
 *   out  : bf16 [o*h], same order as the codes (W^T[o][h]).
 * Requires o*h % 16384 == 0 (whole DQ groups) for double-quantized
 * constants.  Every linear-layer entry point below accepts both forms.     */
int qlora_dequant(const qlora_nf4_t* Wq, void* out, void* stream);

/* qlora_linear_fwd - QLoRA linear forward, Y = X W' + s (X L1) L2
 * (LoRA equation of the walkthrough's background section; key formula).
 *   X      : bf16 [M][h] row-major.        M >= 1.
 *   L1     : bf16 [h][r],  L2 : bf16 [r][o].   8 <= r <= 256, r % 8 == 0.
 *   s      : LoRA scale (alpha / r).
 *   Y      : out [M][o], fp32 (QLORA_DTYPE_F32) or bf16 (QLORA_DTYPE_BF16).
 *   T_save : optional out fp32 [M][r] = X L1 (pass it to qlora_linear_bwd to
 *            skip recomputing it), or NULL.
 *   ws     : device workspace of qlora_linear_fwd_workspace_size() bytes
 *            (at least qlora_linear_fwd_workspace_min_size(); see below).
 * Requires h % 64 == 0, o % 64 == 0, and all pointers 16-byte aligned.
 * W' is bf16, the compute type of the data-type table, on every path; products
 * are bf16 x bf16 accumulated in fp32 on the tensor cores; X L1 is kept in fp32
 * and enters the accumulation of M > 32 tokens as a high + low bf16 pair.
 * For M >= 1024 qlora_linear_fwd_workspace_size() includes o*h*2 bytes for W':
 * given that much, the call dequantizes W' once into the workspace (as
 * qlora_dequant) and a bf16 tensor-core GEMM on SM pairs streams it, which is
 * faster at many tokens; given only the minimum workspace, and for M < 1024,
 * W' is dequantized on the fly inside the GEMM, tile by tile, and never
 * materialised.  Both paths form the same W' and accumulate the same products
 * in fp32 (in stages of different depth).  Calls with M <= 32 (decode)
 * take a memory-bound path that streams the NF4 weight once and splits the
 * reduction over all SMs (fp32 partial sums added atomically, so the last bits
 * of Y may vary from run to run; so may those of T_save for 17 <= M <= 32,
 * whose X L1 is split over K the same way; for M <= 16 its per-CTA partials
 * are summed in a fixed order, and the LoRA term s T L2 is formed in fp32 from
 * fp32 T and the bf16 L2).                                                  */
size_t qlora_linear_fwd_workspace_size(int64_t o, int64_t h, int64_t M, int r);
size_t qlora_linear_fwd_workspace_min_size(int64_t o, int64_t h, int64_t M, int r);
int qlora_linear_fwd(const qlora_nf4_t* Wq, const void* X, int64_t M,
                     const void* L1, const void* L2, int r, float s,
                     void* Y, int y_dtype, float* T_save,
                     void* ws, size_t ws_bytes, void* stream);

/* qlora_linear_bwd - QLoRA linear backward (training flow, step 5): with
 * U = dY L2^T and T = X L1,
 *   dX  = dY W'^T + s U L1^T        (gradient through the frozen weight)
 *   dL1 = s X^T U                   ([h][r], fp32)
 *   dL2 = s T^T dY                  ([r][o], fp32)
 * and no gradient for W.
 *   dY      : bf16 [M][o].
 *   T_saved : fp32 [M][r] from qlora_linear_fwd, or NULL to recompute X L1.
 *   dX      : out [M][h], fp32 or bf16 (dx_dtype).
 *   dL1/dL2 : out fp32, overwritten.
 *   ws      : device workspace of qlora_linear_bwd_workspace_size() bytes
 *             (at least qlora_linear_bwd_workspace_min_size()).
 * Same shape and alignment rules, and the same two paths for dY W'^T (chosen
 * by M and the workspace size), as qlora_linear_fwd.                        */
size_t qlora_linear_bwd_workspace_size(int64_t o, int64_t h, int64_t M, int r);
size_t qlora_linear_bwd_workspace_min_size(int64_t o, int64_t h, int64_t M, int r);
int qlora_linear_bwd(const qlora_nf4_t* Wq, const void* X, const void* dY, int64_t M,
                     const void* L1, const void* L2, int r, float s,
                     const float* T_saved, void* dX, int dx_dtype,
                     float* dL1, float* dL2,
                     void* ws, size_t ws_bytes, void* stream);

/* qlora_linear_fwd_dropout / qlora_linear_bwd_dropout - the same layer with
 * LoRA dropout on the adapter input (walkthrough "训练与推理流程": dropout
 * 0.1 for 7B/13B and 0.05 for 33B/65B on all linear layers).  With keep mask
 * K (one bit per element of X) and scale c = fp32(1 / (1 - p)):
 *   T  = c (X * K) L1,   Y = X W' + s T L2          (the base path keeps X)
 *   dX = dY W'^T + s c K * (U L1^T),  dL1 = s c (X * K)^T U,  dL2 = s T^T dY
 * Element i = m h + k of X is kept when word i % 4 of Philox4x32-10 (Salmon
 * et al., SC 2011) at counter (i / 4 low 32 bits, i / 4 high 32 bits, 0, 0)
 * under key (seed low 32 bits, seed high 32 bits) is at least
 * floor(p 2^32), p taken as the fp32 value passed.  The backward must get the
 * forward's p and seed; draw a new seed per layer and step.  p in [0, 1)
 * (else QLORA_ERR_UNSUPPORTED); p = 0 gives the plain calls' results.  T_save
 * / T_saved hold the dropped and scaled T.  Other arguments, shapes and
 * outputs as qlora_linear_fwd / qlora_linear_bwd; the workspaces are larger
 * (the backward adds M*h*6 bytes: the masked X and an fp32 dX accumulator).
 * In the backward the masked LoRA term of dX is added to dY W'^T by a
 * separate tensor-core product instead of sharing its accumulator.         */
size_t qlora_linear_fwd_dropout_workspace_size(int64_t o, int64_t h, int64_t M, int r);
size_t qlora_linear_bwd_dropout_workspace_size(int64_t o, int64_t h, int64_t M, int r);
size_t qlora_linear_fwd_dropout_workspace_min_size(int64_t o, int64_t h, int64_t M, int r);
size_t qlora_linear_bwd_dropout_workspace_min_size(int64_t o, int64_t h, int64_t M, int r);
int qlora_linear_fwd_dropout(const qlora_nf4_t* Wq, const void* X, int64_t M,
                             const void* L1, const void* L2, int r, float s,
                             float p, uint64_t seed,
                             void* Y, int y_dtype, float* T_save,
                             void* ws, size_t ws_bytes, void* stream);
int qlora_linear_bwd_dropout(const qlora_nf4_t* Wq, const void* X, const void* dY, int64_t M,
                             const void* L1, const void* L2, int r, float s,
                             float p, uint64_t seed,
                             const float* T_saved, void* dX, int dx_dtype,
                             float* dL1, float* dL2,
                             void* ws, size_t ws_bytes, void* stream);

/* Paged optimizer for the LoRA parameters (walkthrough §4 "Paged Optimizer"
 * and "训练" step 6; neura.market "How It Works"): the optimizer state lives
 * in NVIDIA unified memory, which the driver pages between device and host
 * RAM, so a memory spike moves it to the host instead of failing; the update
 * touches it again on the device.  These four calls are the one place where
 * the library allocates: unified memory is the point of the component.
 *   qlora_paged_alloc    : *ptr = unified (managed) memory of `bytes` bytes,
 *                          reachable from host and device.
 *   qlora_paged_free     : frees it (NULL is a no-op).
 *   qlora_paged_advise   : preferred location of [ptr, ptr + bytes): host RAM
 *                          (prefer_host != 0) or the current device; the
 *                          current device keeps a mapping either way.
 *   qlora_paged_prefetch : moves the range to host RAM (to_host != 0) or to
 *                          the current device, ordered on `stream`.       */
int qlora_paged_alloc(size_t bytes, void** ptr);
int qlora_paged_free(void* ptr);
int qlora_paged_advise(void* ptr, size_t bytes, int prefer_host);
int qlora_paged_prefetch(void* ptr, size_t bytes, int to_host, void* stream);

/* AdamW hyper-parameters; step counts from 1.  The pages' recipe: Adam
 * beta2 = 0.999, max grad norm 0.3, a constant learning rate.              */
typedef struct qlora_adamw_t {
    float   lr;
    float   beta1;
    float   beta2;
    float   eps;
    float   weight_decay;
    float   max_grad_norm;
    int32_t step;
} qlora_adamw_t;

/* qlora_grad_sqnorm - *acc += sum g[i]^2 over n fp32 gradients (fp64 sum;
 * acc 8-byte aligned, zeroed by the caller before the first tensor), so that
 * one accumulator collects the global norm of all LoRA gradients.
 * qlora_adamw_step - one AdamW step of n fp32 master parameters (device or
 * unified memory):
 *   g <- g min(1, max_grad_norm / (sqrt(*sqnorm) + 1e-6))   (if sqnorm given)
 *   p <- p (1 - lr wd);  m <- m + (1 - b1)(g - m);  v <- b2 v + (1 - b2) g^2
 *   p <- p - lr / (1 - b1^t) * m / (sqrt(v) / sqrt(1 - b2^t) + eps)
 * in fp32 (the bias corrections in fp64, rounded once); param_bf16
 * (nullable) receives bf16(p), the adapter copy the linear layer reads.  The
 * gradient is not modified.                                                */
int qlora_grad_sqnorm(const float* g, int64_t n, double* acc, void* stream);
int qlora_adamw_step(float* param, const float* grad, float* m, float* v, uint16_t* param_bf16,
                     int64_t n, const qlora_adamw_t* hp, const double* sqnorm, void* stream);

/* qlora_merge_bf16 - merge the trained adapter into the 16-bit dequantized
 * base (QLoRA glossary, pitfalls entry: merge into the bf16 dequantized base,
 * never into the 4-bit codes; walkthrough "推理": the adapter can also stay
 * separate, which qlora_linear_fwd does):
 *   W_m = W' + s L1 L2,  stored like the weight as W_m^T[o][h] in bf16:
 *   out[n][k] = bf16_rn(fp32(W'^T[n][k] + fp32(s * sum_j L1[k][j] L2[j][n])))
 * with W' the doubleDequant of Wq (rounded to bf16 as qlora_dequant does) and
 * the rank-r sum accumulated in fp32 on the tensor cores.  A forward with the
 * merged weight, X W_m, then equals Y of qlora_linear_fwd up to the bf16
 * rounding of W_m.
 *   L1 : bf16 [h][r],  L2 : bf16 [r][o],  8 <= r <= 256, r % 8 == 0.
 *   out: bf16 [o*h] (W^T order), 16-byte aligned; o % 64 == 0.
 * Same weight rules as qlora_dequant (either form of constants).            */
int qlora_merge_bf16(const qlora_nf4_t* Wq, const void* L1, const void* L2, int r, float s,
                     void* out, void* stream);

/* qlora_linear_fwd_noalloc - the forward pass for callers that cannot
 * allocate device memory.  No counterpart in the paper: this is a deployment
 * variant of qlora_linear_fwd.
 *
 * Some hosts give a kernel only its input and output buffers and no way to
 * obtain scratch memory: plug-in interfaces that hand over fixed tensors, or
 * runtimes whose device memory is planned in advance so that nothing may call
 * cudaMalloc while a step runs.  This call takes the same arguments as
 * qlora_linear_fwd minus the workspace, and uses instead a scratch array
 * compiled into the library (a file-scope __device__ array of
 * QLORA_NOALLOC_SCRATCH_BYTES = 8 MiB).  Every GPU on which the library is
 * loaded holds that array until the process exits.
 *   - Limit: problems whose qlora_linear_fwd_workspace_min_size(o, h, M, r)
 *     is larger than QLORA_NOALLOC_SCRATCH_BYTES are rejected with
 *     QLORA_ERR_SCRATCH_LIMIT before anything is launched (for example
 *     o = h = 4096, r = 64 fits up to M = 12288 tokens).  Calls whose W'
 *     does not fit beside that minimum take the on-the-fly dequant path.
 *   - The first call on a device looks up the array's device address with
 *     that device current (cudaGetSymbolAddress) and caches it; make that
 *     first call before any stream capture.  The cached address lives as long
 *     as the device's primary context: after cudaDeviceReset (or any other
 *     teardown of that context) this entry point must not be called again in
 *     the same process.
 *   - It calls no cudaMalloc, cudaFree or other allocating routine.
 *   - All calls share the one array, which keeps the previous call's
 *     contents; the call clears what must start at zero.  Calls that overlap
 *     on the GPU (different streams, or different host threads without an
 *     ordering between them) race on the array: order them on one stream.
 * Status codes, outputs and numerics are those of qlora_linear_fwd.       */
#define QLORA_NOALLOC_SCRATCH_BYTES (8u * 1024u * 1024u)
int qlora_linear_fwd_noalloc(const qlora_nf4_t* Wq, const void* X, int64_t M,
                             const void* L1, const void* L2, int r, float s,
                             void* Y, int y_dtype, float* T_save, void* stream);

/* qlora_debug_wait_tags - failure diagnosis (no counterpart in the method):
 * waits for the device, then returns and clears the set of pipeline waits
 * that gave up since the last call, one bit per wait site (the bit numbers
 * are listed beside the waits in the kernel sources); 0 when none did,
 * 0xFFFFFFFF if the query itself failed.                                   */
unsigned int qlora_debug_wait_tags(void);

/* qlora_debug_wait_probe - failure-path test (no counterpart in the method):
 * launches one tiny kernel whose single pipeline wait is on a barrier that
 * nothing ever completes, bounded by limit_ns (1 us .. 1 s) instead of the
 * pipelines' limit.  It holds no copy or MMA in flight, gives up after the
 * limit and returns, exactly as a stalled pipeline wait does: afterwards
 * qlora_check_status() reports QLORA_ERR_TIMEOUT and qlora_debug_wait_tags()
 * has bit 30 set; both are cleared by reading them.  Returns
 * QLORA_ERR_UNSUPPORTED for a limit outside the range.                     */
int qlora_debug_wait_probe(uint64_t limit_ns, void* stream);

/* qlora_check_status - waits for `stream`, then reports and clears the
 * library's device status word: QLORA_ERR_TIMEOUT if a kernel pipeline wait
 * gave up since the last check (the kernel then skipped its remaining work and
 * its outputs are undefined), QLORA_ERR_CUDA if the stream holds a CUDA error,
 * else QLORA_OK.                                                            */
int qlora_check_status(void* stream);

/* Kernel families, for launch tracing. */
#define QLORA_KERNEL_QUANTIZE     0  /* nf4 quantize */
#define QLORA_KERNEL_DOUBLE_QUANT 1  /* mean reduction + FP8 encode */
#define QLORA_KERNEL_DEQUANT      2  /* doubleDequant to bf16 */
#define QLORA_KERNEL_FUSED_FWD    3  /* X W' (+ LoRA stages), forward: the fused dequant-GEMM, or
                                       (1024+ tokens) the pair-tile bf16 GEMM */
#define QLORA_KERNEL_FUSED_BWD    4  /* dY W'^T (+ LoRA stages), backward dX: same two kernels */
#define QLORA_KERNEL_TGEMM        5  /* rank-r products T, U, dL1, dL2 */
#define QLORA_KERNEL_AUX          6  /* LoRA operand packing and hi/lo split */
#define QLORA_KERNEL_SMALL_M      7  /* small-M (decode) forward */
#define QLORA_KERNEL_MERGE        8  /* adapter merge into the bf16 base */
#define QLORA_KERNEL_OPTIM        9  /* LoRA optimizer step (gradient norm, AdamW) */
#define QLORA_KERNEL_WPRIME       10 /* W' dequantized into a linear call's workspace (1024+ tokens) */
#define QLORA_KERNEL_FAMILIES     11

/* Launch tracing (instrumentation, no counterpart in the method).
 * qlora_launch_count: kernels launched by this library since load.
 * qlora_trace_enable(1) clears old records and brackets every later launch
 * with two CUDA events on its stream; qlora_trace_enable(0) stops and clears.
 * qlora_trace_read waits for the recorded launches of one family, returns the
 * sum of their device times (ms) and their number, and forgets them.
 * Tracing is process-wide; enable it only around code you time.            */
int64_t qlora_launch_count(void);
void qlora_trace_enable(int on);
int qlora_trace_read(int family, double* total_ms, int64_t* launches);
const char* qlora_kernel_family_name(int family);

/* qlora_nf4_boundaries - host-only helper (no GPU needed): the per-absmax
 * decision table the quantizer uses.  For each of the 128 bf16 significands
 * m (absmax c = 1 + m/128) and each threshold j, out[m*16 + j] is the bf16 bit
 * pattern of the largest bf16 v with fp32(v / c) <= t_j (out[m*16 + 15] = 0).
 * code(w) = #{j : w > B_j} then equals the division rule above.  Exposed so
 * that the table can be checked on a CPU.                                   */
int qlora_nf4_boundaries(const float* codebook, uint16_t* out);

#ifdef __cplusplus
}
#endif

#endif /* QLORA_H */
