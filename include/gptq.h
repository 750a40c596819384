/*
 * gptq.h -- C ABI of a B200 (sm_100a) GPTQ layer quantizer.
 *
 * The library quantizes one linear layer W (d_row x d_col, columns = the
 * layer's inputs) with the GPTQ method as the GPTQ pages define it:
 *
 *   1. H = 2 X^T X over the calibration activations X (n x d_col), then
 *      H += lambda I   ("GPTQ (GPT Quantization)", "Algorithme complet
 *      (pseudo-code)", step 1; lambda = damp * mean(diag H), damp being the
 *      AutoGPTQ guide's damp_percent, "Quantizar seu proprio modelo").
 *   2. H^-1 through Cholesky (same pseudo-code, step 2), delivered as the
 *      upper factor U with H^-1 = U^T U.
 *   3. The columns are walked in blocks; each column is quantized with its
 *      group's asymmetric min-max scale and zero point (AutoGPTQ guide,
 *      "Quantizacao group-wise") and its error is fed to the later columns
 *      with the OBQ step W_F <- W_F - e_i / (H^-1)_ii * (H^-1)_{i,F}
 *      ("GPTQ (GPT Quantization)", "Fondation theorique : OBQ"): one column
 *      at a time inside a block, and as one matrix product per block for the
 *      remaining columns (the pseudo-code's "lazy update").
 *   4. Codes are packed into uint32 words, 8 per word at 4 bits ("GPTQ"
 *      article, "Desempenho e Precisao": 175B parameters at 4 bits, about
 *      87.5 GB, i.e. half a byte per weight).
 *
 * Conventions for every entry point:
 *   - All sizes are int64_t and all matrices row-major with the stated
 *     leading dimension (elements, not bytes).
 *   - Matrix arguments are DEVICE pointers to caller-owned memory; the
 *     library never allocates or frees device memory and keeps no pointer
 *     after a call returns.  `ws` is a caller-provided device workspace of at
 *     least gptq_workspace_size() bytes, 256-byte aligned.
 *   - Every call is asynchronous on `stream` (0 = legacy default stream).
 *     Argument errors are returned synchronously before anything is launched.
 *     Errors detected on the device (a non-positive-definite H, a bounded
 *     wait that ran out) are written to `*dev_status` (a device int32 that
 *     the caller zeroes once; the first error written is kept), readable with
 *     gptq_sync_status() after the work has run.  A nonzero status means the
 *     outputs of that call are not valid.
 *   - Calls on the same stream are ordered; calls that share buffers on
 *     different streams must be ordered by the caller.
 *   - gptq_hessian_accumulate, gptq_prepare_hinv, gptq_quantize_layer and
 *     gptq_pack may be captured in a CUDA graph (stream capture on `stream`);
 *     the library's own streams join the capture through its events.  The
 *     first gptq_prepare_hinv and gptq_hessian_accumulate_host calls on a
 *     device create those streams and events, so make them outside capture.
 */
#ifndef GPTQ_B200_GPTQ_H
#define GPTQ_B200_GPTQ_H

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum gptq_status {
    GPTQ_OK = 0,
    GPTQ_ERR_INVALID_ARG = 1,  /* a size, pointer, stride or config is invalid   */
    GPTQ_ERR_UNSUPPORTED = 2,  /* valid but not implemented (e.g. a group size)   */
    GPTQ_ERR_NOT_PD = 3,       /* damped H is not positive definite (device)      */
    GPTQ_ERR_TIMEOUT = 4,      /* a bounded device-side wait ran out (device)     */
    GPTQ_ERR_CUDA = 5,         /* a CUDA runtime call or kernel launch failed     */
    GPTQ_ERR_WORKSPACE = 6     /* ws is NULL, misaligned or smaller than needed   */
} gptq_status;

/* Quantizer settings (the AutoGPTQ guide's BaseQuantizeConfig, "Quantizar seu
 * proprio modelo" and "Configuracoes de quantizacao"). */
typedef struct gptq_config {
    int32_t bits;        /* code width: 2, 3, 4 or 8                                  */
    int32_t group_size;  /* weights per (scale, zero) group along d_col; -1 = one
                            group per row.  Supported: a divisor of block_size of
                            at least 8 (8, 16, 32, 64, 128), a multiple of
                            block_size (256, 1024, ...), or any value >= d_col.   */
    int32_t block_size;  /* columns per lazy-update block; must be 128               */
    int32_t desc_act;    /* nonzero: quantize columns by descending diag(H)          */
    float damp;          /* lambda = damp * mean(diag H); the guide's default 0.01   */
    int32_t pure_minmax; /* 0 (default): each group's range is widened to contain 0,
                            so zero points lie in [0, 2^bits - 1];  nonzero: the
                            group's own [min, max] (a one-signed group gets a finer
                            scale; its zero point may lie outside [0, 2^bits - 1],
                            its codes never do).  A constant group, or one whose
                            zero point would lie more than 2^20 levels away, uses
                            the widened range.                                    */
} gptq_config;

/* Human-readable text of a status code (static storage, never NULL). */
const char *gptq_status_string(int32_t status);

/* Library ABI version (major * 10000 + minor * 100 + patch); 200 added
 * gptq_config.pure_minmax. */
int32_t gptq_version(void);

/* Number of CUDA kernels this library has launched in this process since it
 * was loaded (a host-side counter, for benchmarks and diagnostics). */
int64_t gptq_launch_counter(void);

/*
 * Test hook for the bounded device-side waits (the pages have no counterpart;
 * it exists so the timeout path can be exercised without a faulty GPU).
 * Arms the NEXT launch of one kernel kind -- 1: the Hessian GEMM of
 * gptq_hessian_accumulate; 2: the next fp32-accurate tensor-core GEMM of any
 * call (gptq_prepare_hinv's first one is its first panel solve) -- so that
 * its MMA-issuing thread first waits, bounded by limit_ns (1 .. 10^9), on a
 * barrier that nothing completes.  That wait runs out like any other: the
 * kernel lets its issued copies and MMAs land (normal limit), frees its
 * tensor memory, writes GPTQ_ERR_TIMEOUT to the call's dev_status and
 * returns; the call's outputs are then not valid, later calls are
 * unaffected.  One launch consumes the arming.  Never needed in normal use.
 * Errors: GPTQ_ERR_INVALID_ARG for another kernel number or limit.
 */
gptq_status gptq_debug_arm_wait_probe(int32_t kernel, int64_t limit_ns);

/*
 * Workspace bytes needed by gptq_hessian_accumulate, gptq_prepare_hinv and
 * gptq_quantize_layer for a layer of d_row x d_col with this config (the
 * maximum over the three, so one workspace serves all of them).
 * Errors: GPTQ_ERR_INVALID_ARG for a NULL pointer, nonpositive sizes or an
 * invalid config; GPTQ_ERR_UNSUPPORTED for a config outside the supported set.
 */
gptq_status gptq_workspace_size(const gptq_config *cfg, int64_t d_row, int64_t d_col,
                                size_t *bytes);

/*
 * Stage 1 -- H += 2 X^T X  ("GPTQ (GPT Quantization)", pseudo-code step 1,
 * and the OBQ section's definition H = 2 X^T X).
 *   X     n x d bf16 (raw bit patterns), row-major, leading dimension ldx:
 *         ldx >= d, ldx a multiple of 8 and X 16-byte aligned (the tiles are
 *         fetched by the tensor-memory accelerator).
 *   H     d x d fp32, leading dimension ldh >= d.  Accumulated into: the
 *         caller zeroes H before the first chunk and may call repeatedly over
 *         token chunks.  Only the lower triangle (row >= col) is guaranteed;
 *         some upper-triangle entries near the diagonal are also written.
 *   Arithmetic: products of bf16 values are exact; sums are fp32 on the
 *   tensor cores.  Deterministic (no atomics).
 *   n == 0 is a no-op.  ws may be NULL (this stage needs none).
 */
gptq_status gptq_hessian_accumulate(const uint16_t *X, int64_t n, int64_t d, int64_t ldx,
                                    float *H, int64_t ldh, int32_t *dev_status,
                                    void *ws, size_t ws_bytes, cudaStream_t stream);

/*
 * Stage 1 with X in HOST memory -- H += 2 X^T X over the calibration tokens
 * ("GPTQ (GPT Quantization)", "Fondation theorique : OBQ": H = 2 X^T X, a sum
 * over tokens, so it may be accumulated chunk by chunk as the data arrives).
 *   X_host  n x d bf16 (raw bit patterns) in host memory, row-major with
 *           leading dimension ldx >= d, any alignment.  Pinned (page-locked)
 *           memory lets the copies overlap the GEMM; pageable memory is
 *           accepted but its copies are staged synchronously by the driver.
 *           The caller keeps X_host unchanged until the stream reaches the
 *           end of this call's work.
 *   H, ldh  as gptq_hessian_accumulate (accumulated into; lower triangle).
 *   staging caller-owned DEVICE buffer, 256-byte aligned, of at least
 *           gptq_hessian_staging_size(d, 64) bytes; split into two slots of
 *           `chunk` token rows each (chunk = the largest multiple of 32768
 *           tokens that fits, else of 64).  The copy engine fills one slot
 *           while the tensor cores read the other.  Its contents are
 *           scratch.
 *   Copies run on a stream the library owns (one per device) and are ordered
 *   after everything queued on `stream` before the call; every GEMM runs on
 *   `stream`, so work queued on `stream` afterwards sees the finished H.
 *   When chunk is a multiple of 32768 the result is bitwise identical to
 *   gptq_hessian_accumulate on the same X in device memory.
 *   Errors: GPTQ_ERR_INVALID_ARG (sizes, NULL X_host / H, ldx < d, ldh < d),
 *   GPTQ_ERR_WORKSPACE (staging NULL, misaligned or too small for 64 tokens).
 *   n == 0 is a no-op.
 */
gptq_status gptq_hessian_accumulate_host(const uint16_t *X_host, int64_t n, int64_t d,
                                         int64_t ldx, float *H, int64_t ldh, int32_t *dev_status,
                                         void *staging, size_t staging_bytes,
                                         cudaStream_t stream);

/* Staging bytes gptq_hessian_accumulate_host needs for chunks of
 * chunk_tokens tokens (rounded up to a multiple of 64) of a d-wide X; 0 for
 * invalid sizes. */
size_t gptq_hessian_staging_size(int64_t d, int64_t chunk_tokens);

/*
 * Stages 1b-2 -- dead columns, act-order, damping, and the inverse factor
 * ("GPTQ (GPT Quantization)", pseudo-code steps 1-2: H += lambda I,
 * H_inv = cholesky_inverse(H)).
 *   H     d x d fp32 (lower triangle read), leading dimension ldh.  Consumed:
 *         overwritten with scratch.  d and ldh must be multiples of 4 and H
 *         and U 16-byte aligned (tiles move by the tensor-memory accelerator),
 *         and d at most 57344 (the column walk's limit: U has no other use);
 *         otherwise GPTQ_ERR_UNSUPPORTED.
 *   U     d x d fp32, contiguous (leading dimension d).  Output: the upper
 *         triangular U with U^T U = (P^T H P + lambda I)^-1 in quantization
 *         order (P the act-order permutation); the strictly lower part is 0.
 *         Row i of U is row i of the OBQ-eliminated inverse divided by the
 *         square root of its pivot, so e / (H^-1)_ii * (H^-1)_{i,F} =
 *         (e / U_ii) * U_{i,F}.
 *   perm  int32[d] output: perm[k] = original column quantized k-th (the
 *         identity without desc_act; otherwise a stable sort by descending
 *         diag(H), ties by lower index).
 *   dead  uint8[d] output: 1 where diag(H) == 0 (that column is treated as
 *         H_ii = 1 and its weights as 0).
 *   Device errors: GPTQ_ERR_NOT_PD if a Cholesky pivot is not positive, or
 *   if a diagonal entry of H is not finite (NaN or infinite; perm is then
 *   still a permutation, with such columns ranked last under desc_act).
 */
gptq_status gptq_prepare_hinv(float *H, int64_t d, int64_t ldh, const gptq_config *cfg,
                              float *U, int32_t *perm, uint8_t *dead, int32_t *dev_status,
                              void *ws, size_t ws_bytes, cudaStream_t stream);

/*
 * Stages 3-4 -- the GPTQ column walk with OBQ error feedback.
 *   W       d_row x d_col fp32, leading dimension ldw, in ORIGINAL column
 *           order; any alignment (rows with a 16-byte aligned base and a
 *           pitch of a multiple of 4 floats take the vector and TMA paths).  Scratch: on return column k holds the weights of original
 *           column perm[k] as they were when quantized (after the feedback of
 *           every earlier column).
 *   U, perm, dead  the outputs of gptq_prepare_hinv for this layer's H (any
 *           number of layers sharing one H may reuse them), with the same
 *           desc_act: without act-order perm is the identity and is not read.
 *           A perm entry outside [0, d_col) is reported on the device as
 *           GPTQ_ERR_INVALID_ARG (and read as the identity).  d_col must be a
 *           multiple of 4 (GPTQ_ERR_UNSUPPORTED otherwise) and at most 57344.
 *   codes   d_row x d_col uint8, contiguous: codes[row][k] is the code of
 *           original column perm[k].
 *   scales  fp32 [ceil(d_col / g)][d_row] and zeros int32 (same shape),
 *           group-major, groups in quantization order.  Dequantization:
 *           W_hat[row][perm[k]] = scales[k/g][row] * (codes[row][k] - zeros[k/g][row]).
 *   ws      at least d_row * 512 bytes (GPTQ_ERR_WORKSPACE otherwise).  With
 *           gptq_workspace_size() bytes the lazy update defers up to 8 blocks
 *           and reads its operands' low-precision parts, split once, from the
 *           workspace (d_col^2 * 4 bytes for U's, as much again as the
 *           deferred errors for theirs); smaller workspaces defer fewer blocks
 *           and split in the GEMM.  The split values are the same, so for a
 *           given number of deferred blocks the results are identical.
 */
gptq_status gptq_quantize_layer(float *W, int64_t d_row, int64_t d_col, int64_t ldw,
                                const float *U, const int32_t *perm, const uint8_t *dead,
                                const gptq_config *cfg, uint8_t *codes, float *scales,
                                int32_t *zeros, int32_t *dev_status, void *ws,
                                size_t ws_bytes, cudaStream_t stream);

/*
 * gptq_quantize_layer without a workspace argument.  The GPTQ pages have no
 * counterpart to this entry point: it is a packaging variant of stages 3-4
 * for callers that cannot allocate device memory -- a plugin or operator
 * interface whose enqueue call may not allocate, a process whose memory pool
 * has already reserved nearly all of HBM, or a latency-critical path that
 * cannot afford cudaMalloc / cudaFree (both can synchronize the device).
 *   Arguments and results: exactly those of gptq_quantize_layer, minus ws /
 *   ws_bytes.  The scratch is one fixed device array inside this library of
 *   gptq_noalloc_scratch_bytes() bytes (16 MiB) per device, held by every GPU
 *   that loads the library until the process exits; no allocation is made.
 *   Limit: a layer whose gptq_quantize_layer workspace would exceed that
 *   array (currently d_row * 512 bytes, i.e. d_row <= 32768) is rejected with
 *   GPTQ_ERR_WORKSPACE before anything is launched.  The lazy update defers
 *   the errors of up to 8 blocks of 128 columns in the array (d_row * 512
 *   bytes each); above d_row = 4096 it defers fewer (4 up to 8192, 2 up to
 *   16384, 1 up to 32768), exactly as gptq_quantize_layer does with a 16 MiB
 *   workspace: the same sums grouped into more, shorter products (and, for
 *   layers whose full workspace fits the array, with the lazy update's
 *   operands split ahead, as gptq_quantize_layer does then).
 *   Device: the array used is the current device's, so W, U, perm (with
 *   act-order), dead, codes, scales, zeros and dev_status must be memory of
 *   the current device (or managed memory); otherwise GPTQ_ERR_INVALID_ARG
 *   is returned before anything is launched.
 *   Set-up: the first call on each device (with that device current) looks
 *   up the array's device address and caches it with the device's current
 *   context (a call in a new context, e.g. after cudaDeviceReset, looks it
 *   up again); make that first call before any stream capture on the device.
 *   Sharing: every call uses the same array, which keeps the last call's
 *   contents; nothing in it needs to start at zero.  Calls whose work overlaps
 *   on the GPU (e.g. on two unordered streams) race on the array: order them.
 */
gptq_status gptq_quantize_layer_noalloc(float *W, int64_t d_row, int64_t d_col, int64_t ldw,
                                        const float *U, const int32_t *perm,
                                        const uint8_t *dead, const gptq_config *cfg,
                                        uint8_t *codes, float *scales, int32_t *zeros,
                                        int32_t *dev_status, cudaStream_t stream);

/* Bytes of the fixed scratch array used by gptq_quantize_layer_noalloc. */
size_t gptq_noalloc_scratch_bytes(void);

/*
 * Stage 5 -- pack codes into each row's little-endian bit stream: code k of a
 * row occupies bits [bits*k, bits*k + bits) of the row's uint32 words, so at
 * 4 bits word m holds codes 8m..8m+7 (code 8m+t in bits 4t..4t+3).
 *   codes   d_row x d_col uint8, contiguous; values must be < 2^bits.
 *   packed  d_row x ceil(d_col * bits / 32) uint32, contiguous; a row's last
 *           word is zero-padded past its final code.
 */
gptq_status gptq_pack(const uint8_t *codes, int64_t d_row, int64_t d_col, int32_t bits,
                      uint32_t *packed, cudaStream_t stream);

/*
 * Using the quantized layer -- Y = X W_hat^T with the weights dequantized on
 * the fly ("GPTQ (GPT Quantization)", "Limitations", items 1-2: the
 * quantization is weight-only, the activations stay at 16 bits and the integer
 * weights are dequantized before each product).  Decode form: tokens are taken
 * 8 per launch and each launch streams the packed layer once, so it is meant
 * for a few tokens at a time.
 *   X       n_tok x d_col bf16 (raw bit patterns), row-major, leading
 *           dimension ldx >= d_col, in the layer's ORIGINAL column order.
 *   packed  d_row x (d_col * bits / 32) uint32, contiguous: gptq_pack output
 *           (codes in quantization order).
 *   scales, zeros  fp32 / int32 [ceil(d_col / g)][d_row], as
 *           gptq_quantize_layer writes them.
 *   perm    int32[d_col] from gptq_prepare_hinv (quantization position k holds
 *           original column perm[k]); NULL means the identity.  An entry
 *           outside [0, d_col) is read as k (no access leaves the row).
 *   Y       n_tok x d_row fp32, leading dimension ldy >= d_row (overwritten):
 *           Y[t][n] = sum_k X[t][perm[k]] * scales[k/g][n] * (code[n][k] - zeros[k/g][n]).
 *   Arithmetic: fp32 (per word, the dot of the token values with the codes
 *   and their plain sum; the group's scale and zero point enter once per word).
 *   ws      caller-owned device workspace, 256-byte aligned, of at least
 *           gptq_dequant_matmul_workspace_size(n_tok, d_col) bytes: the
 *           tokens gathered into quantization order (fp32), up to 8 at a time.
 *   Supported: bits 2, 4 or 8 (a word holds whole codes), d_col a multiple of
 *   32 / bits, group size -1, >= d_col or a multiple of 32 / bits (a word
 *   never spans two groups); otherwise GPTQ_ERR_UNSUPPORTED (3-bit codes
 *   straddle words).  Device pointers; n_tok == 0 is a no-op.
 *   Errors: GPTQ_ERR_INVALID_ARG for NULL pointers, bad sizes or strides,
 *   misaligned pointers or an invalid bits / group size; GPTQ_ERR_WORKSPACE
 *   for a missing, misaligned or small workspace.
 */
gptq_status gptq_dequant_matmul(const uint16_t *X, int64_t n_tok, int64_t d_col, int64_t ldx,
                                const uint32_t *packed, const float *scales, const int32_t *zeros,
                                const int32_t *perm, int64_t d_row, int32_t bits,
                                int32_t group_size, float *Y, int64_t ldy, void *ws,
                                size_t ws_bytes, cudaStream_t stream);

/* Workspace bytes gptq_dequant_matmul needs for n_tok tokens of a d_col-wide
 * layer; 0 for invalid sizes. */
size_t gptq_dequant_matmul_workspace_size(int64_t n_tok, int64_t d_col);

/*
 * Using the quantized layer, many-token (prefill) form -- Y = X W_hat^T on the
 * tensor cores ("GPTQ (GPT Quantization)", "Limitations", items 1-2: weights
 * dequantized to 16 bits before each product, activations at 16 bits).  Each
 * stage of 64 codes of a 256-row slice of the packed layer is dequantized
 * into a bf16 tile in shared memory and multiplied with the bf16 activations
 * (tcgen05, fp32 accumulation):
 *   W_hat[n][k] = bf16_rne( fp32 scales[k/g][n] * (code[n][k] - zeros[k/g][n]) )
 *   Y[t][n]     = sum_k X[t][perm[k]] * W_hat[n][k]
 * (the products of two bf16 values are exact; the sums are fp32).
 *   X, packed, scales, zeros, perm, Y, ldx, ldy  as gptq_dequant_matmul; packed
 *           16-byte aligned.
 *   dev_status  device int32 (may be NULL) receiving GPTQ_ERR_TIMEOUT if a
 *           bounded wait runs out.
 *   ws      caller-owned device workspace, 256-byte aligned, of at least
 *           gptq_dequant_gemm_workspace_size(n_tok, d_col) bytes, used when
 *           perm is given or X's rows are not 16-byte aligned (the tokens are
 *           gathered into quantization order as bf16); may be NULL otherwise.
 *   Supported: bits 2, 4 or 8; d_col a multiple of 64; group size -1, >= d_col
 *   or a multiple of 8; n_tok <= 2^24; otherwise GPTQ_ERR_UNSUPPORTED /
 *   GPTQ_ERR_INVALID_ARG.  n_tok == 0 is a no-op.  Deterministic.
 */
gptq_status gptq_dequant_gemm(const uint16_t *X, int64_t n_tok, int64_t d_col, int64_t ldx,
                              const uint32_t *packed, const float *scales, const int32_t *zeros,
                              const int32_t *perm, int64_t d_row, int32_t bits,
                              int32_t group_size, float *Y, int64_t ldy, int32_t *dev_status,
                              void *ws, size_t ws_bytes, cudaStream_t stream);

/* Workspace bytes gptq_dequant_gemm needs (n_tok x d_col bf16); 0 for invalid
 * sizes. */
size_t gptq_dequant_gemm_workspace_size(int64_t n_tok, int64_t d_col);

/*
 * Waits for `stream`, then copies the device status word to *out.
 * Returns GPTQ_ERR_CUDA if the wait or the copy fails, else GPTQ_OK (the
 * device-side status itself is in *out).
 */
gptq_status gptq_sync_status(cudaStream_t stream, const int32_t *dev_status, int32_t *out);

#ifdef __cplusplus
}
#endif

#endif /* GPTQ_B200_GPTQ_H */
