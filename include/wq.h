/*
 * wq.h -- C ABI of the B200 (sm_100a) group-wise weight-only quantization
 * library (libwq.so).
 *
 * The library quantizes fp16 weights group-wise to 3 or 4 bits, packs them in
 * the layout documented below, searches AWQ per-input-channel scales, and
 * runs the W4A16 / W3A16 matmul Y = X * W^T that dequantizes the packed
 * weights on the fly (fp16 activations, fp32 accumulation, fp16 output).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - W is an nn.Linear weight: [N][K] row-major fp16 (N output channels, K
 *    input channels). X is [M][K] row-major fp16, Y is [M][N] row-major fp16.
 *  - A group is `group_size` (32, 64 or 128) consecutive input channels of
 *    one output row ("Quantising Large Language Models for Efficient
 *    Inference", section "Post-training methods for 4-bit weights": one scale
 *    and zero point per group of 64-128 weights within a row; the Lab 5 linear
 *    of "MIT 6.5940 Lab 4 + Lab 5" uses 32).
 *  - Pointers named *_dev are device pointers the caller allocated (e.g. torch
 *    tensors' data_ptr()). The library never frees or retains them.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream). All device work is enqueued asynchronously on it; the host side
 *    validates arguments synchronously and returns before the work runs.
 *  - Argument errors are reported by the return value and enqueue nothing.
 *    Launch failures return WQ_ERR_CUDA. Conditions found on the device (a
 *    step that overflows fp16, a bounded wait that ran out) are latched in a
 *    per-device flag read by wq_get_last_device_error().
 *  - No entry point allocates device memory, except that the first call on a
 *    device looks up the address of the library's device error flag.
 *
 * Quantization contract (bit-exact; identical in the CPU oracle)
 * --------------------------------------------------------------
 *  fp16 inputs are widened exactly to fp32; with AWQ scales s, w' = w * s_k
 *  (exact). Asymmetric, Q = 2^b - 1 ("LLM Quantization: 160GB Model on a
 *  Laptop", section "Asymmetric Quantization", in the integer zero-point form
 *  of "CMU 11-868 L19-L20 Model Quantization", section "absmax and
 *  zero-point"):
 *     mn = min(min_g w', 0), mx = max(max_g w', 0), r = mx - mn      (fp32)
 *     step = (r == 0) ? 1 : fp16_round_toward_+inf(r / Q)          (fp32 div)
 *     zero = clamp(rint(-mn / step), 0, Q)
 *     q    = clamp(rint(w' / step) + zero, 0, Q)       rint: ties to even
 *  Symmetric, qmax = 2^(b-1) - 1 ("LLM Quantization: 160GB Model on a
 *  Laptop", section "Symmetric Quantization"):
 *     step = (max|w'| == 0) ? 1 : fp16_round_toward_+inf(max|w'| / qmax)
 *     q    = clamp(rint(w' / step), -qmax - 1, qmax) + 2^(b-1); zero = 2^(b-1)
 *  Both dequantize as (q - zero) * step. Steps and zeros are stored as fp16.
 *
 * Packed layouts (row-major over output rows; no padding between rows)
 * --------------------------------------------------------------------
 *  4-bit: uint32 [N][K/8]. Word c of a row holds k = 8c .. 8c+7; nibble slot
 *         j (bits 4j..4j+3) holds k = 8c+2j for j < 4 and k = 8c+2(j-4)+1
 *         for j >= 4 (slot order k0,k2,k4,k6,k1,k3,k5,k7), so that
 *         (word >> 4j) & 0x000F000F is the pair (k_2j, k_2j+1) in two 16-bit
 *         lanes. This is the GPU counterpart of the offline nibble reordering
 *         in "MIT 6.5940 Lab 4 + Lab 5", section "Background: why the 4-bit
 *         weights get reordered first".
 *  3-bit: uint32 [N][3K/32]. Three words t = 0,1,2 per 32 consecutive k:
 *         word t, pair j = 0..4: bits 3j..3j+2 hold k = 10t+2j, bits
 *         16+3j..18+3j hold k = 10t+2j+1; bit b of k = 30 is bit 15 of word b
 *         and bit b of k = 31 is bit 31 of word b. Exactly 3 bits per weight.
 *  steps, zeros: fp16 [N][K/group_size] row-major.
 *
 * Rows are independent: linears that read the same input (q|k|v, gate|up)
 * can be packed as one weight by concatenating their packed rows, steps and
 * zeros along N; one wq_w4a16_gemm call then writes all their outputs, in the
 * same column order, with fewer launches than one call per linear.
 *
 * Supported: bits in {3, 4}; group_size in {32, 64, 128} (the AWQ search:
 * 128); K % 128 == 0; N >= 1; M >= 1. Device pointers must be 16-byte aligned
 * (weights, X, packed words) or 4-byte aligned (steps, zeros, Y, s, mu).
 * Inputs must be finite.
 */
#ifndef WQ_H_
#define WQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define WQ_ABI_VERSION 1

typedef enum wq_status {
  WQ_OK = 0,
  WQ_ERR_INVALID_ARG = 1,  /* null pointer, non-positive size, bad config  */
  WQ_ERR_UNSUPPORTED = 2,  /* valid but not implemented (e.g. 2 or 8 bits)  */
  WQ_ERR_ALIGNMENT = 3,    /* a pointer is not aligned as required          */
  WQ_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed          */
  WQ_ERR_TIMEOUT = 5,      /* device: a bounded wait gave up                */
  WQ_ERR_WORKSPACE = 6,    /* workspace pointer null or smaller than needed */
  WQ_ERR_RANGE = 7         /* device: a step or scale is not finite in fp16 */
} wq_status;

typedef struct wq_quant_cfg {
  int32_t bits;        /* 3 or 4                                   */
  int32_t group_size;  /* 32, 64 or 128                            */
  int32_t symmetric;   /* 0: asymmetric zero point, 1: symmetric   */
} wq_quant_cfg;

/* ABI version of the loaded library (WQ_ABI_VERSION). */
/* Version of the packed layout documented above (codes, steps, zeros). A
 * stored quantized weight records it; a reader refuses another value. */
#define WQ_LAYOUT_VERSION 1
int32_t wq_layout_version(void);
int32_t wq_abi_version(void);

/* Static string for a status code. Never NULL. */
const char* wq_status_string(int32_t status);

/* Number of uint32 words of the packed weight for an [N][K] matrix
 * (N*K/8 for 4-bit, 3*N*K/32 for 3-bit); 0 if the config is invalid. */
size_t wq_packed_words(int64_t N, int64_t K, const wq_quant_cfg* cfg);

/* S3 -- quantize + pack.
 * Quantizes W_dev (fp16 [N][K]) group-wise per the contract above, after the
 * optional AWQ scaling W * diag(s) (s_dev: fp16 [K], or NULL for none;
 * "MIT 6.5940 Lab 4 + Lab 5", section "Question 2"), and writes packed_dev
 * (uint32, wq_packed_words(N,K,cfg) words), steps_dev and zeros_dev (fp16
 * [N][K/group_size] each). One kernel launch. A step that is not finite in fp16
 * (a group holding an infinite or NaN weight, or a range too large for fp16)
 * latches WQ_ERR_RANGE in the device flag; that group's codes are then
 * unspecified. */
int32_t wq_quantize_pack(const void* W_dev, const void* s_dev, int64_t N, int64_t K,
                         const wq_quant_cfg* cfg, uint32_t* packed_dev, void* steps_dev,
                         void* zeros_dev, void* stream);

/* Inverse of the packing: W_out_dev (fp16 [N][K]) = fp16_rn((q - zero) * step)
 * for every element. A check/test helper, not on the decode path. */
int32_t wq_unpack_dequant(const uint32_t* packed_dev, const void* steps_dev,
                          const void* zeros_dev, int64_t N, int64_t K,
                          const wq_quant_cfg* cfg, void* W_out_dev, void* stream);

/* Size in bytes of the optional matmul workspace for (M, N, K, cfg): the
 * tensor-core kernel's stream-K schedule (64 KB of arrival counters, then two
 * fp32 partial tiles of 128 x M rounded up to 16 per CTA of the persistent
 * grid); 0 when M < 3 (the GEMV kernels take none) or the config is
 * invalid. The matmul runs without it as well. */
size_t wq_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K, const wq_quant_cfg* cfg);

/* S5/S6 -- weight-only matmul Y = X * deq(W)^T.
 * X_dev fp16 [M][K]; packed_dev/steps_dev/zeros_dev as written by
 * wq_quantize_pack; Y_dev fp16 [M][N] (overwritten). Products are exact in
 * fp32 and accumulated in fp32 ("Quantising Large Language Models",
 * section "Weight-only vs weight-and-activation quantisation": weights are
 * dequantized on the fly inside the matmul; "TinyChat (AWQ on-device
 * runtime)", "Notable features": fused dequant + GEMM). Small M runs a
 * bandwidth-bound GEMV kernel that streams the packed weights once; larger M
 * (3- and 4-bit) runs a tcgen05 tensor-core kernel. X must already be
 * multiplied by diag(s)^-1 when the weight was packed with AWQ scales s.
 * workspace_dev is optional: NULL, or device memory of at least
 * wq_gemm_workspace_bytes(M, N, K, cfg) bytes, 256-byte aligned and
 * zero-filled before its first use. Given it, the tensor-core kernel balances
 * its work over all SMs (stream-K: every CTA of a persistent grid takes the
 * same number of K stages, at most one row tile's worth; a tile split between
 * CTAs is summed from their fp32 partial tiles in CTA order, so the result
 * does not depend on timing) for M <= 16 (WQ_OPT_TC_STREAMK). Its first
 * 64 KB hold arrival counters that every completed call leaves at zero, so
 * calls of any
 * shape may share one workspace as long as they do not overlap in time (same
 * stream); after a call that ended in WQ_ERR_TIMEOUT, zero-fill it again.
 * Without a workspace: one CTA per row tile (and K split over thread-block
 * clusters when the tiles leave SMs idle). The same weight, X and workspace
 * size give the same Y on every call. wq_gemm_workspace_bytes is 0 for M < 3. */
int32_t wq_w4a16_gemm(const void* X_dev, const uint32_t* packed_dev, const void* steps_dev,
                      const void* zeros_dev, int64_t M, int64_t N, int64_t K,
                      const wq_quant_cfg* cfg, void* Y_dev, void* workspace_dev,
                      size_t workspace_bytes, void* stream);

/* S1/S2/S4 -- AWQ activation-aware scale search for the linears that share
 * one input ("MIT 6.5940 Lab 4 + Lab 5", sections "Starting point and setup"
 * and "Question 2"; the loss is the layer-output reconstruction error of
 * "CMU 11-868 L19-L20 Model Quantization", section "Quantizing during
 * training vs. after it").
 *   X_dev      fp16 [T][K] calibration inputs of the linears
 *   W_dev[i]   host array of n_lin (1..8) device pointers, fp16 [N_i[i]][K]
 *   alpha      host array of n_alpha (1..64) exponents (e.g. j/20, j < 20)
 * Computes mu_k = sum_t |x_tk| / T (fp64, exact sum), candidates
 * s_j,k = fp16_rn(max(mu_k, 2^-14)^alpha_j), and for every j the loss
 * L_j = sum_i || X (W_i - Q(W_i diag s_j) diag(s_j)^-1)^T ||_F^2, where Q is
 * this library's quantize-dequantize with `cfg` (the loss GEMM runs on the
 * tensor cores with the error matrix in fp16 and fp32 accumulation; the
 * squares are summed in fp64 in a fixed order, so results are deterministic.
 * Against fp64 the losses come out low by about 2e-9 * K relative -- the
 * accumulator rounds toward zero -- nearly the same for every alpha).
 * cfg->group_size must be 128 (the pages' AWQ setting; else
 * WQ_ERR_UNSUPPORTED). Writes s_out_dev (fp16 [K]) = s_best with best = the
 * first index of the smallest L_j; optionally mu_out_dev (fp64 [K]), loss_out_dev (fp64
 * [n_alpha]) and best_out_dev (int32, device). Quantize the weights with
 * wq_quantize_pack(W, s_out) and feed the matmul X * diag(s)^-1 afterwards.
 * workspace_dev: >= wq_awq_workspace_bytes(...) bytes, 256-byte aligned, no
 * initial contents required. The size depends on WQ_OPT_AWQ_LOSS when it is
 * asked for: the two-kernel path keeps the error matrices of a batch of
 * alphas (up to 1 GiB), the fused path none; a workspace too small for the
 * path selected at the call returns WQ_ERR_WORKSPACE. A non-finite
 * candidate or loss latches WQ_ERR_RANGE in the device flag. */
size_t wq_awq_workspace_bytes(int64_t T, int64_t K, const int64_t* N_i, int32_t n_lin, int32_t n_alpha,
                              const wq_quant_cfg* cfg);
int32_t wq_awq_scale_search(const void* X_dev, int64_t T, int64_t K, const void* const* W_dev,
                            const int64_t* N_i, int32_t n_lin, const wq_quant_cfg* cfg,
                            const double* alpha, int32_t n_alpha, void* s_out_dev, double* mu_out_dev,
                            double* loss_out_dev, int32_t* best_out_dev, void* workspace_dev,
                            size_t workspace_bytes, void* stream);

/* The AWQ search of wq_awq_scale_search without a caller workspace.
 * No counterpart on the pages: an interface addition for callers that
 * cannot allocate device memory -- code hosted by a framework that owns every
 * device allocation (plugin hosts, fixed memory pools), or paths where the
 * device-wide synchronization cudaMalloc may imply is not acceptable. The
 * caller still passes every input and output buffer, with the meanings of
 * wq_awq_scale_search; the results are the same (same kernels; alphas are
 * processed one at a time and the error matrix is built in row chunks).
 * Scratch: one 24 MiB array in the library's own device memory (a file-scope
 * static device variable). Every GPU that loads the library holds it until
 * the process exits. The first call on a device looks up the array's device
 * address with that device current and keeps it for the life of the
 * process; make that first call before any stream capture, and do not use
 * the library on a device after cudaDeviceReset (or any teardown of its
 * primary context) -- the kept address would no longer be valid. With the
 * default fused loss path only the per-tile partial losses live in the
 * array; the two-kernel path also builds the error matrix there, one alpha
 * and at most 16 MiB of rows at a time. All calls share the array, which
 * keeps the last call's contents (nothing in it has to start at zero), so
 * calls that overlap on the GPU --
 * from other streams or threads -- race and must be serialized by the caller.
 * Limits: K <= 16384, n_alpha <= 64 and
 * n_alpha * ceil(T/128) * ceil(sum_i N_i / 128) <= 786432; a larger problem
 * returns WQ_ERR_WORKSPACE and enqueues nothing. Calls no cudaMalloc, no
 * cudaFree and no allocating library routine. */
int32_t wq_awq_scale_search_noalloc(const void* X_dev, int64_t T, int64_t K, const void* const* W_dev,
                                    const int64_t* N_i, int32_t n_lin, const wq_quant_cfg* cfg,
                                    const double* alpha, int32_t n_alpha, void* s_out_dev,
                                    double* mu_out_dev, double* loss_out_dev, int32_t* best_out_dev,
                                    void* stream);

/* W4A8 -- 4-bit weights and 8-bit activations, one scale per group of
 * channels for each ("MIT 6.5940 Lab 4 + Lab 5", section "The five
 * implementation files and grading": the Lab 5 linear is W4A8 with group size
 * 32; the activation codes are the int8 absmax form of "CMU 11-868 L19-L20
 * Model Quantization", section "absmax and zero-point", per group).
 *   wq_quantize_act_int8  X_dev fp16 [M][K] -> q_dev int8 [M][K] and mult_dev
 *       fp32 [M][K/group]: per row and group, mult = 127 / max|x| (fp32
 *       division; 1 for an all-zero group), q = rint(x * mult) (fp32, ties to
 *       even) clipped to [-127, 127]. group in {32, 64, 128}, K % group == 0.
 *   wq_w4a8_gemm  Y[m][n] = sum_g (step[n][g] / mult[m][g]) *
 *       sum_{k in g} (q_w[n][k] - zero[n][g]) * q[m][k]: exact integer dot
 *       products per group (dp4a), scaled and summed in fp32, Y fp16 [M][N].
 *       The weight is wq_quantize_pack's 4-bit layout with cfg->group_size
 *       equal to the activations' group; K <= 16384 (else
 *       WQ_ERR_UNSUPPORTED); q_dev 16-byte aligned.
 *       K <= 8192 runs the row-streaming GEMV (each lane's 32 codes of every
 *       row of X in registers; with WQ_OPT_PDL on, the same rule on the
 *       weight's writer as wq_w4a16_gemm), larger K a kernel that holds the
 *       codes in shared memory.
 * Asynchronous on `stream`, one launch each (wq_w4a8_gemm: one per 4 rows of
 * M). */
int32_t wq_quantize_act_int8(const void* X_dev, int64_t M, int64_t K, int32_t group, int8_t* q_dev,
                             float* mult_dev, void* stream);
int32_t wq_w4a8_gemm(const int8_t* q_dev, const float* mult_dev, const uint32_t* packed_dev,
                     const void* steps_dev, const void* zeros_dev, int64_t M, int64_t N, int64_t K,
                     const wq_quant_cfg* cfg, void* Y_dev, void* stream);

/* GPTQ -- quantize + pack with error feedback ("CMU 11-868 L19-L20 Model
 * Quantization", sections "The algorithm in four steps" and "Why it can
 * actually run: from OBS to GPTQ"), writing the same packed layout, steps
 * and zeros as wq_quantize_pack, so the matmul takes the result as it is.
 *   X_dev  fp16 [T][K] calibration inputs of the linear
 *   W_dev  fp16 [N][K] weight
 * Computes, in fp64 on the device: H = 2 X^T X + lambda I with lambda =
 * damp * mean(diag H) (damp >= 0, e.g. 0.01; an input channel that is zero
 * on every token gets H_kk = 1 and zero weights), G = Cholesky(H^-1)^T (upper,
 * H^-1 = G^T G), then the columns in order in blocks of 128: when a column
 * starts a group its step and zero point come from the group's current
 * weights by the quantizer's decisions above (on their fp32 values); the
 * column's codes; its error divided by G_kk, subtracted from the rest of the
 * block times G's row; after each block, every later column is updated by
 * the block's errors times G (one batched product).
 * workspace_dev: >= wq_gptq_workspace_bytes(N, K, cfg) bytes (two K x K fp64
 * matrices, the N x K fp64 running weights), 256-byte aligned, no initial
 * contents required. H not positive definite (only possible for damp == 0)
 * latches WQ_ERR_RANGE. Many small launches on `stream` (about 5 K / 64). */
size_t wq_gptq_workspace_bytes(int64_t N, int64_t K, const wq_quant_cfg* cfg);
int32_t wq_gptq_quantize_pack(const void* X_dev, int64_t T, const void* W_dev, int64_t N, int64_t K,
                              const wq_quant_cfg* cfg, double damp, uint32_t* packed_dev, void* steps_dev,
                              void* zeros_dev, void* workspace_dev, size_t workspace_bytes, void* stream);

/* AWQ scale folding ("MIT 6.5940 Lab 4 + Lab 5", section "Question 2": the
 * scales searched at each place are folded into the previous LayerNorm or
 * linear layer). After wq_awq_scale_search picked s for a set of linears and
 * they were packed with wq_quantize_pack(W, s), the op that produces their
 * input absorbs diag(s)^-1, so the matmul takes the unscaled activations:
 *   wq_awq_fold_norm         gamma_out[k] = gamma[k] / s[k]: the weight of a
 *                            normalisation layer (RMSNorm / LayerNorm scale)
 *                            feeding q/k/v or gate/up. fp16 [K] each.
 *   wq_awq_fold_linear_rows  W_out[n][k] = W[n][k] / s[n] and b_out[n] =
 *                            b[n] / s[n]: a linear whose output feeds the
 *                            scaled linear (v_proj before o_proj, up_proj
 *                            before down_proj); s has N entries (the scaled
 *                            linear's input channels). W fp16 [N][K]; b and
 *                            b_out fp16 [N], both NULL when there is no bias.
 *                            Fold before that linear is itself quantized.
 * Each result is fp16_rn(the fp32 quotient of IEEE division). Outputs may be
 * the inputs (in place). Pointers: device, 2-byte aligned (16-byte alignment
 * and K % 8 == 0 take the vectorized path). A result that is not finite in
 * fp16 latches WQ_ERR_RANGE in the device flag. One launch each (two with a
 * bias), asynchronous on `stream`. */
int32_t wq_awq_fold_norm(const void* gamma_dev, const void* s_dev, int64_t K, void* gamma_out_dev, void* stream);
int32_t wq_awq_fold_linear_rows(const void* W_dev, const void* b_dev, const void* s_dev, int64_t N, int64_t K,
                                void* W_out_dev, void* b_out_dev, void* stream);

/* Process-wide tuning options. Each is an atomic value, so a thread may set
 * one while another calls the library; a call reads each option it uses
 * once, so it runs wholly under the old or wholly under the new value.
 *  WQ_OPT_GEMM_PATH     WQ_PATH_AUTO (default): GEMV kernel below the
 *                       crossover M, tensor-core kernel at or above it;
 *                       WQ_PATH_GEMV / WQ_PATH_TENSOR_CORE force one kernel.
 *  WQ_OPT_CROSSOVER_M   smallest M sent to the tensor-core kernel (default 3;
 *                       with WQ_PATH_AUTO, M = 3 and 4 at 4 bits with
 *                       K <= 8192 stay on the row GEMV when the weight has
 *                       fewer 128-row tiles than the device has SMs).
 *  WQ_OPT_GEMV_VARIANT  how the GEMV kernel forms sum_k x_k (q_k - zero):
 *                       WQ_GEMV_OFFSET_SUMS (default) multiplies x by the
 *                       unpacked (1024 + q) in fp32 (exact products) and
 *                       removes the offset with per-chunk activation sums;
 *                       WQ_GEMV_INT_DIGITS turns each lane's activations into
 *                       a 24-bit fixed-point image (exact for every value
 *                       within 2^-13 of the lane's largest) and accumulates q
 *                       times its base-256 digits in exact integers (dp4a),
 *                       removing the zero point in integers; row-streaming
 *                       kernel only (the tiled kernel treats it as offset
 *                       sums), and zero points must be integers, as
 *                       wq_quantize_pack writes them;
 *                       WQ_GEMV_EXACT subtracts the zero point in fp16 first,
 *                       so every product is exact (tiled kernel only).
 *  WQ_OPT_GEMV_KERNEL   WQ_GEMV_KERNEL_AUTO (default): for M <= 2, K <= 16384
 *                       and not WQ_GEMV_EXACT, the row-streaming kernel (3-bit
 *                       rows always with offset sums)
 *                       (activations held in registers, warps split K);
 *                       otherwise the tiled kernel (activations in shared
 *                       memory, warps split rows, cluster split-K).
 *                       WQ_GEMV_KERNEL_TILED forces the tiled kernel.
 *  WQ_OPT_PDL           1 (default): GEMV launches allow programmatic dependent
 *                       launch (the kernel fetches its first weights, steps
 *                       and zeros before waiting for the previous kernel in
 *                       the stream); 0: off. So with it on, the kernel just
 *                       before a GEMV in the stream must not write that
 *                       GEMV's packed weights, steps or zeros (this library's
 *                       own kernels never do: they release their dependents
 *                       only at their end or after their last such write);
 *                       set 0 when a caller's kernel does.
 *  WQ_OPT_GEMV_ROWS_SHAPE  rows per batch R, input channels per lane C and
 *                       register stages S of the row-streaming kernel:
 *                       0 default (M = 1: shape 1 for K <= 4096 and for
 *                       K <= 8192 with N*K <= 2^27, else 2; M = 2: shape 1
 *                       for K <= 8192, else 2; M = 3, 4: shape 1), 1 (4, 32, 2),
 *                       2 (4, 64, 2), 3 (2, 64, 2), 4 (4, 32, 3). Shapes with
 *                       C = 32 apply for K <= 8192; above it shape 2 runs.
 *  WQ_OPT_GEMV_GRID     grid of the row-streaming kernel (all CTAs resident, CTA c
 *                       takes row batches c, c + grid, ...): 1 default, a CTA
 *                       for every resident slot; 0 one CTA per batch for small
 *                       problems, else the same number of batches per CTA.
 *  WQ_OPT_TC_STAGES     shared-memory ring depth of the tensor-core kernel:
 *                       0 default (library choice), 2..16 that depth (two CTAs
 *                       per SM when it fits; the call fails with WQ_ERR_CUDA
 *                       when one CTA's shared memory cannot hold it).
 *  WQ_OPT_TC_BK         input channels per stage of the tensor-core kernel: 0
 *                       default (64 when M rounded up to 16 is at least 96,
 *                       else 128), 64 or 128.
 *  WQ_OPT_TC_DEQUANT_WARPS  warps that dequantize in the tensor-core kernel:
 *                       0 default (4), 4 or 8.
 *  WQ_OPT_TC_STREAMK    the tensor-core kernel's stream-K schedule (needs the
 *                       workspace): 0 default (for M <= 16 per launch), 1
 *                       off, 2 whenever the workspace is given. Off when 8
 *                       dequantizing warps or a cluster split are asked for,
 *                       or when two accumulators do not fit the tensor
 *                       memory beside the A buffers (M > 96).
 *  WQ_OPT_TC_KSPLIT     CTAs of a thread-block cluster that share one 128-row
 *                       tile of the tensor-core kernel along K (their fp32
 *                       partial tiles are added in rank order in the first
 *                       CTA's shared memory): 0 default (library choice: the
 *                       largest of 1, 2, 4, 8 with at most one CTA per SM
 *                       and at least 4 stages each), 1, 2, 4 or 8 (the call
 *                       fails with WQ_ERR_CUDA when the first CTA's ring
 *                       cannot hold the other partial tiles or K has fewer
 *                       stages than CTAs).
 *  WQ_OPT_WAIT_LIMIT_MS how long a bounded mbarrier wait in the tensor-core
 *                       kernel may last before it latches WQ_ERR_TIMEOUT
 *                       (1..60000, default 2000).
 *  WQ_OPT_TEST_STALL    test hook, 0 (default) or 1: the tensor-core kernel's
 *                       producer issues no loads, so its consumers' waits run
 *                       out; the kernel then frees its tensor memory, returns,
 *                       and wq_get_last_device_error reports WQ_ERR_TIMEOUT.
 *                       Y is not written. For failure-handling tests only.
 *  WQ_OPT_AWQ_LOSS     how wq_awq_scale_search forms the losses:
 *                       WQ_AWQ_LOSS_FUSED (default) builds each tile of the
 *                       error matrix E = W - Q(W diag s) diag(s)^-1 in shared
 *                       memory inside the tensor-core GEMM, from the weights
 *                       it came from (no E in global memory);
 *                       WQ_AWQ_LOSS_TWO_KERNELS writes E of a batch of alphas
 *                       to the workspace and reads it back in a second
 *                       kernel (twice the HBM traffic of W per alpha). Both
 *                       round E to fp16; the noalloc search follows the same
 *                       option (fused: no error-matrix chunks).
 * wq_set_option returns WQ_ERR_INVALID_ARG for an unknown option or value;
 * wq_get_option returns the current value, or -1 for an unknown option. */
#define WQ_OPT_GEMM_PATH 1
#define WQ_OPT_CROSSOVER_M 2
#define WQ_PATH_AUTO 0
#define WQ_PATH_GEMV 1
#define WQ_PATH_TENSOR_CORE 2
#define WQ_OPT_GEMV_VARIANT 4
#define WQ_GEMV_OFFSET_SUMS 0
#define WQ_GEMV_EXACT 1
#define WQ_GEMV_INT_DIGITS 2
#define WQ_OPT_GEMV_KERNEL 5
#define WQ_GEMV_KERNEL_AUTO 0
#define WQ_GEMV_KERNEL_TILED 2
#define WQ_OPT_GEMV_ROWS_SHAPE 6
#define WQ_OPT_PDL 7
#define WQ_OPT_TC_STAGES 9
#define WQ_OPT_GEMV_GRID 10
#define WQ_OPT_TC_BK 11
#define WQ_OPT_TC_DEQUANT_WARPS 12
#define WQ_OPT_WAIT_LIMIT_MS 13
#define WQ_OPT_TEST_STALL 14
#define WQ_OPT_AWQ_LOSS 15
#define WQ_OPT_TC_KSPLIT 16
#define WQ_OPT_TC_STREAMK 17

#define WQ_AWQ_LOSS_TWO_KERNELS 0
#define WQ_AWQ_LOSS_FUSED 1

int32_t wq_set_option(int32_t option, int64_t value);
int64_t wq_get_option(int32_t option);

/* Synchronizes `stream`, then returns and clears the device flag of the
 * current device (WQ_OK if nothing was latched). Returns WQ_ERR_CUDA if the
 * synchronization itself fails. */
int32_t wq_get_last_device_error(void* stream);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* WQ_H_ */
