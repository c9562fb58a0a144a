// Host-side launchers of the kernels, shared by the C ABI (wq_abi.cu) and the
// files that define them, so every declaration is checked against its
// definition. Internal to the library: the public interface is include/wq.h.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace wq {
cudaError_t launch_quantize_pack(const void* W, const void* s, int64_t N, int64_t K, int bits, int group, bool sym,
                                 uint32_t* packed, void* steps, void* zeros, int* err, cudaStream_t st);
cudaError_t launch_unpack_dequant(const uint32_t* packed, const void* steps, const void* zeros, int64_t N,
                                  int64_t K, int bits, int group, void* out, cudaStream_t st);
cudaError_t launch_gemv(const void* X, const uint32_t* packed, const void* steps, const void* zeros, int64_t M,
                        int64_t N, int64_t K, int bits, void* Y, cudaStream_t st, int variant, bool pdl);
size_t gemv_smem_bytes(int bits, int variant, int M, int N, int K);
bool gemv_rows_supported(int bits, int group, int64_t M, int64_t K);
cudaError_t launch_gemv_rows(const void* X, const uint32_t* packed, const void* steps, const void* zeros, int64_t M,
                             int64_t N, int64_t K, int bits, int group, void* Y, cudaStream_t st, int shape,
                             bool act_int, int grid_mode, bool pdl);
cudaError_t launch_gemm_tc(const void* X, const uint32_t* packed, const void* steps, const void* zeros, int64_t M,
                           int64_t N, int64_t K, int bits, int group, void* Y, int* err, cudaStream_t st,
                           int stages_opt, int bk_opt, int dw_opt, int ksplit_opt, int streamk_opt, void* workspace,
                           size_t workspace_bytes, int wait_ms, bool stall);
// Workspace for the tensor-core kernel's stream-K schedule (M rows of X).
size_t gemm_tc_workspace_bytes(int64_t M, int64_t N, int64_t K, int bits);
// Workspace layout of the AWQ search (wq_awq.cu): mu, the candidate scales,
// the per-tile partial losses, and (two-kernel loss path only) the error
// matrices of one batch of alphas.
struct AwqPlan {
  int64_t N_total;
  int t_tiles, n_tiles, tiles;
  int fused_tiles, t_chunks;  // the fused loss kernel's row tiles and 512-token chunks
  int batch;  // alphas per E batch
  size_t off_mu, off_S, off_partial, off_E, total;
};
AwqPlan plan_awq(int64_t T, int64_t K, const int64_t* N_i, int n_lin, int n_alpha, bool fused);
cudaError_t launch_awq_search(const void* X, int64_t T, int64_t K, const void* const* W, const int64_t* N_i,
                              int n_lin, int bits, bool sym, const double* alpha, int n_alpha, void* s_out,
                              double* mu_out, double* loss_out, int32_t* best_out, void* workspace, int* err,
                              bool fused, cudaStream_t st);
bool awq_noalloc_fits(int64_t T, int64_t K, const int64_t* N_i, int n_lin, int n_alpha, bool fused);
cudaError_t launch_awq_search_noalloc(const void* X, int64_t T, int64_t K, const void* const* W,
                                      const int64_t* N_i, int n_lin, int bits, bool sym, const double* alpha,
                                      int n_alpha, void* s_out, double* mu_out, double* loss_out, int32_t* best_out,
                                      int* err, bool fused, cudaStream_t st);
// AWQ scale folding (wq_fold.cu): out = in / s along rows (s[R]) or columns (s[C]).
cudaError_t launch_fold(const void* in, const void* s, void* out, int64_t R, int64_t C, bool row_axis, int* err,
                        cudaStream_t st);
// W4A8 (wq_w4a8.cu): int8 activations per group, and the dp4a GEMV.
cudaError_t launch_act_int8(const void* X, int64_t M, int64_t K, int group, int8_t* q, float* mult,
                            cudaStream_t st);
size_t w4a8_smem_bytes(int M, int64_t K);
cudaError_t launch_w4a8_gemv(const int8_t* qx, const float* mult, const uint32_t* packed, const void* steps,
                             const void* zeros, int64_t M, int64_t N, int64_t K, int group, void* Y, cudaStream_t st);
// W4A8 on the row-streaming GEMV (wq_gemv_rows.cu), K <= 8192.
cudaError_t launch_w4a8_rows(const int8_t* qx, const float* mult, const uint32_t* packed, const void* steps,
                             const void* zeros, int64_t M, int64_t N, int64_t K, int group, void* Y, cudaStream_t st,
                             bool pdl);
// GPTQ (wq_gptq.cu): workspace layout and the launch sequence.
struct GptqPlan {
  size_t off_H, off_G, off_W, off_Err, off_dead, total;
};
GptqPlan plan_gptq(int64_t N, int64_t K);
cudaError_t launch_gptq(const void* X, int64_t T, const void* W, int64_t N, int64_t K, int bits, int group, bool sym,
                        double damp, uint32_t* packed, void* steps, void* zeros, void* workspace, int* err,
                        cudaStream_t st);
}  // namespace wq
