// C ABI of libwq.so: argument validation, dispatch, and the device error flag.
// Every entry point validates on the host, enqueues on the caller's stream and
// returns; none allocates device memory.
#include <atomic>
#include <mutex>
#include <nvtx3/nvToolsExt.h>

#include "wq_common.cuh"
#include "wq_launch.h"

// One flag per device (each device holds its own copy of a __device__ variable).
__device__ int g_wq_device_error;

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_flag_mu;
int* g_flag_addr[kMaxDevices] = {};

// Address of this device's error flag; looked up once per device with the
// device current. Returns nullptr on failure.
int* device_flag() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_flag_mu);
  if (g_flag_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_wq_device_error) != cudaSuccess) return nullptr;
    g_flag_addr[dev] = static_cast<int*>(p);
  }
  return g_flag_addr[dev];
}

// NVTX range around each entry point (a no-op unless a profiler is attached).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int32_t check_cfg(const wq_quant_cfg* cfg) {
  if (cfg == nullptr) return WQ_ERR_INVALID_ARG;
  if (cfg->bits != 3 && cfg->bits != 4) return cfg->bits >= 2 && cfg->bits <= 8 ? WQ_ERR_UNSUPPORTED : WQ_ERR_INVALID_ARG;
  if (cfg->group_size != 32 && cfg->group_size != 64 && cfg->group_size != wq::kGroup) return WQ_ERR_INVALID_ARG;
  if (cfg->symmetric != 0 && cfg->symmetric != 1) return WQ_ERR_INVALID_ARG;
  return WQ_OK;
}

int32_t check_shape(int64_t N, int64_t K) {
  if (N < 1 || K < wq::kGroup || K % wq::kGroup != 0) return WQ_ERR_INVALID_ARG;
  if (N > (int64_t)INT32_MAX / 2 || K > (int64_t)INT32_MAX / 2) return WQ_ERR_INVALID_ARG;
  return WQ_OK;
}

int32_t cuda_status(cudaError_t e) { return e == cudaSuccess ? WQ_OK : WQ_ERR_CUDA; }

// Process-wide tuning options (wq_set_option). Atomic, so setting one from
// another thread is not a data race; a call reads each option once.
std::atomic<int64_t> g_opt_gemm_path{WQ_PATH_AUTO};
std::atomic<int64_t> g_opt_crossover_m{3};
std::atomic<int64_t> g_opt_pdl{1};
std::atomic<int64_t> g_opt_gemv_variant{WQ_GEMV_OFFSET_SUMS};
std::atomic<int64_t> g_opt_gemv_kernel{WQ_GEMV_KERNEL_AUTO};
std::atomic<int64_t> g_opt_gemv_rows_shape{0};
std::atomic<int64_t> g_opt_tc_stages{0};
std::atomic<int64_t> g_opt_gemv_grid{1};
std::atomic<int64_t> g_opt_tc_bk{0};
std::atomic<int64_t> g_opt_tc_dequant_warps{0};
std::atomic<int64_t> g_opt_tc_streamk{0};
std::atomic<int64_t> g_opt_wait_limit_ms{2000};
std::atomic<int64_t> g_opt_test_stall{0};
std::atomic<int64_t> g_opt_awq_loss{WQ_AWQ_LOSS_FUSED};
std::atomic<int64_t> g_opt_tc_ksplit{0};

}  // namespace

extern "C" {

int32_t wq_abi_version(void) { return WQ_ABI_VERSION; }
int32_t wq_layout_version(void) { return WQ_LAYOUT_VERSION; }

const char* wq_status_string(int32_t s) {
  switch (s) {
    case WQ_OK: return "WQ_OK";
    case WQ_ERR_INVALID_ARG: return "WQ_ERR_INVALID_ARG: invalid argument";
    case WQ_ERR_UNSUPPORTED: return "WQ_ERR_UNSUPPORTED: configuration not supported";
    case WQ_ERR_ALIGNMENT: return "WQ_ERR_ALIGNMENT: pointer alignment";
    case WQ_ERR_CUDA: return "WQ_ERR_CUDA: CUDA runtime error";
    case WQ_ERR_TIMEOUT: return "WQ_ERR_TIMEOUT: bounded device wait gave up";
    case WQ_ERR_WORKSPACE: return "WQ_ERR_WORKSPACE: workspace missing or too small";
    case WQ_ERR_RANGE: return "WQ_ERR_RANGE: value not finite in fp16";
  }
  return "unknown wq status";
}

size_t wq_packed_words(int64_t N, int64_t K, const wq_quant_cfg* cfg) {
  if (check_cfg(cfg) != WQ_OK || check_shape(N, K) != WQ_OK) return 0;
  return cfg->bits == 4 ? (size_t)N * (size_t)K / 8 : (size_t)N * (size_t)K * 3 / 32;
}

int32_t wq_quantize_pack(const void* W, const void* s, int64_t N, int64_t K, const wq_quant_cfg* cfg,
                         uint32_t* packed, void* steps, void* zeros, void* stream) {
  NvtxRange nvtx_range("wq_quantize_pack");
  int32_t st = check_cfg(cfg);
  if (st != WQ_OK) return st;
  if ((st = check_shape(N, K)) != WQ_OK) return st;
  if (!W || !packed || !steps || !zeros) return WQ_ERR_INVALID_ARG;
  if (!aligned(W, 16) || !aligned(packed, 16) || (s && !aligned(s, 16)) || !aligned(steps, 4) ||
      !aligned(zeros, 4))
    return WQ_ERR_ALIGNMENT;
  int* flag = device_flag();
  if (!flag) return WQ_ERR_CUDA;
  return cuda_status(wq::launch_quantize_pack(W, s, N, K, cfg->bits, cfg->group_size, cfg->symmetric != 0, packed,
                                              steps, zeros, flag, static_cast<cudaStream_t>(stream)));
}

int32_t wq_unpack_dequant(const uint32_t* packed, const void* steps, const void* zeros, int64_t N, int64_t K,
                          const wq_quant_cfg* cfg, void* W_out, void* stream) {
  NvtxRange nvtx_range("wq_unpack_dequant");
  int32_t st = check_cfg(cfg);
  if (st != WQ_OK) return st;
  if ((st = check_shape(N, K)) != WQ_OK) return st;
  if (!packed || !steps || !zeros || !W_out) return WQ_ERR_INVALID_ARG;
  if (!aligned(packed, 16) || !aligned(W_out, 16) || !aligned(steps, 4) || !aligned(zeros, 4))
    return WQ_ERR_ALIGNMENT;
  return cuda_status(wq::launch_unpack_dequant(packed, steps, zeros, N, K, cfg->bits, cfg->group_size, W_out,
                                               static_cast<cudaStream_t>(stream)));
}

size_t wq_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K, const wq_quant_cfg* cfg) {
  if (check_cfg(cfg) != WQ_OK || check_shape(N, K) != WQ_OK || M < 3) return 0;
  return wq::gemm_tc_workspace_bytes(M, N, K, cfg->bits);
}

// SMs of the current device (cached per process; one device type per process).
static int num_sms() {
  static std::atomic<int> sms{0};
  int v = sms.load();
  if (v == 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
      v = 148;
    sms.store(v);
  }
  return v;
}

int32_t wq_w4a16_gemm(const void* X, const uint32_t* packed, const void* steps, const void* zeros, int64_t M,
                      int64_t N, int64_t K, const wq_quant_cfg* cfg, void* Y, void* workspace,
                      size_t workspace_bytes, void* stream) {
  NvtxRange nvtx_range("wq_w4a16_gemm");
  int32_t st = check_cfg(cfg);
  if (st != WQ_OK) return st;
  if ((st = check_shape(N, K)) != WQ_OK) return st;
  if (M < 1 || M > (int64_t)INT32_MAX / 2) return WQ_ERR_INVALID_ARG;
  if (!X || !packed || !steps || !zeros || !Y) return WQ_ERR_INVALID_ARG;
  if (!aligned(X, 16) || !aligned(packed, 16) || !aligned(steps, 2) || !aligned(zeros, 2) || !aligned(Y, 2) ||
      (workspace && !aligned(workspace, 256)))
    return WQ_ERR_ALIGNMENT;
  // one reading of every option this call uses
  const int64_t path = g_opt_gemm_path, variant = g_opt_gemv_variant, pdl = g_opt_pdl;
  const int group = cfg->group_size;
  const bool rows_ok = g_opt_gemv_kernel != WQ_GEMV_KERNEL_TILED && variant != WQ_GEMV_EXACT &&
                       wq::gemv_rows_supported(cfg->bits, group, M, K);
  bool tensor_core = M >= g_opt_crossover_m;
  // M = 3, 4 (4-bit, K <= 8192) stay on the row GEMV when the weight has
  // fewer 128-row tiles than the GPU has SMs: there the tensor-core kernel
  // leaves SMs idle or splits K over clusters (8192 x 8192, M = 4: 21 us on
  // the row kernel against 31 us), while wider weights keep every SM's
  // tensor pipe busy (8192 x 28672, M = 4: 56 us against 67 us).
  if (path == WQ_PATH_AUTO && tensor_core && M <= 4 && rows_ok && (N + 127) / 128 < num_sms()) tensor_core = false;
  if (path == WQ_PATH_GEMV) tensor_core = false;
  if (path == WQ_PATH_TENSOR_CORE) tensor_core = true;
  // groups of 32 or 64 channels that the row-streaming kernel does not take
  // (M > 2, 3-bit groups of 32, groups of 32 with K > 8192) run on the tensor
  // cores: the tiled GEMV handles groups of 128 only
  if (group != wq::kGroup && !rows_ok) tensor_core = true;
  if (tensor_core) {
    int* flag = device_flag();
    if (!flag) return WQ_ERR_CUDA;
    return cuda_status(wq::launch_gemm_tc(X, packed, steps, zeros, M, N, K, cfg->bits, group, Y, flag,
                                          static_cast<cudaStream_t>(stream), (int)g_opt_tc_stages,
                                          (int)g_opt_tc_bk, (int)g_opt_tc_dequant_warps, (int)g_opt_tc_ksplit,
                                          (int)g_opt_tc_streamk, workspace, workspace ? workspace_bytes : 0,
                                          (int)g_opt_wait_limit_ms, g_opt_test_stall != 0));
  }
  if (rows_ok)
    return cuda_status(wq::launch_gemv_rows(X, packed, steps, zeros, M, N, K, cfg->bits, group, Y,
                                            static_cast<cudaStream_t>(stream),
                                            (int)g_opt_gemv_rows_shape, variant == WQ_GEMV_INT_DIGITS,
                                            (int)g_opt_gemv_grid, pdl != 0));
  // the tiled kernel forms the integer-digit variant's sums as offset sums
  const int tiled_variant = variant == WQ_GEMV_EXACT ? WQ_GEMV_EXACT : WQ_GEMV_OFFSET_SUMS;
  // The shared copy of an X slice must fit one CTA.
  if (wq::gemv_smem_bytes(cfg->bits, tiled_variant, (int)(M < 8 ? M : 8), (int)N, (int)K) > 200 * 1024)
    return WQ_ERR_UNSUPPORTED;
  return cuda_status(wq::launch_gemv(X, packed, steps, zeros, M, N, K, cfg->bits, Y,
                                     static_cast<cudaStream_t>(stream), tiled_variant, pdl != 0));
}

static int32_t check_awq(int64_t T, int64_t K, const int64_t* N_i, int32_t n_lin, int32_t n_alpha,
                         const wq_quant_cfg* cfg) {
  int32_t st = check_cfg(cfg);
  if (st != WQ_OK) return st;
  if (cfg->group_size != wq::kGroup) return WQ_ERR_UNSUPPORTED;
  if (T < 1 || T > (int64_t)INT32_MAX / 2 || !N_i || n_lin < 1 || n_lin > 8 || n_alpha < 1 || n_alpha > 64)
    return WQ_ERR_INVALID_ARG;
  int64_t tot = 0;
  for (int i = 0; i < n_lin; ++i) {
    if ((st = check_shape(N_i[i], K)) != WQ_OK) return st;
    tot += N_i[i];
  }
  if (tot > (int64_t)INT32_MAX / 2) return WQ_ERR_INVALID_ARG;
  return WQ_OK;
}

size_t wq_awq_workspace_bytes(int64_t T, int64_t K, const int64_t* N_i, int32_t n_lin, int32_t n_alpha,
                              const wq_quant_cfg* cfg) {
  if (check_awq(T, K, N_i, n_lin, n_alpha, cfg) != WQ_OK) return 0;
  return wq::plan_awq(T, K, N_i, n_lin, n_alpha, g_opt_awq_loss == WQ_AWQ_LOSS_FUSED).total;
}

int32_t wq_awq_scale_search(const void* X, int64_t T, int64_t K, const void* const* W, const int64_t* N_i,
                            int32_t n_lin, const wq_quant_cfg* cfg, const double* alpha, int32_t n_alpha,
                            void* s_out, double* mu_out, double* loss_out, int32_t* best_out, void* workspace,
                            size_t workspace_bytes, void* stream) {
  NvtxRange nvtx_range("wq_awq_scale_search");
  int32_t st = check_awq(T, K, N_i, n_lin, n_alpha, cfg);
  if (st != WQ_OK) return st;
  if (!X || !W || !alpha || !s_out) return WQ_ERR_INVALID_ARG;
  for (int i = 0; i < n_lin; ++i) {
    if (!W[i]) return WQ_ERR_INVALID_ARG;
    if (!aligned(W[i], 16)) return WQ_ERR_ALIGNMENT;
  }
  for (int j = 0; j < n_alpha; ++j)
    if (!(alpha[j] == alpha[j])) return WQ_ERR_INVALID_ARG;  // NaN
  if (!aligned(X, 16) || !aligned(s_out, 2) || (mu_out && !aligned(mu_out, 8)) || (loss_out && !aligned(loss_out, 8)) ||
      (best_out && !aligned(best_out, 4)))
    return WQ_ERR_ALIGNMENT;
  const bool fused = g_opt_awq_loss == WQ_AWQ_LOSS_FUSED;  // one reading: the size check and the launch agree
  const size_t need = wq::plan_awq(T, K, N_i, n_lin, n_alpha, fused).total;
  if (!workspace || workspace_bytes < need) return WQ_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return WQ_ERR_ALIGNMENT;
  int* flag = device_flag();
  if (!flag) return WQ_ERR_CUDA;
  return cuda_status(wq::launch_awq_search(X, T, K, W, N_i, n_lin, cfg->bits, cfg->symmetric != 0, alpha, n_alpha,
                                           s_out, mu_out, loss_out, best_out, workspace, flag,
                                           fused, static_cast<cudaStream_t>(stream)));
}

int32_t wq_awq_scale_search_noalloc(const void* X, int64_t T, int64_t K, const void* const* W, const int64_t* N_i,
                                    int32_t n_lin, const wq_quant_cfg* cfg, const double* alpha, int32_t n_alpha,
                                    void* s_out, double* mu_out, double* loss_out, int32_t* best_out, void* stream) {
  NvtxRange nvtx_range("wq_awq_scale_search_noalloc");
  int32_t st = check_awq(T, K, N_i, n_lin, n_alpha, cfg);
  if (st != WQ_OK) return st;
  if (!X || !W || !alpha || !s_out) return WQ_ERR_INVALID_ARG;
  for (int i = 0; i < n_lin; ++i) {
    if (!W[i]) return WQ_ERR_INVALID_ARG;
    if (!aligned(W[i], 16)) return WQ_ERR_ALIGNMENT;
  }
  for (int j = 0; j < n_alpha; ++j)
    if (!(alpha[j] == alpha[j])) return WQ_ERR_INVALID_ARG;  // NaN
  if (!aligned(X, 16) || !aligned(s_out, 2) || (mu_out && !aligned(mu_out, 8)) || (loss_out && !aligned(loss_out, 8)) ||
      (best_out && !aligned(best_out, 4)))
    return WQ_ERR_ALIGNMENT;
  const bool fused = g_opt_awq_loss == WQ_AWQ_LOSS_FUSED;  // one reading: the fit check and the launch agree
  if (!wq::awq_noalloc_fits(T, K, N_i, n_lin, n_alpha, fused)) return WQ_ERR_WORKSPACE;
  int* flag = device_flag();
  if (!flag) return WQ_ERR_CUDA;
  return cuda_status(wq::launch_awq_search_noalloc(X, T, K, W, N_i, n_lin, cfg->bits, cfg->symmetric != 0, alpha,
                                                   n_alpha, s_out, mu_out, loss_out, best_out, flag, fused,
                                                   static_cast<cudaStream_t>(stream)));
}

int32_t wq_quantize_act_int8(const void* X, int64_t M, int64_t K, int32_t group, int8_t* q, float* mult,
                             void* stream) {
  NvtxRange nvtx_range("wq_quantize_act_int8");
  if (group != 32 && group != 64 && group != wq::kGroup) return WQ_ERR_INVALID_ARG;
  if (M < 1 || K < group || K % group != 0 || M > (int64_t)INT32_MAX / 2 || K > (int64_t)INT32_MAX / 2)
    return WQ_ERR_INVALID_ARG;
  if (!X || !q || !mult) return WQ_ERR_INVALID_ARG;
  if (!aligned(X, 2) || !aligned(q, 4) || !aligned(mult, 4)) return WQ_ERR_ALIGNMENT;
  return cuda_status(wq::launch_act_int8(X, M, K, group, q, mult, static_cast<cudaStream_t>(stream)));
}

int32_t wq_w4a8_gemm(const int8_t* q, const float* mult, const uint32_t* packed, const void* steps, const void* zeros,
                     int64_t M, int64_t N, int64_t K, const wq_quant_cfg* cfg, void* Y, void* stream) {
  NvtxRange nvtx_range("wq_w4a8_gemm");
  int32_t st = check_cfg(cfg);
  if (st != WQ_OK) return st;
  if (cfg->bits != 4) return WQ_ERR_UNSUPPORTED;
  if ((st = check_shape(N, K)) != WQ_OK) return st;
  if (M < 1 || M > (int64_t)INT32_MAX / 2) return WQ_ERR_INVALID_ARG;
  if (K > 16384) return WQ_ERR_UNSUPPORTED;  // the activation codes of 4 rows in one CTA's shared memory
  if (!q || !mult || !packed || !steps || !zeros || !Y) return WQ_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(mult, 4) || !aligned(packed, 16) || !aligned(steps, 2) || !aligned(zeros, 2) ||
      !aligned(Y, 2))
    return WQ_ERR_ALIGNMENT;
  // K <= 8192: the row-streaming GEMV (32 channels per lane); above, the
  // slice kernel with the codes in shared memory
  if (K <= 8192)
    return cuda_status(wq::launch_w4a8_rows(q, mult, packed, steps, zeros, M, N, K, cfg->group_size, Y,
                                            static_cast<cudaStream_t>(stream), g_opt_pdl != 0));
  return cuda_status(wq::launch_w4a8_gemv(q, mult, packed, steps, zeros, M, N, K, cfg->group_size, Y,
                                          static_cast<cudaStream_t>(stream)));
}

size_t wq_gptq_workspace_bytes(int64_t N, int64_t K, const wq_quant_cfg* cfg) {
  if (check_cfg(cfg) != WQ_OK || check_shape(N, K) != WQ_OK) return 0;
  return wq::plan_gptq(N, K).total;
}

int32_t wq_gptq_quantize_pack(const void* X, int64_t T, const void* W, int64_t N, int64_t K, const wq_quant_cfg* cfg,
                              double damp, uint32_t* packed, void* steps, void* zeros, void* workspace,
                              size_t workspace_bytes, void* stream) {
  NvtxRange nvtx_range("wq_gptq_quantize_pack");
  int32_t st = check_cfg(cfg);
  if (st != WQ_OK) return st;
  if ((st = check_shape(N, K)) != WQ_OK) return st;
  if (T < 1 || T > (int64_t)INT32_MAX / 2 || !(damp >= 0.0 && damp < 1e6)) return WQ_ERR_INVALID_ARG;
  if (!X || !W || !packed || !steps || !zeros) return WQ_ERR_INVALID_ARG;
  if (!aligned(X, 2) || !aligned(W, 2) || !aligned(packed, 16) || !aligned(steps, 2) || !aligned(zeros, 2))
    return WQ_ERR_ALIGNMENT;
  if (!workspace || workspace_bytes < wq::plan_gptq(N, K).total) return WQ_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return WQ_ERR_ALIGNMENT;
  int* flag = device_flag();
  if (!flag) return WQ_ERR_CUDA;
  return cuda_status(wq::launch_gptq(X, T, W, N, K, cfg->bits, cfg->group_size, cfg->symmetric != 0, damp, packed,
                                     steps, zeros, workspace, flag, static_cast<cudaStream_t>(stream)));
}

int32_t wq_awq_fold_norm(const void* gamma, const void* s, int64_t K, void* gamma_out, void* stream) {
  NvtxRange nvtx_range("wq_awq_fold_norm");
  if (!gamma || !s || !gamma_out) return WQ_ERR_INVALID_ARG;
  if (K < 1 || K > (int64_t)INT32_MAX) return WQ_ERR_INVALID_ARG;
  if (!aligned(gamma, 2) || !aligned(s, 2) || !aligned(gamma_out, 2)) return WQ_ERR_ALIGNMENT;
  int* flag = device_flag();
  if (!flag) return WQ_ERR_CUDA;
  return cuda_status(wq::launch_fold(gamma, s, gamma_out, 1, K, false, flag, static_cast<cudaStream_t>(stream)));
}

int32_t wq_awq_fold_linear_rows(const void* W, const void* b, const void* s, int64_t N, int64_t K, void* W_out,
                                void* b_out, void* stream) {
  NvtxRange nvtx_range("wq_awq_fold_linear_rows");
  if (!W || !s || !W_out || (b == nullptr) != (b_out == nullptr)) return WQ_ERR_INVALID_ARG;
  if (N < 1 || K < 1 || N > (int64_t)INT32_MAX || K > (int64_t)INT32_MAX) return WQ_ERR_INVALID_ARG;
  if (!aligned(W, 2) || !aligned(s, 2) || !aligned(W_out, 2) || (b && (!aligned(b, 2) || !aligned(b_out, 2))))
    return WQ_ERR_ALIGNMENT;
  int* flag = device_flag();
  if (!flag) return WQ_ERR_CUDA;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = wq::launch_fold(W, s, W_out, N, K, true, flag, st);
  if (e == cudaSuccess && b) e = wq::launch_fold(b, s, b_out, 1, N, false, flag, st);
  return cuda_status(e);
}

int32_t wq_set_option(int32_t option, int64_t value) {
  switch (option) {
    case WQ_OPT_GEMM_PATH:
      if (value < WQ_PATH_AUTO || value > WQ_PATH_TENSOR_CORE) return WQ_ERR_INVALID_ARG;
      g_opt_gemm_path = value;
      return WQ_OK;
    case WQ_OPT_CROSSOVER_M:
      if (value < 1) return WQ_ERR_INVALID_ARG;
      g_opt_crossover_m = value;
      return WQ_OK;
    case WQ_OPT_GEMV_KERNEL:
      if (value != WQ_GEMV_KERNEL_AUTO && value != WQ_GEMV_KERNEL_TILED) return WQ_ERR_INVALID_ARG;
      g_opt_gemv_kernel = value;
      return WQ_OK;
    case WQ_OPT_PDL:
      if (value != 0 && value != 1) return WQ_ERR_INVALID_ARG;
      g_opt_pdl = value;
      return WQ_OK;
    case WQ_OPT_GEMV_ROWS_SHAPE:
      if (value < 0 || value > 4) return WQ_ERR_INVALID_ARG;
      g_opt_gemv_rows_shape = value;
      return WQ_OK;
    case WQ_OPT_WAIT_LIMIT_MS:
      if (value < 1 || value > 60000) return WQ_ERR_INVALID_ARG;
      g_opt_wait_limit_ms = value;
      return WQ_OK;
    case WQ_OPT_TEST_STALL:
      if (value != 0 && value != 1) return WQ_ERR_INVALID_ARG;
      g_opt_test_stall = value;
      return WQ_OK;
    case WQ_OPT_AWQ_LOSS:
      if (value != WQ_AWQ_LOSS_TWO_KERNELS && value != WQ_AWQ_LOSS_FUSED) return WQ_ERR_INVALID_ARG;
      g_opt_awq_loss = value;
      return WQ_OK;
    case WQ_OPT_TC_KSPLIT:
      if (value != 0 && value != 1 && value != 2 && value != 4 && value != 8) return WQ_ERR_INVALID_ARG;
      g_opt_tc_ksplit = value;
      return WQ_OK;
    case WQ_OPT_TC_STREAMK:
      if (value != 0 && value != 1 && value != 2) return WQ_ERR_INVALID_ARG;
      g_opt_tc_streamk = value;
      return WQ_OK;
    case WQ_OPT_TC_DEQUANT_WARPS:
      if (value != 0 && value != 4 && value != 8) return WQ_ERR_INVALID_ARG;
      g_opt_tc_dequant_warps = value;
      return WQ_OK;
    case WQ_OPT_TC_BK:
      if (value != 0 && value != 64 && value != 128) return WQ_ERR_INVALID_ARG;
      g_opt_tc_bk = value;
      return WQ_OK;
    case WQ_OPT_GEMV_GRID:
      if (value != 0 && value != 1) return WQ_ERR_INVALID_ARG;
      g_opt_gemv_grid = value;
      return WQ_OK;
    case WQ_OPT_TC_STAGES:
      if (value != 0 && (value < 2 || value > 16)) return WQ_ERR_INVALID_ARG;
      g_opt_tc_stages = value;
      return WQ_OK;
    case WQ_OPT_GEMV_VARIANT:
      if (value != WQ_GEMV_OFFSET_SUMS && value != WQ_GEMV_EXACT && value != WQ_GEMV_INT_DIGITS)
        return WQ_ERR_INVALID_ARG;
      g_opt_gemv_variant = value;
      return WQ_OK;
  }
  return WQ_ERR_INVALID_ARG;
}

int64_t wq_get_option(int32_t option) {
  switch (option) {
    case WQ_OPT_GEMM_PATH: return g_opt_gemm_path;
    case WQ_OPT_CROSSOVER_M: return g_opt_crossover_m;
    case WQ_OPT_GEMV_VARIANT: return g_opt_gemv_variant;
    case WQ_OPT_GEMV_KERNEL: return g_opt_gemv_kernel;
    case WQ_OPT_GEMV_ROWS_SHAPE: return g_opt_gemv_rows_shape;
    case WQ_OPT_TC_STAGES: return g_opt_tc_stages;
    case WQ_OPT_GEMV_GRID: return g_opt_gemv_grid;
    case WQ_OPT_TC_BK: return g_opt_tc_bk;
    case WQ_OPT_TC_DEQUANT_WARPS: return g_opt_tc_dequant_warps;
    case WQ_OPT_WAIT_LIMIT_MS: return g_opt_wait_limit_ms;
    case WQ_OPT_TEST_STALL: return g_opt_test_stall;
    case WQ_OPT_PDL: return g_opt_pdl;
    case WQ_OPT_AWQ_LOSS: return g_opt_awq_loss;
    case WQ_OPT_TC_KSPLIT: return g_opt_tc_ksplit;
    case WQ_OPT_TC_STREAMK: return g_opt_tc_streamk;
  }
  return -1;
}

int32_t wq_get_last_device_error(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return WQ_ERR_CUDA;
  int* flag = device_flag();
  if (!flag) return WQ_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, flag, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return WQ_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpy(flag, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return WQ_ERR_CUDA;
  }
  return v;
}

}  // extern "C"
