// AWQ scale folding: the op that produces the scaled linears' input absorbs
// diag(s)^-1 ("MIT 6.5940 Lab 4 + Lab 5", section "Question 2": the searched
// scales are folded into the previous LayerNorm or linear layer).
//
//   fold into a norm weight        gamma'_k = gamma_k / s_k        (s along columns)
//   fold into a linear's rows      W'[n][k] = W[n][k] / s_n,       (s along rows)
//                                  b'_n = b_n / s_n
//
// Stored form: fp16_rn(fp32 quotient) -- the correctly rounded fp32 quotient
// and one rounding to fp16, the contract the oracle restates. The quotient is
// formed without a division instruction: q0 = fl(w y) with y = rcp_refined(s),
// r = w - s q0 (exact), q = fl(q0 + r y), Markstein's correction, exact for an
// fp16 divisor (11 significant bits) and any fp32 dividend in this range (the
// argument at group_quotient; checked in exact rational arithmetic for fp16
// weights and scales of both signs, subnormals included). r = 0 keeps q0
// itself, so a zero quotient keeps the sign of w / s; infinite or NaN operands
// and a zero divisor take the IEEE division. A result that is not finite in
// fp16 latches WQ_ERR_RANGE. HBM-bound: 2 B read + 2 B written per element
// (+ the scale, from L1/L2); one wave of resident CTAs walks 16-byte chunks
// grid-stride.
#include "wq_common.cuh"
#include "wq_launch.h"
#include "wq_quant_core.cuh"

namespace wq {

// y: rcp_refined(s)
__device__ __forceinline__ __half fold_one(__half wh, float s, float y, bool& bad) {
  const float w = __half2float(wh);
  const float q0 = __fmul_rn(w, y);
  const float r = __fmaf_rn(-q0, s, w);
  float q = r == 0.0f ? q0 : __fmaf_rn(r, y, q0);
  if (!isfinite(q)) q = __fdiv_rn(w, s);  // infinite or NaN operands, zero divisor
  const __half h = __float2half_rn(q);
  bad |= __hisinf(h) || __hisnan(h);
  return h;
}

// out[r][c] = in[r][c] / s[ROW_AXIS ? r : c] for an [R][C] fp16 matrix; C % 8
// == 0 and 16-byte aligned pointers (the host picks the scalar kernel
// otherwise). out may equal in: each element is read, then written, by the
// same thread.
template <bool ROW_AXIS>
__global__ void __launch_bounds__(256) fold_vec_kernel(const __half* in, const __half* __restrict__ s,
                                                       __half* out, int64_t R, int64_t C, int* err) {
  const int64_t chunks = R * (C / 8);
  const int64_t cpr = C / 8;
  bool bad = false;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < chunks; i += (int64_t)gridDim.x * blockDim.x) {
    const uint4 v = *reinterpret_cast<const uint4*>(in + 8 * i);
    const __half* h = reinterpret_cast<const __half*>(&v);
    uint4 o;
    __half* oh = reinterpret_cast<__half*>(&o);
    if constexpr (ROW_AXIS) {
      const float sv = __half2float(s[i / cpr]);
      const float y = rcp_refined(sv);
#pragma unroll
      for (int j = 0; j < 8; ++j) oh[j] = fold_one(h[j], sv, y, bad);
    } else {
      const uint4 sr = *reinterpret_cast<const uint4*>(s + 8 * (i % cpr));
      const __half* sh = reinterpret_cast<const __half*>(&sr);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float sv = __half2float(sh[j]);
        oh[j] = fold_one(h[j], sv, rcp_refined(sv), bad);
      }
    }
    *reinterpret_cast<uint4*>(out + 8 * i) = o;
  }
  if (bad) latch_error(err, WQ_ERR_RANGE);
}

// Any shape and alignment (norm weights of any length, biases).
template <bool ROW_AXIS>
__global__ void __launch_bounds__(256) fold_scalar_kernel(const __half* in, const __half* __restrict__ s,
                                                          __half* out, int64_t R, int64_t C, int* err) {
  bool bad = false;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < R * C; i += (int64_t)gridDim.x * blockDim.x)
  {
    const float sv = __half2float(s[ROW_AXIS ? i / C : i % C]);
    out[i] = fold_one(in[i], sv, rcp_refined(sv), bad);
  }
  if (bad) latch_error(err, WQ_ERR_RANGE);
}

static int fold_grid(int64_t work) {
  static int sms = 0;
  if (sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms <= 0) sms = 148;
  }
  const int64_t want = (work + 255) / 256;
  const int64_t wave = (int64_t)sms * 8;  // 8 CTAs of 256 threads per SM
  return (int)(want < wave ? (want > 0 ? want : 1) : wave);
}

cudaError_t launch_fold(const void* in, const void* s, void* out, int64_t R, int64_t C, bool row_axis, int* err,
                        cudaStream_t st) {
  const __half* ih = static_cast<const __half*>(in);
  const __half* sh = static_cast<const __half*>(s);
  __half* oh = static_cast<__half*>(out);
  const bool vec = C % 8 == 0 && (reinterpret_cast<uintptr_t>(in) % 16) == 0 &&
                   (reinterpret_cast<uintptr_t>(out) % 16) == 0 && (row_axis || (reinterpret_cast<uintptr_t>(s) % 16) == 0);
  if (vec) {
    const int g = fold_grid(R * (C / 8));
    if (row_axis) fold_vec_kernel<true><<<g, 256, 0, st>>>(ih, sh, oh, R, C, err);
    else fold_vec_kernel<false><<<g, 256, 0, st>>>(ih, sh, oh, R, C, err);
  } else {
    const int g = fold_grid(R * C);
    if (row_axis) fold_scalar_kernel<true><<<g, 256, 0, st>>>(ih, sh, oh, R, C, err);
    else fold_scalar_kernel<false><<<g, 256, 0, st>>>(ih, sh, oh, R, C, err);
  }
  return cudaGetLastError();
}

}  // namespace wq
