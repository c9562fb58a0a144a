// S3: group-wise quantize + pack, and the inverse (unpack + dequantize).
//
// Quantizer: "LLM Quantization: 160GB Model on a Laptop", sections "Symmetric
// Quantization" and "Asymmetric Quantization"; integer zero point as in "CMU
// 11-868 L19-L20 Model Quantization", section "absmax and zero-point"; one
// step and zero per 128 input channels of a row ("Quantising Large Language
// Models for Efficient Inference", "Post-training methods for 4-bit weights").
// Optional AWQ input-channel scaling W * diag(s) first ("MIT 6.5940 Lab 4 +
// Lab 5", "Question 2").
//
// Mapping: 4 lanes per group, each lane owns 32 consecutive input channels
// (four 16-byte loads of W; one 16-byte store of 4-bit codes, or the three
// words of a 3-bit chunk); group_quant_decide() reduces the group's range
// with two xor-shuffles. 2 B/weight in, 0.5 (0.375) B/weight out.
#include "wq_quant_core.cuh"

namespace wq {

template <int BITS, bool SYM, bool HAS_S>
__global__ void __launch_bounds__(256)
quantize_pack_kernel(const __half* __restrict__ W, const __half* __restrict__ s, int64_t N, int64_t K,
                     uint32_t* __restrict__ packed, __half* __restrict__ steps,
                     __half* __restrict__ zeros, int* err) {
  const int lane = threadIdx.x & 31;
  const int sub = lane & 3;  // lane within the group
  const int64_t G = K / kGroup;
  const int64_t gidx = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 2;
  const bool valid = gidx < N * G;
  const int64_t n = valid ? gidx / G : 0;
  const int64_t gi = valid ? gidx % G : 0;
  const int64_t k0 = gi * kGroup + sub * 32;

  float w[32];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint4 raw = make_uint4(0, 0, 0, 0);
    if (valid) raw = *reinterpret_cast<const uint4*>(W + n * K + k0 + 8 * c);
    const __half2* h = reinterpret_cast<const __half2*>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __half22float2(h[i]);
      w[8 * c + 2 * i] = f.x;
      w[8 * c + 2 * i + 1] = f.y;
    }
    if (HAS_S) {
      uint4 sraw = make_uint4(0, 0, 0, 0);
      if (valid) sraw = *reinterpret_cast<const uint4*>(s + k0 + 8 * c);
      const __half2* sh = reinterpret_cast<const __half2*>(&sraw);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __half22float2(sh[i]);
        w[8 * c + 2 * i] = __fmul_rn(w[8 * c + 2 * i], f.x);  // exact: 11 x 11 significand bits
        w[8 * c + 2 * i + 1] = __fmul_rn(w[8 * c + 2 * i + 1], f.y);
      }
    }
  }

  const GroupQuant gq = group_quant_decide<BITS, SYM, 32, 4>(w);
  if (valid && sub == 0) {
    if (!isfinite(gq.sf)) latch_error(err, WQ_ERR_RANGE);
    steps[n * G + gi] = gq.step_h;
    zeros[n * G + gi] = __int2half_rn(gq.zero);
  }
  uint32_t q[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) q[i] = group_quant_code<BITS, SYM>(w[i], gq);
  if (!valid) return;

  if (BITS == 4) {
    // word c holds channels 8c..8c+7 in slot order [0, 2, 4, 6, 1, 3, 5, 7]
    uint4 out;
    uint32_t* o = reinterpret_cast<uint32_t*>(&out);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint32_t* v = q + 8 * c;
      o[c] = v[0] | (v[2] << 4) | (v[4] << 8) | (v[6] << 12) | (v[1] << 16) | (v[3] << 20) | (v[5] << 24) |
             (v[7] << 28);
    }
    *reinterpret_cast<uint4*>(packed + (n * K + k0) / 8) = out;
  } else {
    // the lane's 32 channels are one 3-word chunk: word t holds channel pairs
    // (10t + 2j, 10t + 2j + 1) at bits 3j and 16 + 3j, and bit t of channels
    // 30 / 31 at bit 15 / 31
    uint32_t o[3];
#pragma unroll
    for (int t = 0; t < 3; ++t) {
      uint32_t word = 0;
#pragma unroll
      for (int j = 0; j < 5; ++j) word |= (q[10 * t + 2 * j] << (3 * j)) | (q[10 * t + 2 * j + 1] << (16 + 3 * j));
      word |= ((q[30] >> t) & 1u) << 15;
      word |= ((q[31] >> t) & 1u) << 31;
      o[t] = word;
    }
    uint32_t* dst = packed + (n * K + k0) / 32 * 3;
    dst[0] = o[0];
    dst[1] = o[1];
    dst[2] = o[2];
  }
}

// Inverse: one thread per 8 (4-bit) or 32 (3-bit) weights.
template <int BITS>
__global__ void __launch_bounds__(256)
unpack_dequant_kernel(const uint32_t* __restrict__ packed, const __half* __restrict__ steps,
                      const __half* __restrict__ zeros, int64_t N, int64_t K, __half* __restrict__ out) {
  constexpr int PER = BITS == 4 ? 8 : 32;
  const int64_t units = N * K / PER;
  const int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (u >= units) return;
  const int64_t e0 = u * PER;  // first element (row-major)
  const int64_t n = e0 / K;
  const int64_t k = e0 % K;
  const int64_t gidx = n * (K / kGroup) + k / kGroup;
  const float sf = __half2float(steps[gidx]);
  const float z = __half2float(zeros[gidx]);
  int q[PER];
  if (BITS == 4) {
    const uint32_t w = packed[u];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      q[2 * j] = (w >> (4 * j)) & 0xF;
      q[2 * j + 1] = (w >> (4 * (j + 4))) & 0xF;
    }
  } else {
    const uint32_t w3[3] = {packed[3 * u], packed[3 * u + 1], packed[3 * u + 2]};
#pragma unroll
    for (int t = 0; t < 3; ++t) {
#pragma unroll
      for (int j = 0; j < 5; ++j) {
        q[10 * t + 2 * j] = (w3[t] >> (3 * j)) & 7;
        q[10 * t + 2 * j + 1] = (w3[t] >> (16 + 3 * j)) & 7;
      }
    }
    q[30] = ((w3[0] >> 15) & 1) | (((w3[1] >> 15) & 1) << 1) | (((w3[2] >> 15) & 1) << 2);
    q[31] = ((w3[0] >> 31) & 1) | (((w3[1] >> 31) & 1) << 1) | (((w3[2] >> 31) & 1) << 2);
  }
#pragma unroll
  for (int i = 0; i < PER; i += 2) {
    // (q - z) * step is exact in fp32; one rounding to fp16.
    const float a = __fmul_rn((float)q[i] - z, sf);
    const float b = __fmul_rn((float)q[i + 1] - z, sf);
    *reinterpret_cast<__half2*>(out + e0 + i) = __floats2half2_rn(a, b);
  }
}

cudaError_t launch_quantize_pack(const void* W, const void* s, int64_t N, int64_t K, int bits, bool sym,
                                 uint32_t* packed, void* steps, void* zeros, int* err, cudaStream_t st) {
  const int64_t groups = N * (K / kGroup);
  const dim3 grid((unsigned)((groups + 63) / 64));  // 4 lanes per group
  const dim3 block(256);
  auto Wp = static_cast<const __half*>(W);
  auto sp = static_cast<const __half*>(s);
  auto stp = static_cast<__half*>(steps);
  auto zp = static_cast<__half*>(zeros);
#define WQ_QP(B, S, H) quantize_pack_kernel<B, S, H><<<grid, block, 0, st>>>(Wp, sp, N, K, packed, stp, zp, err)
  if (bits == 4) {
    if (sym) { if (s) WQ_QP(4, true, true); else WQ_QP(4, true, false); }
    else     { if (s) WQ_QP(4, false, true); else WQ_QP(4, false, false); }
  } else {
    if (sym) { if (s) WQ_QP(3, true, true); else WQ_QP(3, true, false); }
    else     { if (s) WQ_QP(3, false, true); else WQ_QP(3, false, false); }
  }
#undef WQ_QP
  return cudaGetLastError();
}

cudaError_t launch_unpack_dequant(const uint32_t* packed, const void* steps, const void* zeros, int64_t N,
                                  int64_t K, int bits, void* out, cudaStream_t st) {
  const int per = bits == 4 ? 8 : 32;
  const int64_t units = N * K / per;
  const dim3 grid((unsigned)((units + 255) / 256));
  if (bits == 4)
    unpack_dequant_kernel<4><<<grid, 256, 0, st>>>(packed, static_cast<const __half*>(steps),
                                                   static_cast<const __half*>(zeros), N, K,
                                                   static_cast<__half*>(out));
  else
    unpack_dequant_kernel<3><<<grid, 256, 0, st>>>(packed, static_cast<const __half*>(steps),
                                                   static_cast<const __half*>(zeros), N, K,
                                                   static_cast<__half*>(out));
  return cudaGetLastError();
}

}  // namespace wq
