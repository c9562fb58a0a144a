// S3: group-wise quantize + pack, and the inverse (unpack + dequantize).
//
// Quantizer: "LLM Quantization: 160GB Model on a Laptop", sections "Symmetric
// Quantization" and "Asymmetric Quantization"; integer zero point as in "CMU
// 11-868 L19-L20 Model Quantization", section "absmax and zero-point"; one
// step and zero per group of 32, 64 or 128 input channels of a row
// ("Quantising Large Language Models for Efficient Inference", "Post-training
// methods for 4-bit weights").
// Optional AWQ input-channel scaling W * diag(s) first ("MIT 6.5940 Lab 4 +
// Lab 5", "Question 2").
//
// Mapping: a lane unit is 32 consecutive input channels of one group, g / 32
// lanes per group (four 16-byte loads of W; one 16-byte store of 4-bit codes,
// or the three words of a 3-bit chunk); the group's range is reduced with
// log2(g / 32) xor-shuffles (none for g = 32). One wave of resident CTAs walks the units grid-stride, the
// next unit's loads in flight while the current one is quantized. Per weight:
// the correctly rounded quotient without a division (group_quotient), rint by
// the 1.5 * 2^23 addition (both on packed fp32 pairs, two channels per
// instruction), and one integer multiply-add into the packed word.
// 2 B/weight in, 0.5 (0.375) B/weight out.
#include <type_traits>

#include "wq_quant_core.cuh"
#include "wq_launch.h"

namespace wq {

// A lane's 32 codes packed: four 4-bit words, or one 3-bit chunk of three.
// level(i) returns the offset level of channel i (group_offset_level).
template <int BITS, class F>
__device__ __forceinline__ void pack_lane(F level, int zero, uint32_t (&o)[4]) {
  if constexpr (BITS == 4) {
#pragma unroll
    for (int c = 0; c < 4; ++c) o[c] = pack_word4([&](int i) { return level(8 * c + i); }, zero);
  } else {
    uint32_t t[3];
    pack_chunk3(level, zero, t);
    o[0] = t[0], o[1] = t[1], o[2] = t[2], o[3] = 0;
  }
}

// One lane unit u: channels [32u, 32u + 32) of the row-major weight, 1/LPG of
// group u / LPG (LPG = group size / 32 lanes per group: 4, 2 or 1). The
// group's decision (shared by its LPG lanes), then the lane's 32 codes,
// packed and stored. sk: the unit's 32 AWQ scales.
template <int BITS, bool SYM, bool HAS_S, int LPG>
__device__ __forceinline__ void quantize_unit(const uint4 (&raw)[4], const __half* __restrict__ sk, int64_t u,
                                              bool valid, uint32_t* __restrict__ packed,
                                              __half* __restrict__ steps, __half* __restrict__ zeros, int* err) {
  // with AWQ scaling the products w * s in fp32 (exact: 11 x 11 significand
  // bits; a zero product is +0 whatever the signs, which no decision sees)
  float ws[HAS_S ? 32 : 1];
  GroupQuant gq;
  if constexpr (HAS_S) {
    uint4 sr[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) sr[c] = valid ? *reinterpret_cast<const uint4*>(sk + 8 * c) : make_uint4(0, 0, 0, 0);
    // w * s straight from the fp16 pairs with the mixed fp16 x fp16 -> fp32
    // fma (exact product, plus zero)
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      ws[2 * i] = 0.f;
      ws[2 * i + 1] = 0.f;
      fma2_f16_f32(ws[2 * i], ws[2 * i + 1], (&raw[i >> 2].x)[i & 3], (&sr[i >> 2].x)[i & 3]);
    }
    gq = group_quant_decide<BITS, SYM, 32, LPG>(ws);
  } else {
    gq = group_quant_decide_h<BITS, SYM, LPG>(raw);
  }
  if (valid && (u % LPG) == 0) {
    if (!isfinite(gq.sf)) latch_error(err, WQ_ERR_RANGE);
    steps[u / LPG] = gq.step_h;
    zeros[u / LPG] = __int2half_rn(gq.zero);
  }
  auto value = [&](int i) -> float {
    if constexpr (HAS_S) return ws[i]; else return lane_half(raw, i);
  };

  // the 32 offset levels, two channels per packed fp32 instruction
  const uint64_t rcp2 = f2_pack(gq.rcp, gq.rcp);
  const uint64_t nsf2 = f2_pack(-gq.sf, -gq.sf);
  const uint64_t magic2 = f2_pack(kRoundMagic, kRoundMagic);
  float lv[32];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float2 l = group_offset_level2<BITS, SYM>(value(2 * i), value(2 * i + 1), gq, rcp2, nsf2, magic2);
    lv[2 * i] = l.x;
    lv[2 * i + 1] = l.y;
  }
  uint32_t o[4];
  pack_lane<BITS>([&](int i) { return lv[i]; }, gq.zero, o);
  if (!valid) return;

  if constexpr (BITS == 4) {
    reinterpret_cast<uint4*>(packed)[u] = make_uint4(o[0], o[1], o[2], o[3]);
  } else {
    uint32_t* dst = packed + 3 * u;
    dst[0] = o[0];
    dst[1] = o[1];
    dst[2] = o[2];
  }
}

template <int BITS, bool SYM, bool HAS_S, int LPG>
__global__ void __launch_bounds__(256)
quantize_pack_kernel(const __half* __restrict__ W, const __half* __restrict__ s, int64_t N, int64_t K,
                     uint32_t* __restrict__ packed, __half* __restrict__ steps,
                     __half* __restrict__ zeros, int* err) {
  // Grid-stride over lane units (a lane's 32 channels of one group; unit u
  // starts at element 32u of the row-major weight); the next unit's 64 bytes
  // of W are in flight while this one is quantized.
  const int lane = threadIdx.x & 31;
  const int64_t units = N * K / 32;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const uint4* w4 = reinterpret_cast<const uint4*>(W);
  // the column of unit u, tracked for the AWQ scales only
  const int64_t kunits = K / 32, step_cols = stride % kunits;
  int64_t col = HAS_S ? u % kunits : 0;

  auto load = [&](uint4 (&r)[4]) {
#pragma unroll
    for (int c = 0; c < 4; ++c) r[c] = u < units ? w4[4 * u + c] : make_uint4(0, 0, 0, 0);
  };
  uint4 next[4];
  load(next);
  while (u - lane < units) {  // warp-uniform: the group shuffles need every lane
    const int64_t cur = u;
    const __half* sk = HAS_S ? s + 32 * col : nullptr;
    uint4 raw[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) raw[c] = next[c];
    u += stride;
    if (HAS_S) {
      col += step_cols;
      if (col >= kunits) col -= kunits;
    }
    load(next);
    quantize_unit<BITS, SYM, HAS_S, LPG>(raw, sk, cur, cur < units, packed, steps, zeros, err);
  }
}

// Inverse: one thread per 8 (4-bit) or 32 (3-bit) weights (never across a
// group: groups are 32, 64 or 128 channels).
template <int BITS>
__global__ void __launch_bounds__(256)
unpack_dequant_kernel(const uint32_t* __restrict__ packed, const __half* __restrict__ steps,
                      const __half* __restrict__ zeros, int64_t N, int64_t K, int group, __half* __restrict__ out) {
  constexpr int PER = BITS == 4 ? 8 : 32;
  const int64_t units = N * K / PER;
  const int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (u >= units) return;
  const int64_t e0 = u * PER;  // first element (row-major)
  const int64_t n = e0 / K;
  const int64_t k = e0 % K;
  const int64_t gidx = n * (K / group) + k / group;
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

cudaError_t launch_quantize_pack(const void* W, const void* s, int64_t N, int64_t K, int bits, int group, bool sym,
                                 uint32_t* packed, void* steps, void* zeros, int* err, cudaStream_t st) {
  const int64_t units = N * K / 32;  // lane units of 32 channels
  const dim3 block(256);
  auto Wp = static_cast<const __half*>(W);
  auto sp = static_cast<const __half*>(s);
  auto stp = static_cast<__half*>(steps);
  auto zp = static_cast<__half*>(zeros);
  // one wave of resident blocks (fewer when the matrix is small)
  auto launch = [&](auto kern) {
    static const int resident = [&] {
      int dev = 0, sms = 0, occ = 0;
      cudaGetDevice(&dev);
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, 256, 0);
      return (sms > 0 ? sms : 1) * (occ > 0 ? occ : 1);
    }();
    const int64_t need = (units + 255) / 256;
    const dim3 grid((unsigned)(need < resident ? need : resident));
    kern<<<grid, block, 0, st>>>(Wp, sp, N, K, packed, stp, zp, err);
  };
  auto by_group = [&](auto bits_c, auto sym_c, auto s_c) {
    constexpr int B = decltype(bits_c)::value;
    constexpr bool S = decltype(sym_c)::value, H = decltype(s_c)::value;
    if (group == 32) launch(quantize_pack_kernel<B, S, H, 1>);
    else if (group == 64) launch(quantize_pack_kernel<B, S, H, 2>);
    else launch(quantize_pack_kernel<B, S, H, 4>);
  };
  using T = std::true_type;
  using F = std::false_type;
  using B4 = std::integral_constant<int, 4>;
  using B3 = std::integral_constant<int, 3>;
  if (bits == 4) {
    if (sym) { if (s) by_group(B4{}, T{}, T{}); else by_group(B4{}, T{}, F{}); }
    else     { if (s) by_group(B4{}, F{}, T{}); else by_group(B4{}, F{}, F{}); }
  } else {
    if (sym) { if (s) by_group(B3{}, T{}, T{}); else by_group(B3{}, T{}, F{}); }
    else     { if (s) by_group(B3{}, F{}, T{}); else by_group(B3{}, F{}, F{}); }
  }
  return cudaGetLastError();
}

cudaError_t launch_unpack_dequant(const uint32_t* packed, const void* steps, const void* zeros, int64_t N,
                                  int64_t K, int bits, int group, void* out, cudaStream_t st) {
  const int per = bits == 4 ? 8 : 32;
  const int64_t units = N * K / per;
  const dim3 grid((unsigned)((units + 255) / 256));
  if (bits == 4)
    unpack_dequant_kernel<4><<<grid, 256, 0, st>>>(packed, static_cast<const __half*>(steps),
                                                   static_cast<const __half*>(zeros), N, K, group,
                                                   static_cast<__half*>(out));
  else
    unpack_dequant_kernel<3><<<grid, 256, 0, st>>>(packed, static_cast<const __half*>(steps),
                                                   static_cast<const __half*>(zeros), N, K, group,
                                                   static_cast<__half*>(out));
  return cudaGetLastError();
}

}  // namespace wq
