// Shared device helpers for the wq kernels (sm_100a).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/wq.h"

namespace wq {

constexpr int kGroup = 128;          // quantization group (input channels)
constexpr uint32_t kHalf2Magic = 0x64006400u;  // fp16 1024.0 in both lanes

// Latch the first device-side error of a launch sequence. The flag lives in
// the library (one per device); kernels receive its address.
__device__ __forceinline__ void latch_error(int* flag, int code) {
  if (flag != nullptr) atomicCAS(flag, 0, code);
}

// (a & b) | c in one LOP3.
__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// Streaming 128-bit load of data read exactly once (packed weights): skip L1.
__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ uint32_t ld_stream_u32(const void* p) {
  uint32_t r;
  asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(r) : "l"(p));
  return r;
}

__device__ __forceinline__ float half_bits_to_float(uint16_t h) {
  return __half2float(__ushort_as_half(h));
}

// acc += lo(a) * lo(b) ; acc2 += hi(a) * hi(b), fp16 x fp16 products
// accumulated in fp32 (the products are exact in fp32).
__device__ __forceinline__ void fma2_f16_f32(float& acc_lo, float& acc_hi, uint32_t a, uint32_t b) {
  asm("{\n\t.reg .f16 al, ah, bl, bh;\n\t"
      "mov.b32 {al, ah}, %2;\n\t"
      "mov.b32 {bl, bh}, %3;\n\t"
      "fma.rn.f32.f16 %0, al, bl, %0;\n\t"
      "fma.rn.f32.f16 %1, ah, bh, %1;\n\t}"
      : "+f"(acc_lo), "+f"(acc_hi)
      : "r"(a), "r"(b));
}

}  // namespace wq
