// S5 for M <= 2 (4- and 3-bit) and M <= 4 (4-bit, K <= 8192): row-streaming
// decode GEMV with activations in registers.
//
// The decode GEMV streams the packed weight once ("MIT 6.5940 Lab 4 + Lab 5",
// "Starting point and setup"; "CMU 11-868 L19-L20", "where does the speed
// come from?"), so the instructions spent per weight, not the arithmetic,
// decide how close it gets to HBM bandwidth. This kernel keeps that count
// minimal:
//   * K is split across the warps of a CTA: warp w, lane l owns the LK = 32
//     or 64 consecutive input channels (w*32 + l)*LK .. +LK-1 for the whole
//     kernel. Its activations live in registers, loaded once -- no
//     shared-memory copy of X, no split-K, no clusters.
//   * A CTA streams batches of R consecutive rows (persistent over row
//     batches). Per row a lane issues LK/32 16-byte loads, and a warp reads
//     16*LK contiguous bytes. The next batch is loaded while the current one
//     is computed (two register stages); the first batch is requested before
//     the programmatic-dependent-launch wait, since only X depends on the
//     previous kernel.
//   * Per batch the R x M partials are reduced across lanes with butterflies
//     that halve the value count at each exchange. For ActHalf and ActHalf3
//     the halvings run over the lanes of one quantization group first, so the
//     step, the zero point and the 1024 offsets are applied once per group
//     total (group-first reduction); the remaining lane bits finish the sum.
//     ActInt and ActW4A8 scale per lane (their scales are per lane) before
//     the reduction.
//     Across warps the totals meet in shared memory in warp order
//     (deterministic), once per 32/(R*M) batches, so the CTA meets at a
//     barrier only that often.
//
// Activation classes (how a lane forms its sum over its channels):
//   ActHalf (4-bit, default, WQ_GEMV_OFFSET_SUMS): one LOP3 with 0x6400 in
//     both fp16 lanes gives (1024 + q, 1024 + q') or (1024 + 16q,
//     1024 + 16q'); a mixed fp16 x fp16 -> fp32 FMA multiplies it by the
//     activation pair (exact products, fp32 sums). The offsets and the zero
//     point are removed per group total with the lane's activation class
//     sums.
//   ActHalf3 (3-bit): the same with pairs (1024 + q * {1, 8, 64}) taken from
//     three words per 32 channels.
//   ActInt (4-bit, WQ_GEMV_INT_DIGITS): the lane's activations become one
//     24-bit fixed-point image x_k ~ X_k 2^-F (F per lane and row of X,
//     |X_k| < 2^22, so every fp16 value within 2^-13 of the lane's largest is
//     exact and the others are rounded by at most 2^-23 of it), split into
//     three base-256 digits. A packed code word masked with 0xF0F0F0F0 --
//     before and after a 4-bit shift -- holds 16 q of four channels in its
//     bytes, and dp4a multiplies them by four digits at once. Every product
//     and sum is an exact integer; the zero point is removed per digit in
//     integers, and the only roundings are the fixed-point image and the
//     final fp32 combination of three digit sums per row and lane.
//   ActW4A8 (W4A8): int8 activation codes permuted to the packed byte order,
//     exact dp4a group dot products, scaled by step / multiplier per lane.
#include <type_traits>

#include "wq_common.cuh"
#include "wq_launch.h"

namespace wq {

struct RowsArgs {
  const __half* X;
  const uint32_t* P;
  const __half* steps;
  const __half* zeros;
  __half* Y;
  int N, K;
  int Mv;  // rows of X present (<= the kernel's M; the rest read as zeros and are not stored)
  const int8_t* Xq;   // W4A8: int8 activation codes [M][K] (X unused)
  const float* mult;  // W4A8: their multipliers [M][K / group]
};

// One row batch of this lane: WPR packed words per row (4-bit: 4 per 32
// channels, 3-bit: 3 per 32 channels) and the step and zero of RL rows: all R
// rows, or (group-first reduction) the RL rows whose group totals this lane
// finishes.
template <int R, int WPR, int RL = R>
struct RowsStage {
  uint32_t w[R][WPR];
  __half sc[RL], zh[RL];
};

__device__ __forceinline__ uint2 ld_stream_v2(const void* p) {
  uint2 r;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
  return r;
}

template <int WPR>
__device__ __forceinline__ void load_row_words(uint32_t (&w)[WPR], const uint32_t* p) {
  if constexpr (WPR % 4 == 0) {
#pragma unroll
    for (int c = 0; c < WPR / 4; ++c) {
      const uint4 v = ld_stream_v4(p + 4 * c);
      w[4 * c] = v.x; w[4 * c + 1] = v.y; w[4 * c + 2] = v.z; w[4 * c + 3] = v.w;
    }
  } else {
    static_assert(WPR % 2 == 0, "row words come in 8-byte pairs");
#pragma unroll
    for (int c = 0; c < WPR / 2; ++c) {
      const uint2 v = ld_stream_v2(p + 2 * c);
      w[2 * c] = v.x; w[2 * c + 1] = v.y;
    }
  }
}

// Loads of one row batch for this lane: pw / ps / pz point at the lane's words,
// step and zero in the batch's first row; nrows = rows of the batch inside N
// (0 for a lane past K); the step and zero are those of rows lrow0 .. lrow0 +
// RL - 1 of the batch. Full batches take the unpredicated path.
template <int R, int WPR, int RL>
__device__ __forceinline__ void rows_issue(RowsStage<R, WPR, RL>& s, const uint32_t* pw, const __half* ps,
                                           const __half* pz, size_t row_words, int G, int nrows, int lrow0) {
  if (nrows >= R) {
#pragma unroll
    for (int r = 0; r < R; ++r) load_row_words<WPR>(s.w[r], pw + r * row_words);
#pragma unroll
    for (int i = 0; i < RL; ++i) {
      s.sc[i] = ps[(size_t)(lrow0 + i) * G];
      s.zh[i] = pz[(size_t)(lrow0 + i) * G];
    }
  } else {
#pragma unroll
    for (int r = 0; r < R; ++r) {
      if (r < nrows) {
        load_row_words<WPR>(s.w[r], pw + r * row_words);
      } else {
#pragma unroll
        for (int c = 0; c < WPR; ++c) s.w[r][c] = 0;
      }
    }
#pragma unroll
    for (int i = 0; i < RL; ++i) {
      const bool in = lrow0 + i < nrows;
      s.sc[i] = in ? ps[(size_t)(lrow0 + i) * G] : __float2half(0.f);
      s.zh[i] = in ? pz[(size_t)(lrow0 + i) * G] : __float2half(0.f);
    }
  }
}


// The lane's LK = 32*CPL activations of each of the M rows of X.
template <int M, int CPL>
__device__ __forceinline__ void load_lane_x(uint32_t (&xh)[M][16 * CPL], const RowsArgs& a, int k0, bool active) {
#pragma unroll
  for (int m = 0; m < M; ++m) {
#pragma unroll
    for (int j = 0; j < 4 * CPL; ++j) {
      uint4 v = make_uint4(0, 0, 0, 0);
      if (active && m < a.Mv) v = *reinterpret_cast<const uint4*>(a.X + (size_t)m * a.K + k0 + 8 * j);
      xh[m][4 * j] = v.x; xh[m][4 * j + 1] = v.y; xh[m][4 * j + 2] = v.z; xh[m][4 * j + 3] = v.w;
    }
  }
}

// ---------------------------------------------------------------- ActHalf
// Group totals of a lane's offset term c1 and activation sum: the LPG lanes
// of one quantization group (group size / channels per lane) share step and
// zero, so the zero point and the offsets are removed once per group
// (group-first reduction).
template <int M, int LPG>
__device__ __forceinline__ void group_totals(const float (&c1)[M], const float (&xsum)[M], float (&c1g)[M],
                                             float (&xg)[M]) {
#pragma unroll
  for (int m = 0; m < M; ++m) {
    float c = c1[m], x = xsum[m];
#pragma unroll
    for (int o = 1; o < LPG; o <<= 1) {
      c += __shfl_xor_sync(0xffffffffu, c, o);
      x += __shfl_xor_sync(0xffffffffu, x, o);
    }
    c1g[m] = c;
    xg[m] = x;
  }
}

// step * (T - c1g - zero * xg) for a group total T of activation row m.
template <int M>
__device__ __forceinline__ float group_epilogue(const float (&c1g)[M], const float (&xg)[M], int m, float t,
                                                __half sc, __half zh) {
  // m is a compile-time index wherever this is inlined (unrolled value loops)
  return __half2float(sc) * fmaf(-__half2float(zh), xg[m], t - c1g[m]);
}

template <int M, int CPL>
struct ActHalf {
  static constexpr bool kGroupFirst = true;  // compute() leaves step and zero to the group epilogue
  uint32_t xh[M][16 * CPL];
  float c1g[M], xg[M];

  template <int LPG>
  __device__ __forceinline__ void load(const RowsArgs& a, int k0, bool active) {
    load_lane_x<M, CPL>(xh, a, k0, active);
    float c1[M], xsum[M];
#pragma unroll
    for (int m = 0; m < M; ++m) {
      float x1 = 0.f, x2 = 0.f;  // channel classes {0,1,4,5} and {2,3,6,7} mod 8
#pragma unroll
      for (int i = 0; i < 16 * CPL; ++i) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&xh[m][i]));
        if ((i & 1) == 0) x1 += f.x + f.y;
        else x2 += f.x + f.y;
      }
      c1[m] = 1024.f * x1 + 64.f * x2;
      xsum[m] = x1 + x2;
    }
    group_totals<M, LPG>(c1, xsum, c1g, xg);
  }

  __device__ __forceinline__ float epilogue(int m, float t, __half sc, __half zh) const {
    return group_epilogue<M>(c1g, xg, m, t, sc, zh);
  }

  // acc[r*M + m] = this lane's A1 + A2/16 (sum_k x (1024 + q) with the x16
  // class scaled back), before the offsets, the zero point and the step.
  template <int R, int RL>
  __device__ __forceinline__ void compute(const RowsStage<R, 4 * CPL, RL>& s, float (&acc)[R * M]) const {
#pragma unroll
    for (int r = 0; r < R; ++r) {
      float a[M][4];
#pragma unroll
      for (int m = 0; m < M; ++m) a[m][0] = a[m][1] = a[m][2] = a[m][3] = 0.f;
#pragma unroll
      for (int j = 0; j < 4 * CPL; ++j) {
        const uint32_t w = s.w[r][j];
        const uint32_t w8 = w >> 8;
        const uint32_t p0 = and_or(w, 0x000F000Fu, kHalf2Magic);   // k+0,k+1   x1
        const uint32_t p1 = and_or(w, 0x00F000F0u, kHalf2Magic);   // k+2,k+3   x16
        const uint32_t p2 = and_or(w8, 0x000F000Fu, kHalf2Magic);  // k+4,k+5   x1
        const uint32_t p3 = and_or(w8, 0x00F000F0u, kHalf2Magic);  // k+6,k+7   x16
#pragma unroll
        for (int m = 0; m < M; ++m) {
          fma2_f16_f32(a[m][0], a[m][1], xh[m][4 * j + 0], p0);
          fma2_f16_f32(a[m][2], a[m][3], xh[m][4 * j + 1], p1);
          fma2_f16_f32(a[m][0], a[m][1], xh[m][4 * j + 2], p2);
          fma2_f16_f32(a[m][2], a[m][3], xh[m][4 * j + 3], p3);
        }
      }
#pragma unroll
      for (int m = 0; m < M; ++m)  // sum_k x (q - z) = A1 + A2/16 - (1024 X1 + 64 X2) - z (X1 + X2)
        acc[r * M + m] = fmaf(a[m][2] + a[m][3], 0.0625f, a[m][0] + a[m][1]);
    }
  }
};

// ---------------------------------------------------------------- ActHalf3
// 3-bit rows: per 32 channels three words; word t holds the channel pairs
// (10t + 2j, 10t + 2j + 1) at bits 3j and 16 + 3j (j < 5), and bit t of
// channels 30 / 31 at bit 15 / 31. A LOP3 with 0x6400 leaves pair j of a word
// as (1024 + q, 1024 + q') times 1 (j = 0), 8 (j = 1) or 64 (j = 2); after a
// 9-bit shift pairs 3 and 4 follow as x1 and x8. Three shifted LOP3s gather
// the bits of channels 30 and 31. The offsets and the zero point are removed
// per row with the lane's activation class sums, as in ActHalf.
template <int M, int CPL>
struct ActHalf3 {
  static constexpr bool kGroupFirst = true;  // compute() leaves step and zero to the group epilogue
  uint32_t xh[M][16 * CPL];
  float c1g[M], xg[M];

  __device__ __forceinline__ float epilogue(int m, float t, __half sc, __half zh) const {
    return group_epilogue<M>(c1g, xg, m, t, sc, zh);
  }

  template <int LPG>
  __device__ __forceinline__ void load(const RowsArgs& a, int k0, bool active) {
    load_lane_x<M, CPL>(xh, a, k0, active);
    float c1[M], xsum[M];
#pragma unroll
    for (int m = 0; m < M; ++m) {
      float x1 = 0.f, x8 = 0.f, x64 = 0.f;
#pragma unroll
      for (int i = 0; i < 16 * CPL; ++i) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&xh[m][i]));
        const int wi = i & 15;  // x word within the 32-channel chunk
        const int j = wi % 5;
        if (wi == 15 || j == 0 || j == 3) x1 += f.x + f.y;
        else if (j == 2) x64 += f.x + f.y;
        else x8 += f.x + f.y;
      }
      c1[m] = 1024.f * x1 + 128.f * x8 + 16.f * x64;
      xsum[m] = x1 + x8 + x64;
    }
    group_totals<M, LPG>(c1, xsum, c1g, xg);
  }

  // acc[r*M + m] = this lane's A1 + A8/8 + A64/64, before the offsets, the
  // zero point and the step.
  template <int R, int RL>
  __device__ __forceinline__ void compute(const RowsStage<R, 3 * CPL, RL>& s, float (&acc)[R * M]) const {
#pragma unroll
    for (int r = 0; r < R; ++r) {
      float a[M][6];  // (x1, x8, x64) classes, low and high lanes
#pragma unroll
      for (int m = 0; m < M; ++m)
#pragma unroll
        for (int i = 0; i < 6; ++i) a[m][i] = 0.f;
#pragma unroll
      for (int c = 0; c < CPL; ++c) {
        const uint32_t w0 = s.w[r][3 * c], w1 = s.w[r][3 * c + 1], w2 = s.w[r][3 * c + 2];
        const uint32_t wt[3] = {w0, w1, w2};
#pragma unroll
        for (int t = 0; t < 3; ++t) {
          const uint32_t w = wt[t];
          const uint32_t w9 = w >> 9;
          const uint32_t p0 = and_or(w, 0x00070007u, kHalf2Magic);   // x1
          const uint32_t p1 = and_or(w, 0x00380038u, kHalf2Magic);   // x8
          const uint32_t p2 = and_or(w, 0x01C001C0u, kHalf2Magic);   // x64
          const uint32_t p3 = and_or(w9, 0x00070007u, kHalf2Magic);  // x1
          const uint32_t p4 = and_or(w9, 0x00380038u, kHalf2Magic);  // x8
          const int xw = 16 * c + 5 * t;
#pragma unroll
          for (int m = 0; m < M; ++m) {
            fma2_f16_f32(a[m][0], a[m][1], xh[m][xw + 0], p0);
            fma2_f16_f32(a[m][2], a[m][3], xh[m][xw + 1], p1);
            fma2_f16_f32(a[m][4], a[m][5], xh[m][xw + 2], p2);
            fma2_f16_f32(a[m][0], a[m][1], xh[m][xw + 3], p3);
            fma2_f16_f32(a[m][2], a[m][3], xh[m][xw + 4], p4);
          }
        }
        uint32_t p30 = and_or(w0 >> 15, 0x00010001u, kHalf2Magic);
        p30 = and_or(w1 >> 14, 0x00020002u, p30);
        p30 = and_or(w2 >> 13, 0x00040004u, p30);
#pragma unroll
        for (int m = 0; m < M; ++m) fma2_f16_f32(a[m][0], a[m][1], xh[m][16 * c + 15], p30);
      }
#pragma unroll
      for (int m = 0; m < M; ++m)
        // sum_k x (q - z) = A1 + A8/8 + A64/64 - (1024 X1 + 128 X8 + 16 X64) - z (X1 + X8 + X64)
        acc[r * M + m] = fmaf(a[m][4] + a[m][5], 0.015625f, fmaf(a[m][2] + a[m][3], 0.125f, a[m][0] + a[m][1]));
    }
  }
};

// ---------------------------------------------------------------- ActInt
__device__ __forceinline__ int dp4a_uu(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.u32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ uint32_t pack_bytes(int b0, int b1, int b2, int b3) {
  return (uint32_t)(b0 & 0xFF) | ((uint32_t)(b1 & 0xFF) << 8) | ((uint32_t)(b2 & 0xFF) << 16) |
         ((uint32_t)(b3 & 0xFF) << 24);
}

template <int M, int CPL>
struct ActInt {
  static constexpr bool kGroupFirst = false;  // per-lane fixed-point scale: step applied per lane
  // Digit t of the fixed-point image, four channels per word in the byte
  // order of the masked code words: lo[c] holds channels 8c + (0, 4, 1, 5)
  // (the low nibbles of the word's bytes), hi[c] channels 8c + (2, 6, 3, 7).
  uint32_t lo[M][3][4 * CPL], hi[M][3][4 * CPL];
  int d16[M][3];  // 16 * sum over the lane's channels of digit t
  float inv[M];   // 2^-(F + 4): undoes the image scale and the 16 of the masked codes

  template <int LPG>
  __device__ __forceinline__ void load(const RowsArgs& a, int k0, bool active) {
    uint32_t xh[M][16 * CPL];
    load_lane_x<M, CPL>(xh, a, k0, active);
#pragma unroll
    for (int m = 0; m < M; ++m) {
      float mx = 0.f;
#pragma unroll
      for (int i = 0; i < 16 * CPL; ++i) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&xh[m][i]));
        mx = fmaxf(mx, fmaxf(fabsf(f.x), fabsf(f.y)));
      }
      // 2^(e-1) <= mx < 2^e; F = 22 - e keeps |x| 2^F <= 2^22. mx is 0 or at
      // least 2^-24 (an fp16 value), so e lies in [-23, 17] and F in [5, 45].
      const int e = mx > 0.f ? (int)((__float_as_uint(mx) >> 23) & 0xFF) - 126 : 22;
      const int F = 22 - e;
      const float scale = __uint_as_float((uint32_t)(F + 127) << 23);
      inv[m] = __uint_as_float((uint32_t)(127 - F - 4) << 23);
      int sum[3] = {0, 0, 0};
#pragma unroll
      for (int c = 0; c < 4 * CPL; ++c) {
        int xi[8];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&xh[m][4 * c + h]));
          xi[2 * h] = __float2int_rn(f.x * scale);
          xi[2 * h + 1] = __float2int_rn(f.y * scale);
        }
#pragma unroll
        for (int t = 0; t < 3; ++t) {
          int d[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            d[i] = t == 2 ? (xi[i] >> 16) : ((xi[i] >> (8 * t)) & 0xFF);  // top digit signed
            sum[t] += d[i];
          }
          lo[m][t][c] = pack_bytes(d[0], d[4], d[1], d[5]);
          hi[m][t][c] = pack_bytes(d[2], d[6], d[3], d[7]);
        }
      }
#pragma unroll
      for (int t = 0; t < 3; ++t) d16[m][t] = 16 * sum[t];
    }
  }

  __device__ __forceinline__ float epilogue(int, float t, __half, __half) const { return t; }

  template <int R, int RL>
  __device__ __forceinline__ void compute(const RowsStage<R, 4 * CPL, RL>& s, float (&acc)[R * M]) const {
    static_assert(RL == R, "the integer-digit path applies every row's step per lane");
    // Words outer, rows inner: R*M*3 independent dp4a chains.
    int a[R][M][3];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int m = 0; m < M; ++m) a[r][m][0] = a[r][m][1] = a[r][m][2] = 0;
#pragma unroll
    for (int j = 0; j < 4 * CPL; ++j) {
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const uint32_t w = s.w[r][j];
        const uint32_t l16 = (w << 4) & 0xF0F0F0F0u;  // 16 q of channels 0, 4, 1, 5
        const uint32_t h16 = w & 0xF0F0F0F0u;         // 16 q of channels 2, 6, 3, 7
#pragma unroll
        for (int m = 0; m < M; ++m) {
          a[r][m][0] = dp4a_uu(l16, lo[m][0][j], a[r][m][0]);
          a[r][m][1] = dp4a_uu(l16, lo[m][1][j], a[r][m][1]);
          a[r][m][2] = dp4a_us(l16, lo[m][2][j], a[r][m][2]);
          a[r][m][0] = dp4a_uu(h16, hi[m][0][j], a[r][m][0]);
          a[r][m][1] = dp4a_uu(h16, hi[m][1][j], a[r][m][1]);
          a[r][m][2] = dp4a_us(h16, hi[m][2][j], a[r][m][2]);
        }
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
      // Zero points are integers in [0, 15]; 16 sum_k (q - z) d_t is exact in
      // int32 and below 2^24 in magnitude, so exact in fp32 too.
      const int z = __half2int_rn(s.zh[r]);
      const float sc = __half2float(s.sc[r]);
#pragma unroll
      for (int m = 0; m < M; ++m) {
        const float e0 = (float)(a[r][m][0] - z * d16[m][0]);
        const float e1 = (float)(a[r][m][1] - z * d16[m][1]);
        const float e2 = (float)(a[r][m][2] - z * d16[m][2]);
        acc[r * M + m] = sc * (inv[m] * fmaf(65536.f, e2, fmaf(256.f, e1, e0)));
      }
    }
  }
};

// ---------------------------------------------------------------- ActW4A8
// W4A8 ("MIT 6.5940 Lab 4 + Lab 5", "The five implementation files and
// grading"): the activations are int8 codes with one fp32 multiplier per row
// of X and group of channels. A lane's 32 codes of each row sit in eight
// words permuted into the byte order of the masked code words (lo: channels
// 8c + 0, 4, 1, 5, the low nibbles of a word's bytes; hi: 8c + 2, 6, 3, 7),
// so dp4a multiplies four weights by four codes at once and the lane's dot
// product is an exact integer. The zero point leaves zero * (sum of the
// lane's codes), an integer too; the lane then scales by step / multiplier
// in fp32 (its 32 channels lie in one weight group and one activation group).
__device__ __forceinline__ uint32_t prmt_b32(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

template <int M, int CPL>
struct ActW4A8 {
  static_assert(CPL == 1, "W4A8 rows: 32 channels per lane");
  static constexpr bool kGroupFirst = false;  // step / multiplier applied per lane
  uint32_t lo[M][4], hi[M][4];
  int xs[M];    // sum of the lane's codes
  float rm[M];  // 1 / multiplier of the lane's activation group

  template <int LPG>
  __device__ __forceinline__ void load(const RowsArgs& a, int k0, bool active) {
    const int gsz = 32 * LPG;  // group size
#pragma unroll
    for (int m = 0; m < M; ++m) {
      uint4 v0 = make_uint4(0, 0, 0, 0), v1 = v0;
      float mu = 1.0f;
      if (active && m < a.Mv) {
        const uint4* src = reinterpret_cast<const uint4*>(a.Xq + (size_t)m * a.K + k0);
        v0 = src[0];
        v1 = src[1];
        mu = a.mult[(size_t)m * (a.K / gsz) + k0 / gsz];
      }
      const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
      int sum = 0;
#pragma unroll
      for (int c = 0; c < 4; ++c) {  // channels 8c .. 8c + 7: w[2c] = codes 0..3, w[2c + 1] = codes 4..7
        lo[m][c] = prmt_b32(w[2 * c], w[2 * c + 1], 0x5140u);  // codes 0 4 1 5
        hi[m][c] = prmt_b32(w[2 * c], w[2 * c + 1], 0x7362u);  // codes 2 6 3 7
        sum = __dp4a((int)w[2 * c], 0x01010101, sum);
        sum = __dp4a((int)w[2 * c + 1], 0x01010101, sum);
      }
      xs[m] = sum;
      rm[m] = 1.0f / mu;
    }
  }

  __device__ __forceinline__ float epilogue(int, float t, __half, __half) const { return t; }

  template <int R, int RL>
  __device__ __forceinline__ void compute(const RowsStage<R, 4 * CPL, RL>& s, float (&acc)[R * M]) const {
    static_assert(RL == R, "the W4A8 path applies every row's step per lane");
    int d[R][M];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int m = 0; m < M; ++m) d[r][m] = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const uint32_t w = s.w[r][j];
        const uint32_t ql = w & 0x0F0F0F0Fu;         // q of channels 0, 4, 1, 5
        const uint32_t qh = (w >> 4) & 0x0F0F0F0Fu;  // q of channels 2, 6, 3, 7
#pragma unroll
        for (int m = 0; m < M; ++m) {
          d[r][m] = dp4a_us(ql, lo[m][j], d[r][m]);
          d[r][m] = dp4a_us(qh, hi[m][j], d[r][m]);
        }
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int z = __half2int_rn(s.zh[r]);
      const float sc = __half2float(s.sc[r]);
#pragma unroll
      for (int m = 0; m < M; ++m) acc[r * M + m] = (float)(d[r][m] - z * xs[m]) * (sc * rm[m]);
    }
  }
};

// Sum over the 32 lanes of v[idx] for every idx: afterwards lanes whose low
// (5 - log2 NV) bits are zero hold one total each, for value `index`.
template <int NV>
__device__ __forceinline__ float butterfly_reduce(float (&v)[NV], int lane, int& index) {
  index = 0;
#pragma unroll
  for (int o = 16, c = NV; c > 1; o >>= 1, c >>= 1) {
    const int half = c / 2;
    const bool upper = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float send = upper ? v[i] : v[i + half];
      const float keep = upper ? v[i + half] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
    if (upper) index += half;
  }
  float t = v[0];
#pragma unroll
  for (int o = 16 / NV; o >= 1; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
  return t;
}

// Group-first variant: the transposing halvings run over the low lane bits
// first, so after the LPG lanes of a quantization group (which share step and
// zero) have been combined, each lane holds group totals of consecutive values
// index, index + 1, ...; epi(i, t) turns value index + i's total t into its
// stepped, zero-corrected contribution; the remaining lane bits then finish
// the sum. Afterwards lane l < NV holds the total of value `index` (= l's
// bit-reversal-free position: the halvings assign it), and every lane whose
// low log2(NV) bits equal l's holds the same total.
template <int NV, int LPG>
__device__ __forceinline__ int group_first_index(int lane) {
  int index = 0, c = NV;
#pragma unroll
  for (int o = 1; o < LPG; o <<= 1) {
    if (c > 1) {
      c /= 2;
      if (lane & o) index += c;
    }
  }
  return index;
}

template <int NV, int LPG, class Epi>
__device__ __forceinline__ float group_first_reduce(float (&v)[NV], int lane, int& index, Epi epi) {
  index = 0;
  int c = NV;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    if (o == LPG) {  // the group's lanes are combined: apply step and zero
#pragma unroll
      for (int i = 0; i < NV; ++i)
        if (i < c) v[i] = epi(i, v[i]);
    }
    if (c > 1) {
      const int half = c / 2;
      const bool upper = (lane & o) != 0;
#pragma unroll
      for (int i = 0; i < NV / 2; ++i) {
        if (i < half) {
          const float send = upper ? v[i] : v[i + half];
          const float keep = upper ? v[i + half] : v[i];
          v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
      }
      if (upper) index += half;
      c = half;
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
    }
  }
  return v[0];
}

// At most 8 warps: K <= 8192 with 32 channels per lane, K <= 16384 with 64.
// MINB: minimum CTAs per SM for the register allocation: 3 (85 registers)
// for the M = 1, 32-channel, two-stage instance, 2 (128 registers) for the
// other M = 1 instances (each measured faster, more CTAs per SM), for W4A8
// with 2-4 rows of X and for the M = 2, 32-channel, two-stage offset-sum
// instance; 1 for the other M > 1 instances (a cap would spill).
template <int M, int R, int CPL, int S, int BITS, template <int, int> class Act, int MINB = 1, int GS = kGroup>
__global__ void __launch_bounds__(256, MINB)
gemv_rows_kernel(RowsArgs a) {
  constexpr int WPR = BITS * CPL;  // packed words per row and lane
  constexpr int NV = R * M;
  constexpr int LK = 32 * CPL;  // input channels per lane
  extern __shared__ __align__(16) float red[];  // [2][32 / NV][nseg][NV]
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int nseg = blockDim.x >> 5;
  const int k0 = warp * 32 * LK + lane * LK;  // this lane's first input channel
  const bool active = k0 < a.K;
  static_assert(GS >= 32 * CPL, "a lane's channels lie in one group");
  const int G = a.K / GS;
  const size_t row_words = (size_t)a.K * BITS / 32;
  const int lane_word = k0 * BITS / 32;
  const int lane_group = k0 / GS;
  const int nbatch = (a.N + R - 1) / R;
  const int my = blockIdx.x < nbatch ? (nbatch - 1 - blockIdx.x) / gridDim.x + 1 : 0;

  // Group-first reduction (step and zero applied to group totals): this lane
  // finishes the values gidx .. gidx + CG - 1 of each batch, so it loads the
  // step and zero of their RL rows only.
  constexpr bool GF = Act<M, CPL>::kGroupFirst;
  constexpr int LPG = GS / LK;  // lanes of one quantization group
  constexpr int CG = GF ? (NV / LPG > 1 ? NV / LPG : 1) : NV;
  constexpr int RL = GF ? (CG / M > 1 ? CG / M : 1) : R;
  const int gidx = GF ? group_first_index<NV, LPG>(lane) : 0;
  const int lrow0 = gidx / M;

  // S register stages: batches i+1 .. i+S-1 are in flight while batch i is
  // computed. The first S-1 are requested before the dependent-launch wait.
  RowsStage<R, WPR, RL> st[S];
  auto issue = [&](RowsStage<R, WPR, RL>& stage, int j) {  // local batch j of this CTA
    const int row0 = (blockIdx.x + j * gridDim.x) * R;
    const int left = a.N - row0;
    const size_t sg = (size_t)row0 * G + lane_group;
    rows_issue<R, WPR, RL>(stage, a.P + (size_t)row0 * row_words + lane_word, a.steps + sg, a.zeros + sg,
                           row_words, G, active ? (left < R ? left : R) : 0, lrow0);
  };
#pragma unroll
  for (int j = 0; j < S - 1; ++j)
    if (j < my) issue(st[j], j);
  asm volatile("griddepcontrol.wait;" ::: "memory");

  Act<M, CPL> act;
  act.template load<LPG>(a, k0, active);
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // Cross-warp reduction once per NB batches: each batch's per-warp totals go
  // to a slot of a double-buffered ring; after NB batches one barrier, then
  // NB*NV threads sum the warps in order and write Y.
  constexpr int NB = 32 / NV;
  float acc[NV];
  int slot = 0, half = 0, first = 0;  // first: local batch index of slot 0
  auto flush = [&](int nslots) {
    __syncthreads();
    if (threadIdx.x < nslots * NV) {
      const int sl = threadIdx.x / NV, idx = threadIdx.x % NV;
      float t = 0.f;
      for (int w = 0; w < nseg; ++w) t += red[((half * NB + sl) * nseg + w) * NV + idx];
      const int row0 = (blockIdx.x + (first + sl) * gridDim.x) * R;
      const int r = idx / M, m = idx % M;
      if (row0 + r < a.N && m < a.Mv) a.Y[(size_t)m * a.N + row0 + r] = __float2half_rn(t);
    }
    half ^= 1;
    first += nslots;
    slot = 0;
  };
  auto finish = [&](const RowsStage<R, WPR, RL>& sg) {
    int idx;
    float v;
    if constexpr (GF) {
      // value gidx + i: batch row lrow0 + i / M, activation row i % M (gidx is
      // a multiple of M), so the step and zero are this lane's row i / M
      v = group_first_reduce<NV, LPG>(acc, lane, idx, [&](int i, float t) {
        const int rr = i / M < RL ? i / M : RL - 1;  // i < NV / LPG = RL * M wherever it is called
        return act.epilogue(i % M, t, sg.sc[rr], sg.zh[rr]);
      });
    } else {
      v = butterfly_reduce<NV>(acc, lane, idx);
    }
    const bool writer = GF ? lane < NV : (lane & (32 / NV - 1)) == 0;
    if (writer) red[((half * NB + slot) * nseg + warp) * NV + idx] = v;
    if (++slot == NB) flush(NB);
  };

  for (int i = 0; i < my; i += S) {
#pragma unroll
    for (int j = 0; j < S; ++j) {
      if (i + j < my) {
        const int nx = i + j + S - 1;
        if (nx < my) issue(st[(j + S - 1) % S], nx);
        act.template compute<R, RL>(st[j], acc);
        finish(st[j]);
      }
    }
  }
  if (slot > 0) flush(slot);
}

static int rows_num_sms() {
  static int sms = 0;
  if (sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms <= 0) sms = 148;
  }
  return sms;
}


// Persistent grid, all CTAs resident; CTA c takes row batches c, c + grid, ...
//   mode 0: small problems take one CTA per row batch (most loads in flight
//           at once); larger ones give every CTA the same number of batches.
//   mode 1 (default): every resident slot gets a CTA (grid = min(batches,
//           slots)), so each SM receives batches in turn with its CTAs.
static long rows_grid(long nbatch, int occ, int mode) {
  const long slots = (long)(occ < 1 ? 1 : occ) * rows_num_sms();
  if (mode == 1 || nbatch <= 2 * slots) return nbatch < slots ? nbatch : slots;
  const long per_cta = (nbatch + slots - 1) / slots;
  return (nbatch + per_cta - 1) / per_cta;
}

template <int M, int R, int CPL, int S, int BITS, template <int, int> class Act, int GS>
static cudaError_t launch_rows(const RowsArgs& a, cudaStream_t st, bool pdl, int grid_mode) {
  const int nseg = (a.K + 1024 * CPL - 1) / (1024 * CPL);
  // W4A8 with several rows of X, and the fp32-offset-sum kernel at M = 2 with
  // 32 channels per lane and two stages: capped at 128 registers (two CTAs per
  // SM, no spills); the other M > 1 instances would spill under the cap
  constexpr bool kW4A8 = std::is_same<Act<M, CPL>, ActW4A8<M, CPL>>::value;
  constexpr bool kHalf2x32 = std::is_same<Act<M, CPL>, ActHalf<M, CPL>>::value && M == 2 && CPL == 1 && S == 2;
  constexpr int kMinB = M == 1 ? (CPL == 1 && S == 2 ? 3 : 2) : (kW4A8 || kHalf2x32) ? 2 : 1;
  auto kern = gemv_rows_kernel<M, R, CPL, S, BITS, Act, kMinB, GS>;
  const int threads = 32 * nseg;
  const size_t smem = 2 * (size_t)32 * nseg * sizeof(float);  // [2][32/NV][nseg][NV]
  int occ = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, threads, smem);
  if (e != cudaSuccess) return e;
  if (occ < 1) return cudaErrorInvalidConfiguration;
  const long nbatch = (a.N + R - 1) / R;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)rows_grid(nbatch, occ, grid_mode), 1, 1);
  cfg.blockDim = dim3(threads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

template <int M, int R, int CPL, int S, int GS>
static cudaError_t launch_rows_act(const RowsArgs& a, cudaStream_t st, bool pdl, bool act_int, int grid_mode) {
  return act_int ? launch_rows<M, R, CPL, S, 4, ActInt, GS>(a, st, pdl, grid_mode)
                 : launch_rows<M, R, CPL, S, 4, ActHalf, GS>(a, st, pdl, grid_mode);
}

// shape: rows per batch R, input channels per lane 32*CPL, register stages S
//   0 = default (see launch_gemv_rows), 1 = (4, 32, 2), 2 = (4, 64, 2), 3 = (2, 64, 2), 4 = (4, 32, 3).
// Shapes with 32 channels per lane take K <= 8192; above that shape 2 runs.
// act_int: integer digits (true) or fp16 FMA (false) for the lane's dot products.
// Groups of 32 channels take the 32-channel shapes only (a lane's channels
// must lie in one group).
template <int M, int GS>
static cudaError_t launch_rows_shape(const RowsArgs& a, cudaStream_t st, bool pdl, bool act_int, int shape,
                                     int gm) {
  if constexpr (GS == 32) {
    return shape == 4 ? launch_rows_act<M, 4, 1, 3, GS>(a, st, pdl, act_int, gm)
                      : launch_rows_act<M, 4, 1, 2, GS>(a, st, pdl, act_int, gm);
  } else {
    switch (shape) {
      case 1: return launch_rows_act<M, 4, 1, 2, GS>(a, st, pdl, act_int, gm);
      case 3: return launch_rows_act<M, 2, 2, 2, GS>(a, st, pdl, act_int, gm);
      case 4: return launch_rows_act<M, 4, 1, 3, GS>(a, st, pdl, act_int, gm);
      default: return launch_rows_act<M, 4, 2, 2, GS>(a, st, pdl, act_int, gm);
    }
  }
}

// 3-bit rows: 64 channels per lane (six words, three 8-byte loads), shape 2
// or 3, offset sums only; groups of 64 or 128 channels.
template <int M, int GS>
static cudaError_t launch_rows3(const RowsArgs& a, cudaStream_t st, bool pdl, int shape, int gm) {
  return shape == 3 ? launch_rows<M, 2, 2, 2, 3, ActHalf3, GS>(a, st, pdl, gm)
                    : launch_rows<M, 4, 2, 2, 3, ActHalf3, GS>(a, st, pdl, gm);
}

// M = 3 and 4 (4-bit, K <= 8192, fp32 offset sums) run the M = 4 instance of
// the (4, 32, 2) shape, a missing fourth row reading as zeros.
bool gemv_rows_supported(int bits, int group, int64_t M, int64_t K) {
  if (M > 2 && !(bits == 4 && M <= 4 && K <= 8192)) return false;
  if (!((bits == 4 || bits == 3) && K <= 16384)) return false;
  return group == kGroup || group == 64 || (group == 32 && bits == 4 && K <= 8192);
}

cudaError_t launch_gemv_rows(const void* X, const uint32_t* packed, const void* steps, const void* zeros, int64_t M,
                             int64_t N, int64_t K, int bits, int group, void* Y, cudaStream_t st, int shape,
                             bool act_int, int grid_mode, bool pdl) {
  RowsArgs a;
  a.X = static_cast<const __half*>(X);
  a.P = packed;
  a.steps = static_cast<const __half*>(steps);
  a.zeros = static_cast<const __half*>(zeros);
  a.Y = static_cast<__half*>(Y);
  a.N = (int)N;
  a.K = (int)K;
  a.Mv = (int)M;
  if (M > 2) {  // 4-bit, K <= 8192: (4, 32, 2) with fp32 offset sums
    if (group == 32) return launch_rows<4, 4, 1, 2, 4, ActHalf, 32>(a, st, pdl, grid_mode);
    if (group == 64) return launch_rows<4, 4, 1, 2, 4, ActHalf, 64>(a, st, pdl, grid_mode);
    return launch_rows<4, 4, 1, 2, 4, ActHalf, kGroup>(a, st, pdl, grid_mode);
  }
  if (bits == 3) {
    if (group == 64)
      return M == 1 ? launch_rows3<1, 64>(a, st, pdl, shape, grid_mode) : launch_rows3<2, 64>(a, st, pdl, shape, grid_mode);
    return M == 1 ? launch_rows3<1, kGroup>(a, st, pdl, shape, grid_mode)
                  : launch_rows3<2, kGroup>(a, st, pdl, shape, grid_mode);
  }
  // measured fastest: at M = 1, (4, 32, 2) under an 85-register cap for
  // 4096-channel rows and for 8192-channel rows of at most 2^27 weights (more
  // CTAs per SM), else (4, 64, 2) (fewer cross-warp sums per weight); at
  // M = 2, (4, 32, 2) under a 128-register cap up to 8192-channel rows
  // (8192 x 28672: 39.5 us against 41.3 with (4, 64, 2); 11008 x 4096: 9.8
  // against 12.3), else (4, 64, 2)
  if (shape == 0) {
    if (M == 1) shape = (K <= 4096 || (K <= 8192 && N * K <= (int64_t(1) << 27))) ? 1 : 2;
    else shape = K <= 8192 ? 1 : 2;
  }
  if (K > 8192 && (shape == 1 || shape == 4)) shape = 2;  // at most 8 warps
  if (group == 32)
    return M == 1 ? launch_rows_shape<1, 32>(a, st, pdl, act_int, shape, grid_mode)
                  : launch_rows_shape<2, 32>(a, st, pdl, act_int, shape, grid_mode);
  if (group == 64)
    return M == 1 ? launch_rows_shape<1, 64>(a, st, pdl, act_int, shape, grid_mode)
                  : launch_rows_shape<2, 64>(a, st, pdl, act_int, shape, grid_mode);
  return M == 1 ? launch_rows_shape<1, kGroup>(a, st, pdl, act_int, shape, grid_mode)
                : launch_rows_shape<2, kGroup>(a, st, pdl, act_int, shape, grid_mode);
}

// W4A8 rows (K <= 8192, 32 channels per lane; the (4, 32, 2) shape): X in
// chunks of up to 4 rows, a missing row reading as zeros.
cudaError_t launch_w4a8_rows(const int8_t* qx, const float* mult, const uint32_t* packed, const void* steps,
                             const void* zeros, int64_t M, int64_t N, int64_t K, int group, void* Y, cudaStream_t st,
                             bool pdl) {
  for (int64_t m0 = 0; m0 < M; m0 += 4) {
    const int mc = (int)(M - m0 < 4 ? M - m0 : 4);
    RowsArgs a;
    a.X = nullptr;
    a.Xq = qx + m0 * K;
    a.mult = mult + m0 * (K / group);
    a.P = packed;
    a.steps = static_cast<const __half*>(steps);
    a.zeros = static_cast<const __half*>(zeros);
    a.Y = static_cast<__half*>(Y) + m0 * N;
    a.N = (int)N;
    a.K = (int)K;
    a.Mv = mc;
    auto go = [&](auto gs) -> cudaError_t {
      constexpr int GS = decltype(gs)::value;
      if (mc == 1) return launch_rows<1, 4, 1, 2, 4, ActW4A8, GS>(a, st, pdl, 1);
      if (mc == 2) return launch_rows<2, 4, 1, 2, 4, ActW4A8, GS>(a, st, pdl, 1);
      return launch_rows<4, 4, 1, 2, 4, ActW4A8, GS>(a, st, pdl, 1);
    };
    cudaError_t e = group == 32   ? go(std::integral_constant<int, 32>{})
                    : group == 64 ? go(std::integral_constant<int, 64>{})
                                  : go(std::integral_constant<int, kGroup>{});
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace wq
