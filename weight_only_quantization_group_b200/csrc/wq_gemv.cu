// S5: W4A16 / W3A16 decode GEMV for small M (1..8 rows of X per launch).
//
// Single-batch decode is a GEMV and is bound by the bytes of weight it must
// stream ("MIT 6.5940 Lab 4 + Lab 5", "Starting point and setup": the
// [1,8192]x[8192,8192] arithmetic-intensity argument; "CMU 11-868 L19-L20",
// "Back to the question: where does the speed come from?"). The kernel reads
// every packed word once, dequantizes in registers, and never materialises a
// 16-bit weight.
//
// Work split: a CTA of 8 warps owns RB = 8*R output rows and one K slice
// (split-K across the y grid dimension). Each warp owns R rows; in one step a
// lane covers LK consecutive input channels (4-bit: 32 = one 16-byte load per
// row; 3-bit: 128 = three 16-byte loads per row), so a warp streams 32*LK
// contiguous channels of each of its rows. With S > 1 slices, the S CTAs of a
// row block form a thread-block cluster and reduce their partial sums through
// distributed shared memory in slice order (deterministic, no workspace).
//
// Dequantization without a 16-bit weight: a LOP3 of a packed word with a
// 0x000F000F-style mask and 0x6400 in both lanes yields the half2 pair
// (1024 + q_a, 1024 + q_b) (or 1024 + 2^i q for a field i bits up). A mixed
// fp16 x fp16 -> fp32 FMA multiplies it by the matching activation pair: the
// product is exact in fp32, so
//     sum_k x_k (q_k - z) = sum_c A_c / 2^{i_c} - sum_c 1024 X_c / 2^{i_c} - z X
// where A_c accumulates x * (1024 + 2^{i_c} q) over the channels of field
// class c and X_c is the sum of those activations. The X sums depend only on
// X, so the prologue computes them once per CTA. The group step multiplies
// the 32-channel partial and adds into an fp32 accumulator.
#include <cooperative_groups.h>

#include "wq_common.cuh"

namespace cg = cooperative_groups;

namespace wq {

__device__ __forceinline__ __half2 u2h_bits(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }
__device__ __forceinline__ uint32_t h2u_bits(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }

template <int BITS>
struct GemvTraits;
template <>
struct GemvTraits<4> {
  static constexpr int LK = 32;     // input channels per lane per step
  static constexpr int WPL = 4;     // packed words per lane per row per step
};
template <>
struct GemvTraits<3> {
  static constexpr int LK = 128;
  static constexpr int WPL = 12;
};

template <int BITS>
struct GemvLayout {
  static constexpr int LK = GemvTraits<BITS>::LK;
  static constexpr int STEP = 32 * LK;       // channels a warp covers per step
  static constexpr int PIECES = LK / 8;      // 16-byte activation pieces per lane
  // Position (in halves) of local channel k in the lane-interleaved shared
  // copy of X: piece i of lane l in step t sits at ((t*PIECES + i)*32 + l)*8,
  // so the warp's 16-byte loads of one piece index hit 32 consecutive slots.
  __device__ __forceinline__ static int perm(int k) {
    return (((k / STEP) * PIECES + (k % LK) / 8) * 32 + (k % STEP) / LK) * 8 + (k % 8);
  }
};

struct GemvArgs {
  const __half* X;
  const uint32_t* P;
  const __half* steps;
  const __half* zeros;
  __half* Y;
  int N, K;
  int gps;        // groups per K slice
  int xs_stride;  // halves per token in the shared X copy (multiple of STEP)
};

// Class sums of one 32-channel chunk of activations (fp32, channel order).
template <int BITS>
__device__ __forceinline__ float2 chunk_corr(const __half* xs_tok, int kc) {
  using L = GemvLayout<BITS>;
  float c[3] = {0.f, 0.f, 0.f};  // 4-bit: x1, x16 ; 3-bit: x1, x8, x64
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const float v = __half2float(xs_tok[L::perm(kc + j)]);
    int cls;
    if (BITS == 4) {
      cls = ((j & 7) == 2 || (j & 7) == 3 || (j & 7) == 6 || (j & 7) == 7) ? 1 : 0;
    } else {
      const int pr = j >> 1;  // pair index in the chunk
      if (pr == 15) cls = 0;
      else {
        const int pj = pr % 5;
        cls = (pj == 0 || pj == 3) ? 0 : (pj == 1 || pj == 4) ? 1 : 2;
      }
    }
    c[cls] += v;
  }
  if (BITS == 4) return make_float2(1024.f * c[0] + 64.f * c[1], c[0] + c[1]);
  return make_float2(1024.f * c[0] + 128.f * c[1] + 16.f * c[2], c[0] + c[1] + c[2]);
}

template <int BITS, int M, int R, bool EXACT>
__global__ void __launch_bounds__(256)
gemv_kernel(GemvArgs a) {
  using L = GemvLayout<BITS>;
  constexpr int LK = L::LK;
  constexpr int STEP = L::STEP;
  constexpr int PIECES = L::PIECES;
  constexpr int CHUNKS = LK / 32;
  constexpr int WPL = GemvTraits<BITS>::WPL;
  constexpr int RB = 8 * R;

  extern __shared__ __align__(16) uint8_t smem[];
  __half* xs = reinterpret_cast<__half*>(smem);                                   // [M][xs_stride]
  float2* corr = reinterpret_cast<float2*>(smem + (size_t)M * a.xs_stride * 2);   // [M][xs_stride/32]
  float* part = reinterpret_cast<float*>(corr + (size_t)M * (a.xs_stride / 32));  // [RB][M]

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int G = a.K / kGroup;
  const int g0 = blockIdx.y * a.gps;
  const int g1 = min(G, g0 + a.gps);
  const int k0 = g0 * kGroup;
  const int Ls = (g1 - g0) * kGroup;  // slice length (channels)
  const int cstride = a.xs_stride / 32;

  // Prologue: lane-interleaved copy of X[:, k0:k0+Ls] and its class sums.
  for (int idx = tid; idx < M * (Ls / 8); idx += blockDim.x) {
    const int m = idx / (Ls / 8);
    const int k = (idx % (Ls / 8)) * 8;
    const uint4 v = *reinterpret_cast<const uint4*>(a.X + (size_t)m * a.K + k0 + k);
    *reinterpret_cast<uint4*>(xs + (size_t)m * a.xs_stride + L::perm(k)) = v;
  }
  __syncthreads();
  for (int idx = tid; !EXACT && idx < M * (Ls / 32); idx += blockDim.x) {
    const int m = idx / (Ls / 32);
    const int c = idx % (Ls / 32);
    corr[m * cstride + c] = chunk_corr<BITS>(xs + (size_t)m * a.xs_stride, c * 32);
  }
  __syncthreads();

  const int row0 = blockIdx.x * RB + warp * R;
  const size_t row_words = (size_t)a.K * BITS / 32;
  float acc[R][M];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int m = 0; m < M; ++m) acc[r][m] = 0.f;

  for (int kb = 0; kb < Ls; kb += STEP) {
    const int kl = kb + lane * LK;  // this lane's first local channel
    if (kl >= Ls) continue;
    const int kg = k0 + kl;         // global channel
    uint32_t wd[R][WPL];
    float sc[R][CHUNKS], zr[R][CHUNKS];
    __half zh[R][CHUNKS];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int row = row0 + r;
      if (row < a.N) {
        const uint32_t* src = a.P + row * row_words + (size_t)kg * BITS / 32;
#pragma unroll
        for (int v = 0; v < WPL / 4; ++v) {
          const uint4 q4 = ld_stream_v4(src + 4 * v);
          wd[r][4 * v] = q4.x; wd[r][4 * v + 1] = q4.y; wd[r][4 * v + 2] = q4.z; wd[r][4 * v + 3] = q4.w;
        }
#pragma unroll
        for (int c = 0; c < CHUNKS; ++c) {
          const size_t gidx = (size_t)row * G + (kg + 32 * c) / kGroup;
          sc[r][c] = __half2float(a.steps[gidx]);
          zh[r][c] = a.zeros[gidx];
          zr[r][c] = __half2float(zh[r][c]);
        }
      } else {
#pragma unroll
        for (int v = 0; v < WPL; ++v) wd[r][v] = 0;
#pragma unroll
        for (int c = 0; c < CHUNKS; ++c) { sc[r][c] = 0.f; zr[r][c] = 0.f; zh[r][c] = __float2half(0.f); }
      }
    }

#pragma unroll
    for (int c = 0; c < CHUNKS; ++c) {
      // Magic-number unpack of this chunk for every row (shared by all tokens).
      uint32_t p[R][16];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        if (BITS == 4) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint32_t w = wd[r][4 * c + j];
            const uint32_t w8 = w >> 8;
            p[r][4 * j + 0] = and_or(w, 0x000F000Fu, kHalf2Magic);   // k+0,k+1   x1
            p[r][4 * j + 1] = and_or(w, 0x00F000F0u, kHalf2Magic);   // k+2,k+3   x16
            p[r][4 * j + 2] = and_or(w8, 0x000F000Fu, kHalf2Magic);  // k+4,k+5   x1
            p[r][4 * j + 3] = and_or(w8, 0x00F000F0u, kHalf2Magic);  // k+6,k+7   x16
          }
        } else {
          const uint32_t* w3 = &wd[r][3 * c];
#pragma unroll
          for (int t = 0; t < 3; ++t) {
            const uint32_t w = w3[t];
            const uint32_t w9 = w >> 9;
            p[r][5 * t + 0] = and_or(w, 0x00070007u, kHalf2Magic);   // x1
            p[r][5 * t + 1] = and_or(w, 0x00380038u, kHalf2Magic);   // x8
            p[r][5 * t + 2] = and_or(w, 0x01C001C0u, kHalf2Magic);   // x64
            p[r][5 * t + 3] = and_or(w9, 0x00070007u, kHalf2Magic);  // x1
            p[r][5 * t + 4] = and_or(w9, 0x00380038u, kHalf2Magic);  // x8
          }
          uint32_t h = and_or(w3[0] >> 15, 0x00010001u, kHalf2Magic);
          h = and_or(w3[1] >> 14, 0x00020002u, h);
          p[r][15] = and_or(w3[2] >> 13, 0x00040004u, h);           // k30,k31 x1
        }
        if (EXACT) {
          // (1024 + 2^i q) / 2^i - (1024 / 2^i + z) = q - z, exact in fp16.
          const __half z = zh[r][c];
          const __half2 z1 = __half2half2(__hadd(z, __float2half(1024.f)));
          if (BITS == 4) {
            const __half2 z16 = __half2half2(__hneg(__hadd(z, __float2half(64.f))));
            const __half2 i16 = __float2half2_rn(0.0625f);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              p[r][4 * j + 0] = h2u_bits(__hsub2(u2h_bits(p[r][4 * j + 0]), z1));
              p[r][4 * j + 1] = h2u_bits(__hfma2(u2h_bits(p[r][4 * j + 1]), i16, z16));
              p[r][4 * j + 2] = h2u_bits(__hsub2(u2h_bits(p[r][4 * j + 2]), z1));
              p[r][4 * j + 3] = h2u_bits(__hfma2(u2h_bits(p[r][4 * j + 3]), i16, z16));
            }
          } else {
            const __half2 z8 = __half2half2(__hneg(__hadd(z, __float2half(128.f))));
            const __half2 z64 = __half2half2(__hneg(__hadd(z, __float2half(16.f))));
            const __half2 i8 = __float2half2_rn(0.125f), i64 = __float2half2_rn(0.015625f);
#pragma unroll
            for (int t = 0; t < 3; ++t) {
              p[r][5 * t + 0] = h2u_bits(__hsub2(u2h_bits(p[r][5 * t + 0]), z1));
              p[r][5 * t + 1] = h2u_bits(__hfma2(u2h_bits(p[r][5 * t + 1]), i8, z8));
              p[r][5 * t + 2] = h2u_bits(__hfma2(u2h_bits(p[r][5 * t + 2]), i64, z64));
              p[r][5 * t + 3] = h2u_bits(__hsub2(u2h_bits(p[r][5 * t + 3]), z1));
              p[r][5 * t + 4] = h2u_bits(__hfma2(u2h_bits(p[r][5 * t + 4]), i8, z8));
            }
            p[r][15] = h2u_bits(__hsub2(u2h_bits(p[r][15]), z1));
          }
        }
      }

#pragma unroll
      for (int m = 0; m < M; ++m) {
        const __half* xt = xs + (size_t)m * a.xs_stride;
        uint32_t xh[16];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint4 v = *reinterpret_cast<const uint4*>(
              xt + ((((kb / STEP) * PIECES + 4 * c + j) * 32) + lane) * 8);
          xh[4 * j] = v.x; xh[4 * j + 1] = v.y; xh[4 * j + 2] = v.z; xh[4 * j + 3] = v.w;
        }
        const float2 cr = EXACT ? make_float2(0.f, 0.f) : corr[m * cstride + (kl + 32 * c) / 32];
#pragma unroll
        for (int r = 0; r < R; ++r) {
          float t;
          if (EXACT) {
            // p already holds (q - z): exact products, plain fp32 sums.
            float al = 0.f, ah = 0.f, bl = 0.f, bh = 0.f;
#pragma unroll
            for (int j = 0; j < 16; j += 2) {
              fma2_f16_f32(al, ah, xh[j], p[r][j]);
              fma2_f16_f32(bl, bh, xh[j + 1], p[r][j + 1]);
            }
            acc[r][m] = fmaf(sc[r][c], (al + ah) + (bl + bh), acc[r][m]);
            continue;
          }
          if (BITS == 4) {
            float a1l = 0.f, a1h = 0.f, a2l = 0.f, a2h = 0.f;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              fma2_f16_f32(a1l, a1h, xh[4 * j + 0], p[r][4 * j + 0]);
              fma2_f16_f32(a2l, a2h, xh[4 * j + 1], p[r][4 * j + 1]);
              fma2_f16_f32(a1l, a1h, xh[4 * j + 2], p[r][4 * j + 2]);
              fma2_f16_f32(a2l, a2h, xh[4 * j + 3], p[r][4 * j + 3]);
            }
            t = (a1l + a1h) + (a2l + a2h) * 0.0625f - cr.x;
          } else {
            float a1l = 0.f, a1h = 0.f, a8l = 0.f, a8h = 0.f, a64l = 0.f, a64h = 0.f;
#pragma unroll
            for (int tt = 0; tt < 3; ++tt) {
              fma2_f16_f32(a1l, a1h, xh[5 * tt + 0], p[r][5 * tt + 0]);
              fma2_f16_f32(a8l, a8h, xh[5 * tt + 1], p[r][5 * tt + 1]);
              fma2_f16_f32(a64l, a64h, xh[5 * tt + 2], p[r][5 * tt + 2]);
              fma2_f16_f32(a1l, a1h, xh[5 * tt + 3], p[r][5 * tt + 3]);
              fma2_f16_f32(a8l, a8h, xh[5 * tt + 4], p[r][5 * tt + 4]);
            }
            fma2_f16_f32(a1l, a1h, xh[15], p[r][15]);
            t = (a1l + a1h) + (a8l + a8h) * 0.125f + (a64l + a64h) * 0.015625f - cr.x;
          }
          acc[r][m] = fmaf(sc[r][c], fmaf(-zr[r][c], cr.y, t), acc[r][m]);
        }
      }
    }
  }

  // Warp reduction of every (row, token) partial.
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int m = 0; m < M; ++m) {
      float v = acc[r][m];
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      acc[r][m] = v;
    }

  if (gridDim.y == 1) {
    if (lane == 0) {
#pragma unroll
      for (int r = 0; r < R; ++r)
        if (row0 + r < a.N)
#pragma unroll
          for (int m = 0; m < M; ++m) a.Y[(size_t)m * a.N + row0 + r] = __float2half_rn(acc[r][m]);
    }
    return;
  }

  // Split-K: partials of the S slices are summed through the cluster's
  // distributed shared memory, in slice order.
  if (lane == 0) {
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int m = 0; m < M; ++m) part[(warp * R + r) * M + m] = acc[r][m];
  }
  cg::cluster_group cl = cg::this_cluster();
  cl.sync();
  const int S = gridDim.y;
  const int rank = (int)cl.block_rank();
  const int per = (RB * M + S - 1) / S;
  if (tid < per) {
    const int idx = rank * per + tid;
    if (idx < RB * M) {
      float v = 0.f;
      for (int q = 0; q < S; ++q) v += cl.map_shared_rank(part, q)[idx];
      const int row = blockIdx.x * RB + idx / M;
      const int m = idx % M;
      if (row < a.N) a.Y[(size_t)m * a.N + row] = __float2half_rn(v);
    }
  }
  cl.sync();
}

// ---------------------------------------------------------------------------
// Host side: launch configuration.
// ---------------------------------------------------------------------------

struct GemvPlan {
  int R, S, gps, xs_stride;
  size_t smem;
};

static int num_sms_cached() {
  static int sms = 0;
  if (sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms <= 0) sms = 148;
  }
  return sms;
}

static GemvPlan plan_gemv(int bits, int M, int N, int K) {
  GemvPlan p;
  p.R = 2;
  const int RB = 8 * p.R;
  const int G = K / kGroup;
  const int step = bits == 4 ? 1024 : 4096;
  const long row_blocks = (N + RB - 1) / RB;
  const long target = 4L * num_sms_cached();
  int S = 1;
  while (S < 8 && row_blocks * S < target && (G / (2 * S)) >= 1) S *= 2;
  // Keep the shared X slice small enough for several CTAs per SM.
  const size_t per_chan = (size_t)M * 2 + (size_t)M * 8 / 32;
  while (S < 8 && (size_t)((G + S - 1) / S) * kGroup * per_chan > 64 * 1024) S *= 2;
  if (S > G) S = G;
  int gps = (G + S - 1) / S;
  S = (G + gps - 1) / gps;
  p.S = S;
  p.gps = gps;
  p.xs_stride = ((gps * kGroup + step - 1) / step) * step;
  p.smem = (size_t)M * p.xs_stride * 2 + (size_t)M * (p.xs_stride / 32) * 8 + (size_t)RB * M * 4;
  return p;
}

template <int BITS, int M>
static cudaError_t launch_gemv_m(const GemvArgs& a, const GemvPlan& p, cudaStream_t st, bool exact) {
  auto kern = exact ? gemv_kernel<BITS, M, 2, true> : gemv_kernel<BITS, M, 2, false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)p.smem);
  if (e != cudaSuccess) return e;
  const int RB = 16;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((a.N + RB - 1) / RB, p.S, 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.dynamicSmemBytes = p.smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = p.S;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = p.S > 1 ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

template <int BITS>
static cudaError_t launch_gemv_bits(const GemvArgs& a, int M, const GemvPlan& p, cudaStream_t st, bool exact) {
  switch (M) {
    case 1: return launch_gemv_m<BITS, 1>(a, p, st, exact);
    case 2: return launch_gemv_m<BITS, 2>(a, p, st, exact);
    case 3: return launch_gemv_m<BITS, 3>(a, p, st, exact);
    case 4: return launch_gemv_m<BITS, 4>(a, p, st, exact);
    case 5: return launch_gemv_m<BITS, 5>(a, p, st, exact);
    case 6: return launch_gemv_m<BITS, 6>(a, p, st, exact);
    case 7: return launch_gemv_m<BITS, 7>(a, p, st, exact);
    case 8: return launch_gemv_m<BITS, 8>(a, p, st, exact);
  }
  return cudaErrorInvalidValue;
}

// Y[M][N] for any M >= 1: slabs of up to 8 rows of X per launch.
cudaError_t launch_gemv(const void* X, const uint32_t* packed, const void* steps, const void* zeros, int64_t M,
                        int64_t N, int64_t K, int bits, void* Y, cudaStream_t st, bool exact) {
  for (int64_t m0 = 0; m0 < M; m0 += 8) {
    const int mc = (int)((M - m0) < 8 ? (M - m0) : 8);
    GemvArgs a;
    a.X = static_cast<const __half*>(X) + m0 * K;
    a.P = packed;
    a.steps = static_cast<const __half*>(steps);
    a.zeros = static_cast<const __half*>(zeros);
    a.Y = static_cast<__half*>(Y) + m0 * N;
    a.N = (int)N;
    a.K = (int)K;
    const GemvPlan p = plan_gemv(bits, mc, (int)N, (int)K);
    a.gps = p.gps;
    a.xs_stride = p.xs_stride;
    cudaError_t e = bits == 4 ? launch_gemv_bits<4>(a, mc, p, st, exact) : launch_gemv_bits<3>(a, mc, p, st, exact);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace wq
