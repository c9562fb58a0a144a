// S5': W4A16 / W3A16 decode GEMV for small M (1..8 rows of X per launch),
// the fallback behind the row-streaming kernel (wq_gemv_rows.cu): taken when
// the GEMV path runs a call that kernel does not take (K > 16384,
// WQ_GEMV_EXACT, more rows of X than its instances hold) or when forced with
// WQ_GEMV_KERNEL_TILED; groups of 128.
//
// Single-batch decode is a GEMV and is bound by the bytes of weight it must
// stream ("MIT 6.5940 Lab 4 + Lab 5", "Starting point and setup": the
// [1,8192]x[8192,8192] arithmetic-intensity argument; "CMU 11-868 L19-L20",
// "Back to the question: where does the speed come from?"). The kernel reads
// every packed word once, dequantizes in registers, and never materialises a
// 16-bit weight.
//
// Work split. A CTA of 8 warps owns row blocks of RB = 8*R output rows and one
// K slice (split-K along the y grid dimension); the grid is sized to the
// resident CTA count and each CTA walks row blocks with stride gridDim.x.
// Each warp owns R rows of a row block; in one step a lane covers LK
// consecutive input channels (4-bit: 32 = one 16-byte load per row; 3-bit:
// 128 = three 16-byte loads per row). Loads of the next step are issued
// before the current step is computed (two register stages), and the first
// step's loads are issued before the kernel waits on its predecessor in the
// stream (programmatic dependent launch): the weights never depend on the
// previous kernel, only X does. With S > 1 slices, the S CTAs of a row block
// form a thread-block cluster and reduce their partial sums through
// distributed shared memory in slice order (deterministic, no workspace).
//
// Dequantization without a 16-bit weight (two formulations, selectable):
//  OFFSET  LOP3 of a packed word with a 0x000F000F-style mask and 0x6400 in
//          both lanes yields the half2 (1024 + 2^i q_a, 1024 + 2^i q_b); a
//          mixed fp16 x fp16 -> fp32 FMA multiplies it by the activation pair
//          (exact products); the 1024 offset is removed per 32-channel chunk
//          with activation sums precomputed once per CTA.
//  EXACT   as OFFSET, but (q - zero) is formed in fp16 first (exact), so no
//          offset correction is needed.
#include <cooperative_groups.h>

#include "wq_common.cuh"
#include "wq_launch.h"

namespace cg = cooperative_groups;

namespace wq {

enum GemvVariant { kOffset = 0, kExact = 1 };

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

// Lane-interleaved shared copy of X: piece i (8 channels) of lane l in step t
// sits at ((t*PIECES + i)*32 + l)*8 elements, so the warp's 16-byte loads of
// one piece index hit 32 consecutive 16-byte slots.
template <int BITS, int VAR>
struct GemvLayout {
  static constexpr int LK = GemvTraits<BITS>::LK;
  static constexpr int STEP = 32 * LK;                   // channels a warp covers per step
  static constexpr int EPP = 8;                          // elements per 16-byte piece
  static constexpr int PIECES = LK / EPP;                // pieces per lane per step
  __device__ __forceinline__ static int perm(int k) {
    return (((k / STEP) * PIECES + (k % LK) / EPP) * 32 + (k % STEP) / LK) * EPP + (k % EPP);
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
  int xs_stride;  // elements per token in the shared X copy (multiple of STEP)
};

// Class sums of one 32-channel chunk of activations (fp32, channel order):
// returns (sum_c off_c * X_c, sum_c X_c) for the offset formulations.
template <int BITS, int VAR>
__device__ __forceinline__ float2 chunk_corr(const __half* xs_tok, int kc) {
  using L = GemvLayout<BITS, VAR>;
  float c[3] = {0.f, 0.f, 0.f};
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const float v = __half2float(xs_tok[L::perm(kc + j)]);
    int cls;
    if (BITS == 4) {
      cls = ((j & 7) == 2 || (j & 7) == 3 || (j & 7) == 6 || (j & 7) == 7) ? 1 : 0;
    } else {
      const int pr = j >> 1;
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

template <int BITS, int R>
struct GemvStage {
  static constexpr int CHUNKS = GemvTraits<BITS>::LK / 32;
  uint32_t wd[R][GemvTraits<BITS>::WPL];
  __half sc[R][CHUNKS];
  __half zh[R][CHUNKS];
};

template <int BITS, int VAR, int M, int R>
__device__ __forceinline__ void gemv_issue(GemvStage<BITS, R>& s, const GemvArgs& a, int rb, int kl, int Ls,
                                           int k0, int warp) {
  constexpr int WPL = GemvTraits<BITS>::WPL;
  constexpr int CHUNKS = GemvStage<BITS, R>::CHUNKS;
  const int G = a.K / kGroup;
  const size_t row_words = (size_t)a.K * BITS / 32;
  const int kg = k0 + kl;
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int row = rb * (8 * R) + warp * R + r;
    if (row < a.N && kl < Ls) {
      const uint32_t* src = a.P + row * row_words + (size_t)kg * BITS / 32;
#pragma unroll
      for (int v = 0; v < WPL / 4; ++v) {
        const uint4 q4 = ld_stream_v4(src + 4 * v);
        s.wd[r][4 * v] = q4.x; s.wd[r][4 * v + 1] = q4.y; s.wd[r][4 * v + 2] = q4.z; s.wd[r][4 * v + 3] = q4.w;
      }
#pragma unroll
      for (int c = 0; c < CHUNKS; ++c) {
        const size_t gidx = (size_t)row * G + (kg + 32 * c) / kGroup;
        s.sc[r][c] = a.steps[gidx];
        s.zh[r][c] = a.zeros[gidx];
      }
    } else {
#pragma unroll
      for (int v = 0; v < WPL; ++v) s.wd[r][v] = 0;
#pragma unroll
      for (int c = 0; c < CHUNKS; ++c) { s.sc[r][c] = __float2half(0.f); s.zh[r][c] = __float2half(0.f); }
    }
  }
}

// One step of one lane: its LK channels of each of its R rows, for all M
// tokens. Packed words are consumed word by word (8 channels) so that only
// one word's unpacked values per row are live at a time.
template <int BITS, int VAR, int M, int R>
__device__ __forceinline__ void gemv_compute(const GemvStage<BITS, R>& s, float (&acc)[R][M], const __half* xs,
                                             const float2* corr, int xs_stride, int cstride, int kb, int kl,
                                             int lane) {
  using L = GemvLayout<BITS, VAR>;
  constexpr int STEP = L::STEP;
  constexpr int PIECES = L::PIECES;
  constexpr int CHUNKS = GemvStage<BITS, R>::CHUNKS;
  const int pbase = (kb / STEP) * PIECES;
#pragma unroll
  for (int c = 0; c < CHUNKS; ++c) {
    // per (row, token) class accumulators: [0..1] class x1, [2..3] x16 (4-bit)
    // or x8, [4..5] x64 (3-bit); lo/hi halves kept apart for ILP
    float cs[R][M][6];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int m = 0; m < M; ++m)
#pragma unroll
        for (int i = 0; i < 6; ++i) cs[r][m][i] = 0.f;
    __half2 z1[R], z16[R], z8[R], z64[R];
    if (VAR == kExact) {
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const __half z = s.zh[r][c];
        z1[r] = __half2half2(__hadd(z, __float2half(1024.f)));
        z16[r] = __half2half2(__hneg(__hadd(z, __float2half(64.f))));
        z8[r] = __half2half2(__hneg(__hadd(z, __float2half(128.f))));
        z64[r] = __half2half2(__hneg(__hadd(z, __float2half(16.f))));
      }
    }
    const __half2 i16 = __float2half2_rn(0.0625f), i8 = __float2half2_rn(0.125f),
                  i64 = __float2half2_rn(0.015625f);
    if (BITS == 4) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {  // packed word j: channels 8j..8j+7
        uint4 xv[M];
#pragma unroll
        for (int m = 0; m < M; ++m)
          xv[m] = *reinterpret_cast<const uint4*>(xs + (size_t)m * xs_stride +
                                                  ((pbase + 4 * c + j) * 32 + lane) * 8);
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const uint32_t w = s.wd[r][4 * c + j];
          const uint32_t w8 = w >> 8;
          uint32_t p0 = and_or(w, 0x000F000Fu, kHalf2Magic);   // k+0,k+1   x1
          uint32_t p1 = and_or(w, 0x00F000F0u, kHalf2Magic);   // k+2,k+3   x16
          uint32_t p2 = and_or(w8, 0x000F000Fu, kHalf2Magic);  // k+4,k+5   x1
          uint32_t p3 = and_or(w8, 0x00F000F0u, kHalf2Magic);  // k+6,k+7   x16
          if (VAR == kExact) {
            p0 = h2u_bits(__hsub2(u2h_bits(p0), z1[r]));
            p1 = h2u_bits(__hfma2(u2h_bits(p1), i16, z16[r]));
            p2 = h2u_bits(__hsub2(u2h_bits(p2), z1[r]));
            p3 = h2u_bits(__hfma2(u2h_bits(p3), i16, z16[r]));
          }
#pragma unroll
          for (int m = 0; m < M; ++m) {
            fma2_f16_f32(cs[r][m][0], cs[r][m][1], xv[m].x, p0);
            fma2_f16_f32(cs[r][m][2], cs[r][m][3], xv[m].y, p1);
            fma2_f16_f32(cs[r][m][0], cs[r][m][1], xv[m].z, p2);
            fma2_f16_f32(cs[r][m][2], cs[r][m][3], xv[m].w, p3);
          }
        }
      }
    } else {
      // 3-bit: 16 channel pairs from 3 words; pair i <-> activation pair i
      uint32_t xh[M][16];
#pragma unroll
      for (int m = 0; m < M; ++m)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint4 v = *reinterpret_cast<const uint4*>(xs + (size_t)m * xs_stride +
                                                          ((pbase + 4 * c + j) * 32 + lane) * 8);
          xh[m][4 * j] = v.x; xh[m][4 * j + 1] = v.y; xh[m][4 * j + 2] = v.z; xh[m][4 * j + 3] = v.w;
        }
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const uint32_t* w3 = &s.wd[r][3 * c];
#pragma unroll
        for (int t = 0; t < 3; ++t) {
          const uint32_t w = w3[t];
          const uint32_t w9 = w >> 9;
          uint32_t q0 = and_or(w, 0x00070007u, kHalf2Magic);   // x1
          uint32_t q1 = and_or(w, 0x00380038u, kHalf2Magic);   // x8
          uint32_t q2 = and_or(w, 0x01C001C0u, kHalf2Magic);   // x64
          uint32_t q3 = and_or(w9, 0x00070007u, kHalf2Magic);  // x1
          uint32_t q4 = and_or(w9, 0x00380038u, kHalf2Magic);  // x8
          if (VAR == kExact) {
            q0 = h2u_bits(__hsub2(u2h_bits(q0), z1[r]));
            q1 = h2u_bits(__hfma2(u2h_bits(q1), i8, z8[r]));
            q2 = h2u_bits(__hfma2(u2h_bits(q2), i64, z64[r]));
            q3 = h2u_bits(__hsub2(u2h_bits(q3), z1[r]));
            q4 = h2u_bits(__hfma2(u2h_bits(q4), i8, z8[r]));
          }
#pragma unroll
          for (int m = 0; m < M; ++m) {
            fma2_f16_f32(cs[r][m][0], cs[r][m][1], xh[m][5 * t + 0], q0);
            fma2_f16_f32(cs[r][m][2], cs[r][m][3], xh[m][5 * t + 1], q1);
            fma2_f16_f32(cs[r][m][4], cs[r][m][5], xh[m][5 * t + 2], q2);
            fma2_f16_f32(cs[r][m][0], cs[r][m][1], xh[m][5 * t + 3], q3);
            fma2_f16_f32(cs[r][m][2], cs[r][m][3], xh[m][5 * t + 4], q4);
          }
        }
        uint32_t h = and_or(w3[0] >> 15, 0x00010001u, kHalf2Magic);
        h = and_or(w3[1] >> 14, 0x00020002u, h);
        h = and_or(w3[2] >> 13, 0x00040004u, h);                  // k30,k31 x1
        if (VAR == kExact) h = h2u_bits(__hsub2(u2h_bits(h), z1[r]));
#pragma unroll
        for (int m = 0; m < M; ++m) fma2_f16_f32(cs[r][m][0], cs[r][m][1], xh[m][15], h);
      }
    }
    // Chunk epilogue: remove the offsets, apply the group step.
#pragma unroll
    for (int m = 0; m < M; ++m) {
      const float2 cr = VAR == kExact ? make_float2(0.f, 0.f) : corr[m * cstride + (kl + 32 * c) / 32];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const float* q = cs[r][m];
        float t;
        if (VAR == kExact) {
          t = (q[0] + q[1]) + (q[2] + q[3]) + (BITS == 3 ? (q[4] + q[5]) : 0.f);
        } else if (BITS == 4) {
          t = fmaf(q[2] + q[3], 0.0625f, q[0] + q[1]) - cr.x;
          t = fmaf(-__half2float(s.zh[r][c]), cr.y, t);
        } else {
          t = (q[0] + q[1]) + (q[2] + q[3]) * 0.125f + (q[4] + q[5]) * 0.015625f - cr.x;
          t = fmaf(-__half2float(s.zh[r][c]), cr.y, t);
        }
        acc[r][m] = fmaf(__half2float(s.sc[r][c]), t, acc[r][m]);
      }
    }
  }
}

template <int BITS, int VAR, int M, int R>
__global__ void __launch_bounds__(256)
gemv_kernel(GemvArgs a) {
  using L = GemvLayout<BITS, VAR>;
  constexpr int STEP = L::STEP;
  constexpr int LK = L::LK;
  constexpr int RB = 8 * R;

  extern __shared__ __align__(16) uint8_t smem[];
  __half* xs = reinterpret_cast<__half*>(smem);                                               // [M][xs_stride]
  float2* corr = reinterpret_cast<float2*>(smem + (size_t)M * a.xs_stride * sizeof(__half));  // [M][xs_stride/32]
  float* part = reinterpret_cast<float*>(corr + (size_t)M * (a.xs_stride / 32));              // [2][RB][M]

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int G = a.K / kGroup;
  const int g0 = blockIdx.y * a.gps;
  const int g1 = min(G, g0 + a.gps);
  const int k0 = g0 * kGroup;
  const int Ls = (g1 - g0) * kGroup;  // slice length (channels)
  const int cstride = a.xs_stride / 32;
  const int nsteps = (Ls + STEP - 1) / STEP;
  const int n_rb = (a.N + RB - 1) / RB;
  const int my_rb = blockIdx.x < n_rb ? (n_rb - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  const int n_it = my_rb * nsteps;

  GemvStage<BITS, R> s0, s1;
  // (rb, st): the iteration being computed; (nrb, nst): the next one to fetch.
  int rb = blockIdx.x, st = 0;
  int nrb = rb, nst = 0;
  auto advance = [&](int& b, int& t) {
    if (++t == nsteps) {
      t = 0;
      b += gridDim.x;
    }
  };
  // The weights do not depend on the previous kernel: fetch the first step now.
  if (n_it > 0) gemv_issue<BITS, VAR, M, R>(s0, a, nrb, nst * STEP + lane * LK, Ls, k0, warp);
  advance(nrb, nst);
  asm volatile("griddepcontrol.wait;" ::: "memory");

  // Prologue: lane-interleaved copy of X[:, k0:k0+Ls] and its class sums.
  for (int idx = tid; idx < M * (Ls / 8); idx += blockDim.x) {
    const int m = idx / (Ls / 8);
    const int k = (idx % (Ls / 8)) * 8;
    const uint4 v = *reinterpret_cast<const uint4*>(a.X + (size_t)m * a.K + k0 + k);
    *reinterpret_cast<uint4*>(xs + (size_t)m * a.xs_stride + L::perm(k)) = v;
  }
  __syncthreads();
  for (int idx = tid; VAR != kExact && idx < M * (Ls / 32); idx += blockDim.x) {
    const int m = idx / (Ls / 32);
    const int c = idx % (Ls / 32);
    corr[m * cstride + c] = chunk_corr<BITS, VAR>(xs + (size_t)m * a.xs_stride, c * 32);
  }
  __syncthreads();
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  const bool split = gridDim.y > 1;
  cg::cluster_group cl = cg::this_cluster();
  float acc[R][M];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int m = 0; m < M; ++m) acc[r][m] = 0.f;
  int pb = 0;

  auto finish_rb = [&](int b) {
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int m = 0; m < M; ++m) {
        float v = acc[r][m];
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        acc[r][m] = v;
      }
    if (!split) {
      if (lane == 0) {
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const int row = b * RB + warp * R + r;
          if (row < a.N)
#pragma unroll
            for (int m = 0; m < M; ++m) a.Y[(size_t)m * a.N + row] = __float2half_rn(acc[r][m]);
        }
      }
    } else {
      float* pp = part + pb * RB * M;
      if (lane == 0) {
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
          for (int m = 0; m < M; ++m) pp[(warp * R + r) * M + m] = acc[r][m];
      }
      cl.sync();
      const int S = gridDim.y;
      const int rank = (int)cl.block_rank();
      const int per = (RB * M + S - 1) / S;
      if (tid < per) {
        const int idx = rank * per + tid;
        if (idx < RB * M) {
          float v = 0.f;
          for (int q = 0; q < S; ++q) v += cl.map_shared_rank(pp, q)[idx];
          const int row = b * RB + idx / M;
          const int m = idx % M;
          if (row < a.N) a.Y[(size_t)m * a.N + row] = __float2half_rn(v);
        }
      }
      pb ^= 1;
    }
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int m = 0; m < M; ++m) acc[r][m] = 0.f;
  };

  // Two register stages: compute from one while the other is being filled.
  for (int it = 0; it < n_it; it += 2) {
    if (it + 1 < n_it) gemv_issue<BITS, VAR, M, R>(s1, a, nrb, nst * STEP + lane * LK, Ls, k0, warp);
    advance(nrb, nst);
    {
      const int kb = st * STEP, kl = kb + lane * LK;
      if (kl < Ls) gemv_compute<BITS, VAR, M, R>(s0, acc, xs, corr, a.xs_stride, cstride, kb, kl, lane);
      if (st == nsteps - 1) finish_rb(rb);
      advance(rb, st);
    }
    if (it + 1 < n_it) {
      if (it + 2 < n_it) gemv_issue<BITS, VAR, M, R>(s0, a, nrb, nst * STEP + lane * LK, Ls, k0, warp);
      advance(nrb, nst);
      const int kb = st * STEP, kl = kb + lane * LK;
      if (kl < Ls) gemv_compute<BITS, VAR, M, R>(s1, acc, xs, corr, a.xs_stride, cstride, kb, kl, lane);
      if (st == nsteps - 1) finish_rb(rb);
      advance(rb, st);
    }
  }
  if (split) cl.sync();  // keep shared memory alive until every peer has read it
}

// ---------------------------------------------------------------------------
// Host side: launch configuration.
// ---------------------------------------------------------------------------

struct GemvPlan {
  int R, S, gps, xs_stride, grid_x;
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

// Rows per warp: enough independent 16-byte loads in flight per lane without
// exhausting registers (two register stages of R rows).
__host__ __device__ constexpr int gemv_rows_per_warp(int bits, int M) {
  return bits == 4 ? (M <= 2 ? 4 : (M <= 4 ? 2 : 1)) : (M <= 2 ? 2 : 1);
}

// regs_per_thread: of the kernel instance that will run (0 = unknown).
static GemvPlan plan_gemv(int bits, int var, int M, int N, int K, int regs_per_thread = 0) {
  GemvPlan p;
  p.R = gemv_rows_per_warp(bits, M);
  const int RB = 8 * p.R;
  const int G = K / kGroup;
  const int step = bits == 4 ? 1024 : 4096;
  const int xbytes = 2;
  (void)var;
  const long row_blocks = (N + RB - 1) / RB;
  auto smem_for = [&](int S) {
    const int gps = (G + S - 1) / S;
    const int xs = ((gps * kGroup + step - 1) / step) * step;
    return (size_t)M * xs * xbytes + (size_t)M * (xs / 32) * 8 + 2 * (size_t)RB * M * 4;
  };
  // Resident CTAs per SM, from registers and shared memory.
  auto occupancy = [&](size_t smem) {
    int occ = regs_per_thread > 0 ? 65536 / (regs_per_thread * 256) : 2;
    const int by_smem = (int)((228 * 1024) / (smem + 1024));
    if (by_smem < occ) occ = by_smem;
    return occ < 1 ? 1 : (occ > 4 ? 4 : occ);
  };
  int S = 1;
  // Split K until every SM has work (and the X slice fits a few CTAs per SM).
  while (S < 8 && (G / (2 * S)) >= 1 &&
         (row_blocks * S < (long)occupancy(smem_for(S)) * num_sms_cached() || smem_for(S) > 64 * 1024))
    S *= 2;
  if (S > G) S = G;
  const int gps = (G + S - 1) / S;
  S = (G + gps - 1) / gps;
  p.S = S;
  p.gps = gps;
  p.xs_stride = ((gps * kGroup + step - 1) / step) * step;
  p.smem = smem_for(S);
  // Persistent grid: every CTA gets the same number of row blocks and all
  // CTAs are resident at once.
  const long slots = (long)occupancy(p.smem) * num_sms_cached();
  long per_cta = (row_blocks * S + slots - 1) / slots;
  if (per_cta < 1) per_cta = 1;
  p.grid_x = (int)((row_blocks + per_cta - 1) / per_cta);
  return p;
}

template <int BITS, int VAR, int M, int R>
static int gemv_regs() {
  static int regs = 0;
  if (regs == 0) {
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, gemv_kernel<BITS, VAR, M, R>) == cudaSuccess) regs = fa.numRegs;
  }
  return regs;
}

template <int BITS, int VAR, int M, int R>
static cudaError_t launch_gemv_k(GemvArgs a, int N, int K, cudaStream_t st, bool pdl) {
  auto kern = gemv_kernel<BITS, VAR, M, R>;
  const GemvPlan p = plan_gemv(BITS, VAR, M, N, K, gemv_regs<BITS, VAR, M, R>());
  a.gps = p.gps;
  a.xs_stride = p.xs_stride;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)p.smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.grid_x, p.S, 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.dynamicSmemBytes = p.smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (p.S > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = 1;
    attr[n].val.clusterDim.y = p.S;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr + (pdl ? 0 : 1);
  cfg.numAttrs = pdl ? n : n - 1;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

template <int BITS, int VAR, int M>
static cudaError_t launch_gemv_m(const GemvArgs& a, cudaStream_t st, bool pdl) {
  return launch_gemv_k<BITS, VAR, M, gemv_rows_per_warp(BITS, M)>(a, a.N, a.K, st, pdl);
}

template <int BITS, int VAR>
static cudaError_t launch_gemv_bits(const GemvArgs& a, int M, cudaStream_t st, bool pdl) {
  switch (M) {
    case 1: return launch_gemv_m<BITS, VAR, 1>(a, st, pdl);
    case 2: return launch_gemv_m<BITS, VAR, 2>(a, st, pdl);
    case 3: return launch_gemv_m<BITS, VAR, 3>(a, st, pdl);
    case 4: return launch_gemv_m<BITS, VAR, 4>(a, st, pdl);
    case 5: return launch_gemv_m<BITS, VAR, 5>(a, st, pdl);
    case 6: return launch_gemv_m<BITS, VAR, 6>(a, st, pdl);
    case 7: return launch_gemv_m<BITS, VAR, 7>(a, st, pdl);
    case 8: return launch_gemv_m<BITS, VAR, 8>(a, st, pdl);
  }
  return cudaErrorInvalidValue;
}

// Y[M][N] for any M >= 1: slabs of up to 8 rows of X per launch.
// variant: 0 offset sums, 1 exact.
cudaError_t launch_gemv(const void* X, const uint32_t* packed, const void* steps, const void* zeros, int64_t M,
                        int64_t N, int64_t K, int bits, void* Y, cudaStream_t st, int variant, bool pdl) {
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
    cudaError_t e;
    if (bits == 4) {
      e = variant == kExact ? launch_gemv_bits<4, kExact>(a, mc, st, pdl) : launch_gemv_bits<4, kOffset>(a, mc, st, pdl);
    } else {
      e = variant == kExact ? launch_gemv_bits<3, kExact>(a, mc, st, pdl) : launch_gemv_bits<3, kOffset>(a, mc, st, pdl);
    }
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// Upper bound of the shared memory the GEMV needs for (M slab, K); used for
// host-side validation.
size_t gemv_smem_bytes(int bits, int variant, int M, int N, int K) {
  return plan_gemv(bits, variant, M < 8 ? M : 8, N, K).smem;
}

}  // namespace wq
