// S5 for M <= 2 (4-bit): row-streaming decode GEMV with activations in registers.
//
// The decode GEMV streams the packed weight once ("MIT 6.5940 Lab 4 + Lab 5",
// "Starting point and setup"; "CMU 11-868 L19-L20", "where does the speed
// come from?"), so the instructions spent per weight, not the arithmetic,
// decide how close it gets to HBM bandwidth. This kernel keeps that count
// minimal:
//   * K is split across the warps of a CTA: warp w, lane l owns the LK = 32
//     or 64 consecutive input channels (w*32 + l)*LK .. +LK-1 for the whole
//     kernel. Its activations (and their class sums for the offset
//     correction) live in registers, loaded once -- no shared-memory copy of
//     X, no split-K, no clusters.
//   * A CTA streams batches of R consecutive rows (persistent over row
//     batches). Per row a lane issues LK/32 16-byte loads, and a warp reads
//     16*LK contiguous bytes. The next batch is loaded while the
//     current one is computed (two register stages); the first batch is
//     requested before the programmatic-dependent-launch wait, since only X
//     depends on the previous kernel.
//   * Dequantization: one LOP3 with 0x6400 in both fp16 lanes gives
//     (1024 + q, 1024 + q') or (1024 + 16q, 1024 + 16q'); a mixed fp16 x fp16
//     -> fp32 FMA multiplies it by the activation pair (exact products). The
//     offsets and the zero point are removed per row with the lane's
//     activation class sums, and the group step multiplies the lane's partial.
//   * Per batch the R x M partials are reduced across lanes with a butterfly
//     that halves the value count at each exchange. Across warps they are
//     summed through shared memory in warp order (deterministic), once per
//     32/(R*M) batches, so the CTA meets at a barrier only that often.
#include "wq_common.cuh"

namespace wq {

struct RowsArgs {
  const __half* X;
  const uint32_t* P;
  const __half* steps;
  const __half* zeros;
  __half* Y;
  int N, K;
};

template <int R, int CPL>
struct RowsStage {
  uint4 w[R][CPL];
  __half sc[R], zh[R];
};

template <int R, int CPL>
__device__ __forceinline__ void rows_issue(RowsStage<R, CPL>& s, const RowsArgs& a, int row0, bool active,
                                           size_t row_words, int G, int lane_word, int lane_group) {
  const uint32_t* pw = a.P + (size_t)row0 * row_words + lane_word;
  const size_t sg = (size_t)row0 * G + lane_group;
#pragma unroll
  for (int r = 0; r < R; ++r) {
    if (active && row0 + r < a.N) {
#pragma unroll
      for (int c = 0; c < CPL; ++c) s.w[r][c] = ld_stream_v4(pw + r * row_words + 4 * c);
      s.sc[r] = a.steps[sg + (size_t)r * G];
      s.zh[r] = a.zeros[sg + (size_t)r * G];
    } else {
#pragma unroll
      for (int c = 0; c < CPL; ++c) s.w[r][c] = make_uint4(0, 0, 0, 0);
      s.sc[r] = __float2half(0.f);
      s.zh[r] = __float2half(0.f);
    }
  }
}

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

template <int M, int R, int CPL>
__device__ __forceinline__ void rows_compute(const RowsStage<R, CPL>& s, float (&acc)[R * M],
                                             const uint32_t (&xh)[M][16 * CPL], const float (&c1)[M],
                                             const float (&xsum)[M]) {
#pragma unroll
  for (int r = 0; r < R; ++r) {
    float a[M][4];
#pragma unroll
    for (int m = 0; m < M; ++m) a[m][0] = a[m][1] = a[m][2] = a[m][3] = 0.f;
#pragma unroll
    for (int j = 0; j < 4 * CPL; ++j) {
      const uint4 wv = s.w[r][j >> 2];
      const uint32_t w = (j & 3) == 0 ? wv.x : (j & 3) == 1 ? wv.y : (j & 3) == 2 ? wv.z : wv.w;
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
    const float sc = __half2float(s.sc[r]);
    const float z = __half2float(s.zh[r]);
#pragma unroll
    for (int m = 0; m < M; ++m) {
      // sum_k x (q - z) = A1 + A2/16 - (1024 X1 + 64 X2) - z (X1 + X2)
      float t = fmaf(a[m][2] + a[m][3], 0.0625f, a[m][0] + a[m][1]) - c1[m];
      t = fmaf(-z, xsum[m], t);
      acc[r * M + m] = sc * t;
    }
  }
}

// K <= 16384: at most 16 warps of 32 channels per lane, or 8 of 64.
template <int M, int R, int CPL>
__global__ void __launch_bounds__(CPL == 1 ? 512 : 256)
gemv_rows_kernel(RowsArgs a) {
  constexpr int NV = R * M;
  constexpr int LK = 32 * CPL;  // input channels per lane
  extern __shared__ __align__(16) float red[];  // [2][32 / NV][nseg][NV]
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int nseg = blockDim.x >> 5;
  const int k0 = warp * 32 * LK + lane * LK;  // this lane's first input channel
  const bool active = k0 < a.K;
  const int G = a.K / kGroup;
  const size_t row_words = (size_t)a.K / 8;
  const int lane_word = k0 / 8;
  const int lane_group = k0 / kGroup;
  const int nbatch = (a.N + R - 1) / R;
  const int my = blockIdx.x < nbatch ? (nbatch - 1 - blockIdx.x) / gridDim.x + 1 : 0;

  RowsStage<R, CPL> s0, s1;
  if (my > 0) rows_issue<R, CPL>(s0, a, blockIdx.x * R, active, row_words, G, lane_word, lane_group);
  asm volatile("griddepcontrol.wait;" ::: "memory");

  // Activations of this lane's LK channels, and their class sums.
  uint32_t xh[M][16 * CPL];
  float c1[M], xsum[M];
#pragma unroll
  for (int m = 0; m < M; ++m) {
#pragma unroll
    for (int j = 0; j < 4 * CPL; ++j) {
      uint4 v = make_uint4(0, 0, 0, 0);
      if (active) v = *reinterpret_cast<const uint4*>(a.X + (size_t)m * a.K + k0 + 8 * j);
      xh[m][4 * j] = v.x; xh[m][4 * j + 1] = v.y; xh[m][4 * j + 2] = v.z; xh[m][4 * j + 3] = v.w;
    }
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
      if (row0 + r < a.N) a.Y[(size_t)m * a.N + row0 + r] = __float2half_rn(t);
    }
    half ^= 1;
    first += nslots;
    slot = 0;
  };
  auto finish = [&]() {
    int idx;
    const float v = butterfly_reduce<NV>(acc, lane, idx);
    if ((lane & (32 / NV - 1)) == 0) red[((half * NB + slot) * nseg + warp) * NV + idx] = v;
    if (++slot == NB) flush(NB);
  };

  for (int i = 0; i < my; i += 2) {
    const int b = blockIdx.x + i * gridDim.x;
    if (i + 1 < my) rows_issue<R, CPL>(s1, a, (b + gridDim.x) * R, active, row_words, G, lane_word, lane_group);
    rows_compute<M, R, CPL>(s0, acc, xh, c1, xsum);
    finish();
    if (i + 1 < my) {
      if (i + 2 < my)
        rows_issue<R, CPL>(s0, a, (b + 2 * gridDim.x) * R, active, row_words, G, lane_word, lane_group);
      rows_compute<M, R, CPL>(s1, acc, xh, c1, xsum);
      finish();
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

bool gemv_rows_supported(int bits, int64_t M, int64_t K) { return bits == 4 && M <= 2 && K <= 16384; }

template <int M, int R, int CPL>
static cudaError_t launch_rows(const RowsArgs& a, cudaStream_t st, bool pdl) {
  auto kern = gemv_rows_kernel<M, R, CPL>;
  const int nseg = (a.K + 1024 * CPL - 1) / (1024 * CPL);
  const int threads = 32 * nseg;
  const size_t smem = 2 * (size_t)32 * nseg * sizeof(float);  // [2][32/NV][nseg][NV]
  int occ = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, threads, smem);
  if (e != cudaSuccess) return e;
  if (occ < 1) occ = 1;
  // Persistent grid, all CTAs resident. Small problems take one CTA per row
  // batch (most loads in flight at once); larger ones give every CTA the same
  // number of batches.
  const long nbatch = (a.N + R - 1) / R;
  const long slots = (long)occ * rows_num_sms();
  long grid;
  if (nbatch <= 2 * slots) {
    grid = nbatch < slots ? nbatch : slots;
  } else {
    const long per_cta = (nbatch + slots - 1) / slots;
    grid = (nbatch + per_cta - 1) / per_cta;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid, 1, 1);
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

// shape: 0 = default; 1 = (R 4, 32 channels/lane); 2 = (R 4, 64); 3 = (R 8, 32); 4 = (R 2, 64).
cudaError_t launch_gemv_rows(const void* X, const uint32_t* packed, const void* steps, const void* zeros, int64_t M,
                             int64_t N, int64_t K, void* Y, cudaStream_t st, int shape, bool pdl) {
  RowsArgs a;
  a.X = static_cast<const __half*>(X);
  a.P = packed;
  a.steps = static_cast<const __half*>(steps);
  a.zeros = static_cast<const __half*>(zeros);
  a.Y = static_cast<__half*>(Y);
  a.N = (int)N;
  a.K = (int)K;
  if (shape == 0) shape = 2;
  if (M == 1) {
    switch (shape) {
      case 1: return launch_rows<1, 4, 1>(a, st, pdl);
      case 3: return launch_rows<1, 8, 1>(a, st, pdl);
      case 4: return launch_rows<1, 2, 2>(a, st, pdl);
      default: return launch_rows<1, 4, 2>(a, st, pdl);
    }
  }
  switch (shape) {
    case 1: return launch_rows<2, 4, 1>(a, st, pdl);
    case 3: return launch_rows<2, 8, 1>(a, st, pdl);
    case 4: return launch_rows<2, 2, 2>(a, st, pdl);
    default: return launch_rows<2, 4, 2>(a, st, pdl);
  }
}

}  // namespace wq
