// S1, S2, S4: AWQ activation-aware scale search.
//
// "MIT 6.5940 Lab 4 + Lab 5", "Starting point and setup": forward hooks record
// the mean absolute value of each linear layer's input over calibration
// tokens; "Question 2": scale salient input channels by s (and the activation
// by 1/s), searching the scale with "compute scale, scale up, quantize, scale
// down" at each place of the block; the error measured is the layer output
// reconstruction error of "CMU 11-868 L19-L20", "Quantizing during training
// vs. after it" (||WX - W^X||^2).
//
// Pipeline, all on the caller's stream:
//   absmean      mu_k = sum_t |x_tk| / T        (fp64; the sum is exact)
//   candidates   s_j,k = fp16_rn(max(mu_k, 2^-14) ^ alpha_j)
//   loss (default): one launch of awq_loss_fused, a tcgen05 GEMM that builds
//                each tile of E_j = W - Q(W diag s_j) diag(s_j)^-1 in shared
//                memory (same decision code as the packer) and sums the
//                squares of D = E_j X^T in fp64: no E in global memory, one
//                partial per (alpha, row tile, 512-token chunk)
//   loss (two-kernel option, WQ_OPT_AWQ_LOSS), per batch of alphas:
//     awq_error  E_j in fp16, every linear of the group stacked row-wise
//     awq_loss   tcgen05 GEMM D = E_j X^T per 128x128 tile, epilogue sums D^2
//                in fp64 -> one partial per (alpha, tile)
//   finalize     L_j = sum of the partials, one warp per alpha in a fixed
//                order (deterministic), first argmin, s_out = s_best
#include <cstring>
#include <mutex>

#include "wq_quant_core.cuh"
#include "wq_sm100.cuh"
#include "wq_launch.h"

namespace wq {

using namespace sm100;

constexpr int kAwqMaxLinears = 8;
constexpr int kAwqMaxAlpha = 64;
constexpr size_t kAwqEBudget = size_t(1) << 30;  // bytes of E kept per alpha batch
constexpr long long kAwqSpinLimit = 4000000000LL;

// ------------------------------------------------------------------ S1
// A block owns 32 columns (one per lane); its 8 warps take every 8th row and
// the warps' sums meet in shared memory in warp order. fp16 magnitudes are
// multiples of 2^-24 below 2^16, so while T <= 2^13 every partial sum stays
// below 2^53 units of 2^-24: exact in fp64, whatever the order of the
// additions. Beyond that the fixed order keeps the result deterministic.
__global__ void __launch_bounds__(256) absmean_kernel(const __half* __restrict__ X, int T, int K,
                                                      double* __restrict__ mu) {
  __shared__ double part[8][32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int k = blockIdx.x * 32 + lane;
  double acc = 0.0;
  if (k < K) {
#pragma unroll 8
    for (int t = warp; t < T; t += 8) acc += fabs((double)__half2float(X[(size_t)t * K + k]));
  }
  part[warp][lane] = acc;
  __syncthreads();
  if (warp == 0 && k < K) {
    double v = 0.0;
#pragma unroll
    for (int w = 0; w < 8; ++w) v += part[w][lane];
    mu[k] = v / (double)T;
  }
}

// ------------------------------------------------------------------ S2
struct AlphaList {
  double v[kAwqMaxAlpha];
};

__global__ void __launch_bounds__(256) candidates_kernel(const double* __restrict__ mu, int K, AlphaList al,
                                                         int n_alpha, __half* __restrict__ S, int* err) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  const int j = blockIdx.y;
  if (k >= K || j >= n_alpha) return;
  const double m = fmax(mu[k], 6.103515625e-05);  // 2^-14
  const double p = pow(m, al.v[j]);
  const __half h = __double2half(p);
  if (!isfinite(__half2float(h))) latch_error(err, WQ_ERR_RANGE);
  S[(size_t)j * K + k] = h;
}

// ------------------------------------------------------------------ S4a: E
struct LinearSet {
  const __half* W[kAwqMaxLinears];
  int row_off[kAwqMaxLinears + 1];  // prefix sums of N_i
  int n_lin;
  int n_total;                      // row_off[n_lin]
};

// 1/x to within one ulp (x a normal fp32: the AWQ scales are at least
// (2^-14)^0.95); the products it feeds are rounded to fp16.
__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// E for one 8-channel chunk: w - deq(w * s) / s, with deq = (level - zero) *
// step exact in fp32 (the offset level minus 1.5 * 2^23 is level - zero,
// exactly); E is rounded to fp16 next, so an approximate 1/s is enough.
template <int BITS, bool SYM>
__device__ __forceinline__ uint4 chunk_errors(uint4 x, uint4 sv, const GroupQuant& gq) {
  const __half2* h = reinterpret_cast<const __half2*>(&x);
  const __half2* sh = reinterpret_cast<const __half2*>(&sv);
  uint4 out;
  uint32_t* o = reinterpret_cast<uint32_t*>(&out);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __half22float2(h[i]);
    const float2 g = __half22float2(sh[i]);
    const float l0 = __fsub_rn(group_offset_level<BITS, SYM>(__fmul_rn(f.x, g.x), gq), kRoundMagic);
    const float l1 = __fsub_rn(group_offset_level<BITS, SYM>(__fmul_rn(f.y, g.y), gq), kRoundMagic);
    const float d0 = __fmul_rn(l0, gq.sf), d1 = __fmul_rn(l1, gq.sf);
    const __half2 hv = __floats2half2_rn(f.x - d0 * rcp_approx(g.x), f.y - d1 * rcp_approx(g.y));
    o[i] = *reinterpret_cast<const uint32_t*>(&hv);
  }
  return out;
}

template <int BITS, bool SYM>
__global__ void __launch_bounds__(256)
awq_error_kernel(LinearSet ls, int K, const __half* __restrict__ S, int alpha0, int nb, __half* __restrict__ E) {
  // 4 lanes per group, 32 consecutive input channels per lane; the lane's W
  // is read once and its error rows are written for all nb alphas.
  const int sub = threadIdx.x & 3;
  const int N = ls.n_total;
  const int G = K / kGroup;
  const int64_t gidx = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 2;
  const bool valid = gidx < (int64_t)N * G;
  const int n = valid ? (int)(gidx / G) : 0;
  const int gi = valid ? (int)(gidx % G) : 0;
  const int k0 = gi * kGroup + sub * 32;
  // Which stacked linear owns row n (unrolled so the parameter arrays stay in
  // the constant bank).
  const __half* Wrow = ls.W[0];
  int roff = 0;
#pragma unroll
  for (int i = 1; i < kAwqMaxLinears; ++i)
    if (i < ls.n_lin && n >= ls.row_off[i]) {
      Wrow = ls.W[i];
      roff = ls.row_off[i];
    }
  uint4 xraw[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    xraw[c] = make_uint4(0, 0, 0, 0);
    if (valid) xraw[c] = *reinterpret_cast<const uint4*>(Wrow + (size_t)(n - roff) * K + k0 + 8 * c);
  }

  for (int b = 0; b < nb; ++b) {
    const __half* s = S + (size_t)(alpha0 + b) * K;
    uint4 sraw[4];
    float w[32];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      sraw[c] = make_uint4(0x3C003C00u, 0x3C003C00u, 0x3C003C00u, 0x3C003C00u);  // s = 1 off the end
      if (valid) sraw[c] = *reinterpret_cast<const uint4*>(s + k0 + 8 * c);
      const __half2* h = reinterpret_cast<const __half2*>(&xraw[c]);
      const __half2* sh = reinterpret_cast<const __half2*>(&sraw[c]);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __half22float2(h[i]);
        const float2 g = __half22float2(sh[i]);
        w[8 * c + 2 * i] = __fmul_rn(f.x, g.x);  // exact
        w[8 * c + 2 * i + 1] = __fmul_rn(f.y, g.y);
      }
    }
    const GroupQuant gq = group_quant_decide<BITS, SYM, 32, 4>(w);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint4 out = chunk_errors<BITS, SYM>(xraw[c], sraw[c], gq);
      if (valid) *reinterpret_cast<uint4*>(E + ((size_t)b * N + n) * K + k0 + 8 * c) = out;
    }
  }
}

// ------------------------------------------------------------------ S4b: loss GEMM
constexpr int kLossThreads = 192;
constexpr int kLossStageBytes = 2 * 128 * 64 * 2;  // A (E) + B (X) tiles, 32 KB

struct LossArgs {
  double* partial;   // [n_alpha][tiles]
  int alpha0;
  int K;
  int t_tiles, n_tiles;
  int stages;
  int* err;
};

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int c0, int c1, int c2,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
      : "memory");
}

__global__ void __launch_bounds__(kLossThreads, 1)
awq_loss_kernel(const __grid_constant__ CUtensorMap tmE, const __grid_constant__ CUtensorMap tmX, LossArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int S = a.stages;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)S * kLossStageBytes);
  uint64_t* empty = full + S;
  uint64_t* accum = empty + S;
  double* red = reinterpret_cast<double*>(accum + 1);  // [4]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(red + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tt = blockIdx.x, nt = blockIdx.y, b = blockIdx.z;
  const int KT = a.K / 64;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accum, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tensormap(&tmE);
      prefetch_tensormap(&tmX);
      int issued = 0;
      for (int kt = 0, s = 0, u = 0; kt < KT; ++kt) {  // s = kt % S, u = kt / S
        if (*abort_flag) break;
        if (u > 0 && !mbar_wait(&empty[s], (u - 1) & 1, a.err, kAwqSpinLimit)) { *abort_flag = 1; break; }
        uint8_t* st = smem + (size_t)s * kLossStageBytes;
        mbar_arrive_expect_tx(&full[s], kLossStageBytes);
        tma_load_3d(st, &tmE, kt * 64, nt * 128, b, &full[s]);
        tma_load_2d(st + kLossStageBytes / 2, &tmX, kt * 64, tt * 128, &full[s]);
        issued = kt + 1;
        if (++s == S) { s = 0; ++u; }
      }
      for (int kt = issued > S ? issued - S : 0; kt < issued; ++kt)
        mbar_wait(&full[kt % S], (kt / S) & 1, a.err, kAwqSpinLimit);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_f16_f32(128, 128);
      int committed = -1;
      for (int kt = 0, s = 0, u = 0; kt < KT; ++kt) {  // s = kt % S, u = kt / S
        if (*abort_flag) break;
        if (!mbar_wait(&full[s], u & 1, a.err, kAwqSpinLimit)) { *abort_flag = 1; break; }
        tc_fence_after();
        const uint32_t base = smem_u32(smem + (size_t)s * kLossStageBytes);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          mma_f16_ss(tmem, desc_kmajor_sw128(base + 32 * j), desc_kmajor_sw128(base + kLossStageBytes / 2 + 32 * j),
                     idesc, (kt > 0 || j > 0) ? 1u : 0u);
        mma_commit(&empty[s]);
        committed = kt;
        if (++s == S) { s = 0; ++u; }
      }
      mma_commit(accum);
      if (*abort_flag && committed >= 0)
        mbar_wait(&empty[committed % S], (committed / S) & 1, a.err, kAwqSpinLimit);
    }
  } else {
    const int q = warp & 3;
    bool done = !__any_sync(0xffffffffu, *abort_flag != 0);
    if (done) done = __all_sync(0xffffffffu, mbar_wait(accum, 0, a.err, kAwqSpinLimit));
    double acc = 0.0;
    if (done) {
      tc_fence_after();
#pragma unroll 1
      for (int c0 = 0; c0 < 128; c0 += 16) {
        uint32_t v[16];
        tmem_ld16(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)c0, v);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const double d = (double)__uint_as_float(v[i]);
          acc = fma(d, d, acc);
        }
      }
    } else {
      *abort_flag = 1;
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) red[q] = acc;
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (warp == 2 && lane == 0 && !*abort_flag) {
      const double tot = ((red[0] + red[1]) + red[2]) + red[3];
      a.partial[((size_t)(a.alpha0 + b) * a.n_tiles + nt) * a.t_tiles + tt] = tot;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// ------------------------------------------------------------------ S4, fused: E built inside the loss GEMM
// One CTA: one alpha, 128 rows of one linear (the MMA's A operand, M = 128)
// and 512 calibration tokens (B, two N = 256 halves; D fills the 512 fp32
// columns of tensor memory). The error matrix never reaches global memory:
//
//   W producer (warp 0)  one quantization group of W per stage (TMA, two
//                        64-channel boxes, 128-byte swizzle), and the group's
//                        s (fp16) and -1/s (fp32) in a small ring;
//   error rows (2-5)     each thread owns one row: it copies the row's 128
//                        weights to registers (which frees the W stage),
//                        decides the group's step and zero point from w * s
//                        with the packer's decision code, and writes
//                        E = w - deq(Q(w s)) / s in fp16 into a ring of
//                        64-channel slots, in the swizzled K-major layout the
//                        MMA reads; then the epilogue (sum of D^2 in fp64);
//   MMA (warp 1)         owns tensor memory; per 64-channel slot, 4 K steps x
//                        2 token halves of tcgen05.mma;
//   X producer (warp 6)  64 channels x 512 tokens of X per stage (TMA).
//
// The three producers run independently, so W is fetched a group ahead of
// the error rows, and the error rows run up to two groups ahead of the MMA.
// (A variant that also multiplied E - fp16(E) into the same accumulator,
// for about 22 significant bits of E, measured no closer to the fp64 losses:
// at K >= 4096 the accumulator's own rounding toward zero, about -1e-5 of
// the loss, dominates, and the second product doubled it.)
constexpr int kFusedThreads = 224;
constexpr int kFusedTokens = 512;                       // tokens per CTA = TMEM columns
constexpr int kFusedXStages = 2;
constexpr int kFusedESlots = 4;                         // 64-channel E slots (two groups)
constexpr int kFusedSSlots = 2;
constexpr int kFusedXStage = kFusedTokens * 64 * 2;     // 64 KB
constexpr int kFusedESlot = 128 * 64 * 2;               // 16 KB
constexpr int kFusedWStage = 128 * kGroup * 2;          // 32 KB (two 16 KB boxes)
constexpr int kFusedSSlot = kGroup * 2 + kGroup * 4;    // s as fp16, then -1/s as fp32
constexpr int kFusedEOff = kFusedXStages * kFusedXStage;
constexpr int kFusedWOff = kFusedEOff + kFusedESlots * kFusedESlot;
constexpr int kFusedSOff = kFusedWOff + kFusedWStage;
constexpr int kFusedBarOff = kFusedSOff + kFusedSSlots * kFusedSSlot;
// x_full[2], x_empty[2], w_full, w_empty, e_full[4], e_empty[4], accum
constexpr int kFusedBars = 2 * kFusedXStages + 2 + 2 * kFusedESlots + 1;
constexpr int kFusedSmem = kFusedBarOff + kFusedBars * 8 + 4 * 8 + 16;
constexpr size_t kFusedSmemLaunch = 1024 + (size_t)kFusedSmem;  // + alignment slack
static_assert(kFusedSmemLaunch <= 232448, "one CTA's shared memory");

struct FusedWMaps {
  CUtensorMap m[kAwqMaxLinears];  // W_i as [N_i][K] fp16, box 64 x 128, 128-byte swizzle
};

struct FusedArgs {
  const __half* S;                    // [n_alpha][K] candidate scales
  double* partial;                    // [n_alpha][tiles][t_chunks]
  int K;
  int n_alpha;
  int tiles;                          // tile_off[n_lin]
  int t_chunks;                       // ceil(T / 512)
  int tile_off[kAwqMaxLinears + 1];   // prefix sums of ceil(N_i / 128)
  int n_lin;
  int* err;
};

template <int BITS, bool SYM>
__global__ void __launch_bounds__(kFusedThreads, 1)
awq_loss_fused_kernel(const __grid_constant__ FusedWMaps wm, const __grid_constant__ CUtensorMap tmX, FusedArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* x_full = reinterpret_cast<uint64_t*>(smem + kFusedBarOff);
  uint64_t* x_empty = x_full + kFusedXStages;
  uint64_t* w_full = x_empty + kFusedXStages;
  uint64_t* w_empty = w_full + 1;
  uint64_t* e_full = w_empty + 1;
  uint64_t* e_empty = e_full + kFusedESlots;
  uint64_t* accum = e_empty + kFusedESlots;
  double* red = reinterpret_cast<double*>(accum + 1);  // [4]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(red + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int alpha = (int)(blockIdx.x % (unsigned)a.n_alpha);
  const int tile = (int)(blockIdx.x / (unsigned)a.n_alpha);
  const int tc = blockIdx.y;
  const int G = a.K / kGroup;
  const int KT = 2 * G;  // 64-channel slots
  // The linear that owns the tile, and the tile's first row within it (the
  // loop is unrolled so the parameter arrays are never indexed at run time).
  int lin = 0, toff = 0;
#pragma unroll
  for (int i = 1; i < kAwqMaxLinears; ++i)
    if (i < a.n_lin && tile >= a.tile_off[i]) {
      lin = i;
      toff = a.tile_off[i];
    }
  const int row0 = (tile - toff) * 128;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kFusedXStages; ++s) {
      mbar_init(&x_full[s], 1);
      mbar_init(&x_empty[s], 1);
    }
    mbar_init(w_full, 1 + 32);  // the TMA's expect_tx arrival + one per producer lane (s ring)
    mbar_init(w_empty, 128);    // every error row has copied its weights
    for (int s = 0; s < kFusedESlots; ++s) {
      mbar_init(&e_full[s], 128);
      mbar_init(&e_empty[s], 1);
    }
    mbar_init(accum, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kFusedTokens);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------------- W producer
    const CUtensorMap* wmap = &wm.m[lin];
    const __half* s = a.S + (size_t)alpha * a.K;
    if (lane == 0) prefetch_tensormap(wmap);
    int issued = 0;
    for (int g = 0; g < G; ++g) {
      // The stage is free once every error row has copied group g - 1; by then
      // they are also done with the s slot of group g - 2.
      bool w = true;
      if (lane == 0 && g > 0) w = !*abort_flag && mbar_wait(w_empty, (g - 1) & 1, a.err, kAwqSpinLimit);
      if (__shfl_sync(0xffffffffu, w ? 1 : 0, 0) == 0) {
        if (lane == 0) *abort_flag = 1;
        break;
      }
      if (lane == 0) {
        uint8_t* wdst = smem + kFusedWOff;
        mbar_arrive_expect_tx(w_full, kFusedWStage);
        tma_load_2d(wdst, wmap, g * kGroup, row0, w_full);
        tma_load_2d(wdst + kFusedWStage / 2, wmap, g * kGroup + 64, row0, w_full);
      }
      issued = g + 1;
      uint8_t* slot = smem + kFusedSOff + (g % kFusedSSlots) * kFusedSSlot;
      __half* sh = reinterpret_cast<__half*>(slot);
      float* rs = reinterpret_cast<float*>(slot + kGroup * 2);
#pragma unroll
      for (int i = 0; i < kGroup / 32; ++i) {
        const int c = lane + 32 * i;
        const __half v = s[g * kGroup + c];
        sh[c] = v;
        rs[c] = -rcp_refined(__half2float(v));  // within 2^-24 (1 + 2^-19): no bias in E
      }
      mbar_arrive(w_full);  // this lane's s values are in place
    }
    // The last load must land before the CTA may exit.
    if (lane == 0 && issued > 0) mbar_wait(w_full, (issued - 1) & 1, a.err, kAwqSpinLimit);
  } else if (warp == 6) {
    // ---------------------------------------------------------------- X producer
    if (lane == 0) {
      prefetch_tensormap(&tmX);
      const int t0 = tc * kFusedTokens;
      int issued = 0;
      for (int kt = 0; kt < KT; ++kt) {
        const int xs = kt % kFusedXStages;
        if (kt >= kFusedXStages &&
            (*abort_flag || !mbar_wait(&x_empty[xs], ((kt / kFusedXStages) - 1) & 1, a.err, kAwqSpinLimit))) {
          *abort_flag = 1;
          break;
        }
        uint8_t* xdst = smem + xs * kFusedXStage;
        mbar_arrive_expect_tx(&x_full[xs], kFusedXStage);
#pragma unroll
        for (int b = 0; b < kFusedTokens / 128; ++b)  // rows past T read as zeros
          tma_load_2d(xdst + b * (128 * 64 * 2), &tmX, kt * 64, t0 + 128 * b, &x_full[xs]);
        issued = kt + 1;
      }
      for (int kt = issued > kFusedXStages ? issued - kFusedXStages : 0; kt < issued; ++kt)
        mbar_wait(&x_full[kt % kFusedXStages], (kt / kFusedXStages) & 1, a.err, kAwqSpinLimit);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      const uint32_t idesc = idesc_f16_f32(128, 256);
      bool ok = true;
      for (int kt = 0; kt < KT; ++kt) {
        const int es = kt % kFusedESlots, xs = kt % kFusedXStages;
        if (*abort_flag || !mbar_wait(&e_full[es], (kt / kFusedESlots) & 1, a.err, kAwqSpinLimit) ||
            !mbar_wait(&x_full[xs], (kt / kFusedXStages) & 1, a.err, kAwqSpinLimit)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t abase = smem_u32(smem + kFusedEOff + es * kFusedESlot);
        const uint32_t bbase = smem_u32(smem + xs * kFusedXStage);
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
          for (int n = 0; n < 2; ++n)
            mma_f16_ss(tmem + 256u * n, desc_kmajor_sw128(abase + 32 * j),
                       desc_kmajor_sw128(bbase + n * (kFusedXStage / 2) + 32 * j), idesc,
                       (kt > 0 || j > 0) ? 1u : 0u);
        mma_commit(&x_empty[xs]);
        mma_commit(&e_empty[es]);
      }
      mma_commit(accum);
      if (!ok) {
        *abort_flag = 1;
        mbar_wait(accum, 0, a.err, kAwqSpinLimit);  // no MMA of ours still reads shared memory
      }
    }
  } else {
    // ---------------------------------------------------------------- error rows
    const uint32_t r = threadIdx.x - 64;  // the E row (A row, TMEM lane) this thread builds
    for (int g = 0; g < G; ++g) {
      if (*abort_flag || !mbar_wait(w_full, g & 1, a.err, kAwqSpinLimit)) {
        *abort_flag = 1;
        break;
      }
      uint4 wr[16];  // the row's 128 weights, channel order
#pragma unroll
      for (int c = 0; c < 16; ++c)
        wr[c] = *reinterpret_cast<const uint4*>(smem + kFusedWOff + (c >> 3) * (kFusedWStage / 2) +
                                                sw128_offset(r, (uint32_t)(c & 7)));
      mbar_arrive(w_empty);  // the W stage may be refilled
      const uint8_t* slot = smem + kFusedSOff + (g % kFusedSSlots) * kFusedSSlot;
      const uint4* sh = reinterpret_cast<const uint4*>(slot);                 // 8 scales per uint4
      const float4* rs = reinterpret_cast<const float4*>(slot + kGroup * 2);  // 4 of -1/s per float4

      // The group's range of w * s (exact fp16 x fp16 products in fp32).
      float lo = 0.0f, hi = 0.0f;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const uint4 sv = sh[c];
        const uint32_t* wv = &wr[c].x;
        const uint32_t* svv = &sv.x;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float p0 = 0.0f, p1 = 0.0f;
          fma2_f16_f32(p0, p1, wv[i], svv[i]);
          if (c == 0 && i == 0) {
            lo = p0;
            hi = SYM ? fabsf(p0) : p0;
          } else if (SYM) {
            hi = max_nan(hi, fabsf(p0));
          } else {
            lo = min_nan(lo, p0);
            hi = max_nan(hi, p0);
          }
          if (SYM) {
            hi = max_nan(hi, fabsf(p1));
          } else {
            lo = min_nan(lo, p1);
            hi = max_nan(hi, p1);
          }
        }
      }
      const GroupQuant gq = group_quant_from_range<BITS, SYM>(lo, hi);
      // The error pass on pairs of channels. Per channel it is the sequence of
      // the packer's group_offset_level (Markstein-corrected quotient, plus
      // 1.5 * 2^23, clamp) and then deq = (level - 1.5 * 2^23) * step, formed
      // as one fma with -1.5 * 2^23 * step (exact: the product has 13
      // significant bits and the result at most 15), and e = w + deq * (-1/s).
      const uint64_t rcp2 = f2_pack(gq.rcp, gq.rcp);
      const uint64_t nsf2 = f2_pack(-gq.sf, -gq.sf);
      const uint64_t sf2 = f2_pack(gq.sf, gq.sf);
      const uint64_t magic2 = f2_pack(kRoundMagic, kRoundMagic);
      const float nms = __fmul_rn(-kRoundMagic, gq.sf);
      const uint64_t nms2 = f2_pack(nms, nms);

      // E, one 64-channel slot at a time.
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int kt = 2 * g + h, es = kt % kFusedESlots;
        if (kt >= kFusedESlots &&
            (*abort_flag || !mbar_wait(&e_empty[es], ((kt / kFusedESlots) - 1) & 1, a.err, kAwqSpinLimit))) {
          *abort_flag = 1;
          break;
        }
        uint8_t* eslot = smem + kFusedEOff + es * kFusedESlot;
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
          const int c = 8 * h + c8;
          const uint4 sv = sh[c];
          const float4 r0 = rs[2 * c], r1 = rs[2 * c + 1];
          const float rv[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
          const uint32_t* wv = &wr[c].x;
          const uint32_t* svv = &sv.x;
          uint4 out;
          uint32_t* o = &out.x;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            float p0 = 0.0f, p1 = 0.0f;
            fma2_f16_f32(p0, p1, wv[i], svv[i]);  // w * s, exact
            const uint64_t ws2 = f2_pack(p0, p1);
            const uint64_t q0 = f2_mul(ws2, rcp2);
            const uint64_t rr = f2_fma(q0, nsf2, ws2);          // ws - q0 * step, exact
            uint64_t lv = f2_add(f2_fma(rr, rcp2, q0), magic2);  // rounded quotient + 1.5 * 2^23
            if (!SYM) {
              const float2 l = f2_unpack(lv);
              lv = f2_pack(fminf(l.x, gq.hi_b), fminf(l.y, gq.hi_b));
            }
            const uint64_t deq = f2_fma(lv, sf2, nms2);          // (level - zero) * step, exact
            const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&wv[i]));
            const float2 e = f2_unpack(f2_fma(deq, f2_pack(rv[2 * i], rv[2 * i + 1]), f2_pack(f.x, f.y)));
            const __half2 eh = __floats2half2_rn(e.x, e.y);
            o[i] = *reinterpret_cast<const uint32_t*>(&eh);
          }
          *reinterpret_cast<uint4*>(eslot + sw128_offset(r, (uint32_t)c8)) = out;
        }
        fence_proxy_async_smem();  // these generic writes -> the MMA's async-proxy reads
        mbar_arrive(&e_full[es]);
      }
      if (*abort_flag) break;
    }

    // ---------------------------------------------------------------- epilogue
    const int q = warp & 3;  // this warp's TMEM lane quarter
    bool done = !__any_sync(0xffffffffu, *abort_flag != 0);
    if (done) done = __all_sync(0xffffffffu, mbar_wait(accum, 0, a.err, kAwqSpinLimit));
    double acc = 0.0;
    if (done) {
      tc_fence_after();
#pragma unroll 1
      for (int c0 = 0; c0 < kFusedTokens; c0 += 16) {
        uint32_t v[16];
        tmem_ld16(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)c0, v);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const double d = (double)__uint_as_float(v[i]);
          acc = fma(d, d, acc);
        }
      }
    } else {
      *abort_flag = 1;
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) red[q] = acc;
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (warp == 2 && lane == 0 && !*abort_flag) {
      const double tot = ((red[0] + red[1]) + red[2]) + red[3];
      a.partial[((size_t)alpha * a.tiles + tile) * a.t_chunks + tc] = tot;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kFusedTokens);
  }
}

// ------------------------------------------------------------------ finalize
// One warp per alpha: lane l sums tiles l, l + 32, ... in that order, then a
// fixed butterfly; the sums are deterministic.
__global__ void __launch_bounds__(256)
awq_finalize_kernel(const double* __restrict__ partial, int tiles, int n_alpha, const __half* __restrict__ S, int K,
                    double* loss_out, int32_t* best_out, __half* __restrict__ s_out, int* err) {
  __shared__ double loss[kAwqMaxAlpha];
  __shared__ int best;
  const int t = threadIdx.x;
  const int lane = t & 31, warp = t >> 5;
  for (int j = warp; j < n_alpha; j += blockDim.x >> 5) {
    double v = 0.0;
    for (int i = lane; i < tiles; i += 32) v += partial[(size_t)j * tiles + i];
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) {
      loss[j] = v;
      if (loss_out) loss_out[j] = v;
    }
  }
  __syncthreads();
  if (t == 0) {
    int bi = 0;
    bool bad = !isfinite(loss[0]);
    for (int j = 1; j < n_alpha; ++j) {
      if (!isfinite(loss[j])) bad = true;
      if (loss[j] < loss[bi]) bi = j;
    }
    if (bad) latch_error(err, WQ_ERR_RANGE);
    best = bi;
    if (best_out) *best_out = bi;
  }
  __syncthreads();
  for (int k = t; k < K; k += blockDim.x) s_out[k] = S[(size_t)best * K + k];
}

// ------------------------------------------------------------------ host
typedef CUresult (*EncodeTiledFnA)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFnA awq_encode_fn() {
  static EncodeTiledFnA fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFnA>(p);
  }
  return fn;
}

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Workspace layout: mu, the candidate scales, the partial losses, and (two-
// kernel path only) the error matrices of one batch of alphas.
AwqPlan plan_awq(int64_t T, int64_t K, const int64_t* N_i, int n_lin, int n_alpha, bool fused) {
  AwqPlan p;
  p.N_total = 0;
  for (int i = 0; i < n_lin; ++i) p.N_total += N_i[i];
  p.t_tiles = (int)((T + 127) / 128);
  p.n_tiles = (int)((p.N_total + 127) / 128);
  p.tiles = p.t_tiles * p.n_tiles;
  p.fused_tiles = 0;
  for (int i = 0; i < n_lin; ++i) p.fused_tiles += (int)((N_i[i] + 127) / 128);
  p.t_chunks = (int)((T + kFusedTokens - 1) / kFusedTokens);
  const size_t partials = (size_t)n_alpha * (size_t)(p.tiles > p.fused_tiles * p.t_chunks ? p.tiles
                                                                                        : p.fused_tiles * p.t_chunks);
  const size_t e_one = (size_t)p.N_total * (size_t)K * 2;
  int b = (int)(kAwqEBudget / (e_one ? e_one : 1));
  if (b < 1) b = 1;
  if (b > n_alpha) b = n_alpha;
  p.batch = b;
  size_t off = 0;
  p.off_mu = off;
  off = align256(off + (size_t)K * 8);
  p.off_S = off;
  off = align256(off + (size_t)n_alpha * K * 2);
  p.off_partial = off;
  off = align256(off + partials * 8);
  p.off_E = off;
  if (!fused) off = align256(off + (size_t)p.batch * e_one);
  p.total = off;
  return p;
}

// The loss of every alpha by the fused kernel: one launch over
// (alpha, row tile of one linear) x 512-token chunks, then the finalize.
template <int BITS, bool SYM>
static cudaError_t launch_fused_loss(EncodeTiledFnA enc, const CUtensorMap& tmX, const AwqPlan& p, int64_t K,
                                     const void* const* W, const int64_t* N_i, int n_lin, const __half* S,
                                     int n_alpha, double* partial, int* err, cudaStream_t st) {
  FusedWMaps wm;
  memset(&wm, 0, sizeof(wm));
  FusedArgs fa;
  fa.S = S;
  fa.partial = partial;
  fa.K = (int)K;
  fa.n_alpha = n_alpha;
  fa.t_chunks = p.t_chunks;
  fa.n_lin = n_lin;
  fa.err = err;
  fa.tile_off[0] = 0;
  for (int i = 0; i < kAwqMaxLinears; ++i) {
    if (i < n_lin) {
      cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)N_i[i]};
      cuuint64_t strides[1] = {(cuuint64_t)K * 2};
      cuuint32_t box[2] = {64, 128};
      cuuint32_t es[2] = {1, 1};
      if (enc(&wm.m[i], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(W[i]), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
      fa.tile_off[i + 1] = fa.tile_off[i] + (int)((N_i[i] + 127) / 128);
    } else {
      fa.tile_off[i + 1] = fa.tile_off[i];
    }
  }
  fa.tiles = fa.tile_off[n_lin];
  if ((int64_t)fa.tiles * n_alpha > (int64_t)INT32_MAX || p.t_chunks > 65535) return cudaErrorInvalidConfiguration;
  cudaError_t e = cudaFuncSetAttribute(awq_loss_fused_kernel<BITS, SYM>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kFusedSmemLaunch);
  if (e != cudaSuccess) return e;
  awq_loss_fused_kernel<BITS, SYM><<<dim3((unsigned)(fa.tiles * n_alpha), (unsigned)p.t_chunks), kFusedThreads,
                                     kFusedSmemLaunch, st>>>(wm, tmX, fa);
  return cudaGetLastError();
}

cudaError_t launch_awq_search(const void* X, int64_t T, int64_t K, const void* const* W, const int64_t* N_i,
                              int n_lin, int bits, bool sym, const double* alpha, int n_alpha, void* s_out,
                              double* mu_out, double* loss_out, int32_t* best_out, void* workspace, int* err,
                              bool fused, cudaStream_t st) {
  EncodeTiledFnA enc = awq_encode_fn();
  if (!enc) return cudaErrorNotSupported;
  const AwqPlan p = plan_awq(T, K, N_i, n_lin, n_alpha, fused);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  double* mu = mu_out ? mu_out : reinterpret_cast<double*>(ws + p.off_mu);
  __half* S = reinterpret_cast<__half*>(ws + p.off_S);
  double* partial = reinterpret_cast<double*>(ws + p.off_partial);
  __half* E = reinterpret_cast<__half*>(ws + p.off_E);
  const __half* Xh = static_cast<const __half*>(X);

  absmean_kernel<<<(unsigned)((K + 31) / 32), 256, 0, st>>>(Xh, (int)T, (int)K, mu);
  AlphaList al;
  for (int j = 0; j < kAwqMaxAlpha; ++j) al.v[j] = j < n_alpha ? alpha[j] : 0.0;
  candidates_kernel<<<dim3((unsigned)((K + 255) / 256), (unsigned)n_alpha), 256, 0, st>>>(mu, (int)K, al, n_alpha,
                                                                                         S, err);
  LinearSet ls;
  ls.n_lin = n_lin;
  ls.row_off[0] = 0;
  for (int i = 0; i < kAwqMaxLinears; ++i) {
    ls.W[i] = i < n_lin ? static_cast<const __half*>(W[i]) : nullptr;
    if (i < n_lin) ls.row_off[i + 1] = ls.row_off[i] + (int)N_i[i];
  }
  for (int i = n_lin; i < kAwqMaxLinears; ++i) ls.row_off[i + 1] = ls.row_off[n_lin];
  ls.n_total = ls.row_off[n_lin];

  CUtensorMap tmX;
  {
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)T};
    cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    cuuint32_t box[2] = {64, 128};
    cuuint32_t es[2] = {1, 1};
    if (enc(&tmX, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<__half*>(Xh), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  if (fused) {
    cudaError_t e;
#define WQ_FL(BI, SY) e = launch_fused_loss<BI, SY>(enc, tmX, p, K, W, N_i, n_lin, S, n_alpha, partial, err, st)
    if (bits == 4) { if (sym) WQ_FL(4, true); else WQ_FL(4, false); }
    else { if (sym) WQ_FL(3, true); else WQ_FL(3, false); }
#undef WQ_FL
    if (e != cudaSuccess) return e;
    awq_finalize_kernel<<<1, 256, 0, st>>>(partial, p.fused_tiles * p.t_chunks, n_alpha, S, (int)K, loss_out,
                                            best_out, static_cast<__half*>(s_out), err);
    return cudaGetLastError();
  }
  const int stages = 3;
  const size_t smem = 1024 + (size_t)stages * kLossStageBytes + (2 * stages + 1) * 8 + 4 * 8 + 16;
  cudaError_t e = cudaFuncSetAttribute(awq_loss_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int64_t groups = p.N_total * (K / kGroup);

  for (int a0 = 0; a0 < n_alpha; a0 += p.batch) {
    const int B = (n_alpha - a0) < p.batch ? (n_alpha - a0) : p.batch;
    const dim3 eg((unsigned)((groups + 63) / 64));  // 4 lanes per group, all B alphas per thread
#define WQ_AE(BI, SY) awq_error_kernel<BI, SY><<<eg, 256, 0, st>>>(ls, (int)K, S, a0, B, E)
    if (bits == 4) { if (sym) WQ_AE(4, true); else WQ_AE(4, false); }
    else { if (sym) WQ_AE(3, true); else WQ_AE(3, false); }
#undef WQ_AE
    CUtensorMap tmE;
    {
      cuuint64_t dims[3] = {(cuuint64_t)K, (cuuint64_t)p.N_total, (cuuint64_t)B};
      cuuint64_t strides[2] = {(cuuint64_t)K * 2, (cuuint64_t)p.N_total * (cuuint64_t)K * 2};
      cuuint32_t box[3] = {64, 128, 1};
      cuuint32_t es[3] = {1, 1, 1};
      if (enc(&tmE, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, E, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    }
    LossArgs la;
    la.partial = partial;
    la.alpha0 = a0;
    la.K = (int)K;
    la.t_tiles = p.t_tiles;
    la.n_tiles = p.n_tiles;
    la.stages = stages;
    la.err = err;
    awq_loss_kernel<<<dim3((unsigned)p.t_tiles, (unsigned)p.n_tiles, (unsigned)B), kLossThreads, smem, st>>>(
        tmE, tmX, la);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  awq_finalize_kernel<<<1, 256, 0, st>>>(partial, p.tiles, n_alpha, S, (int)K, loss_out, best_out,
                                          static_cast<__half*>(s_out), err);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// The same search without caller scratch (wq_awq_scale_search_noalloc).
//
// For callers that cannot allocate device memory, the scratch lives in a
// file-scope device array owned by the library. Its regions hold mu, the
// candidate scales, the per-tile partial losses and the error-matrix rows of
// one chunk; the search runs one alpha at a time and builds E in row chunks
// of at most kAwqStaticE bytes, so the array stays small for any N.
// ---------------------------------------------------------------------------

constexpr int kAwqStaticMaxK = 16384;
constexpr size_t kAwqStaticMu = size_t(kAwqStaticMaxK) * 8;                   // 128 KiB
constexpr size_t kAwqStaticS = size_t(kAwqMaxAlpha) * kAwqStaticMaxK * 2;     // 2 MiB
constexpr size_t kAwqStaticPartial = size_t(6) << 20;                          // 6 MiB
constexpr size_t kAwqStaticE = size_t(16) << 20;                               // 16 MiB
constexpr size_t kAwqStaticBytes = kAwqStaticMu + kAwqStaticS + kAwqStaticPartial + kAwqStaticE;

static __device__ __align__(256) uint8_t g_awq_static_scratch[kAwqStaticBytes];

// Device address of the array for the current device, looked up once per
// device (with that device current). nullptr on failure.
static uint8_t* awq_static_scratch() {
  static std::mutex mu;
  static uint8_t* addr[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_awq_static_scratch) != cudaSuccess) return nullptr;
    addr[dev] = static_cast<uint8_t*>(p);
  }
  return addr[dev];
}

bool awq_noalloc_fits(int64_t T, int64_t K, const int64_t* N_i, int n_lin, int n_alpha, bool fused) {
  if (K > kAwqStaticMaxK || n_alpha > kAwqMaxAlpha) return false;
  const AwqPlan p = plan_awq(T, K, N_i, n_lin, n_alpha, fused);  // tile counts only
  const int64_t tiles = fused ? (int64_t)p.fused_tiles * p.t_chunks : (int64_t)p.tiles;
  return (size_t)n_alpha * (size_t)tiles * 8 <= kAwqStaticPartial;
}

cudaError_t launch_awq_search_noalloc(const void* X, int64_t T, int64_t K, const void* const* W,
                                      const int64_t* N_i, int n_lin, int bits, bool sym, const double* alpha,
                                      int n_alpha, void* s_out, double* mu_out, double* loss_out, int32_t* best_out,
                                      int* err, bool fused, cudaStream_t st) {
  EncodeTiledFnA enc = awq_encode_fn();
  if (!enc) return cudaErrorNotSupported;
  uint8_t* ws = awq_static_scratch();
  if (!ws) return cudaErrorInvalidSymbol;
  const AwqPlan p = plan_awq(T, K, N_i, n_lin, n_alpha, fused);  // tile counts only; no memory of its own
  double* mu = mu_out ? mu_out : reinterpret_cast<double*>(ws);
  __half* S = reinterpret_cast<__half*>(ws + kAwqStaticMu);
  double* partial = reinterpret_cast<double*>(ws + kAwqStaticMu + kAwqStaticS);
  __half* E = reinterpret_cast<__half*>(ws + kAwqStaticMu + kAwqStaticS + kAwqStaticPartial);
  const __half* Xh = static_cast<const __half*>(X);

  absmean_kernel<<<(unsigned)((K + 31) / 32), 256, 0, st>>>(Xh, (int)T, (int)K, mu);
  AlphaList al;
  for (int j = 0; j < kAwqMaxAlpha; ++j) al.v[j] = j < n_alpha ? alpha[j] : 0.0;
  candidates_kernel<<<dim3((unsigned)((K + 255) / 256), (unsigned)n_alpha), 256, 0, st>>>(mu, (int)K, al, n_alpha,
                                                                                         S, err);
  CUtensorMap tmX;
  {
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)T};
    cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    cuuint32_t box[2] = {64, 128};
    cuuint32_t es[2] = {1, 1};
    if (enc(&tmX, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<__half*>(Xh), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  if (fused) {  // no error matrix: the partial losses are the only scratch
    cudaError_t e;
#define WQ_FL(BI, SY) e = launch_fused_loss<BI, SY>(enc, tmX, p, K, W, N_i, n_lin, S, n_alpha, partial, err, st)
    if (bits == 4) { if (sym) WQ_FL(4, true); else WQ_FL(4, false); }
    else { if (sym) WQ_FL(3, true); else WQ_FL(3, false); }
#undef WQ_FL
    if (e != cudaSuccess) return e;
    awq_finalize_kernel<<<1, 256, 0, st>>>(partial, p.fused_tiles * p.t_chunks, n_alpha, S, (int)K, loss_out,
                                            best_out, static_cast<__half*>(s_out), err);
    return cudaGetLastError();
  }
  const int stages = 3;
  const size_t smem = 1024 + (size_t)stages * kLossStageBytes + (2 * stages + 1) * 8 + 4 * 8 + 16;
  cudaError_t e = cudaFuncSetAttribute(awq_loss_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int64_t rows_chunk = (int64_t)(kAwqStaticE / ((size_t)K * 2)) / 128 * 128;
  int64_t off[kAwqMaxLinears + 1];
  off[0] = 0;
  for (int i = 0; i < n_lin; ++i) off[i + 1] = off[i] + N_i[i];

  for (int j = 0; j < n_alpha; ++j) {
    for (int64_t r0 = 0; r0 < p.N_total; r0 += rows_chunk) {
      const int64_t r1 = (r0 + rows_chunk) < p.N_total ? (r0 + rows_chunk) : p.N_total;
      // the stacked linears' rows [r0, r1)
      LinearSet lc = {};
      lc.row_off[0] = 0;
      int nl = 0;
      for (int i = 0; i < n_lin; ++i) {
        const int64_t lo = off[i] > r0 ? off[i] : r0;
        const int64_t hi = off[i + 1] < r1 ? off[i + 1] : r1;
        if (lo >= hi) continue;
        lc.W[nl] = static_cast<const __half*>(W[i]) + (lo - off[i]) * K;
        lc.row_off[nl + 1] = lc.row_off[nl] + (int)(hi - lo);
        ++nl;
      }
      for (int i = nl; i < kAwqMaxLinears; ++i) lc.row_off[i + 1] = lc.row_off[nl];
      lc.n_lin = nl;
      lc.n_total = (int)(r1 - r0);
      const int64_t groups = (r1 - r0) * (K / kGroup);
      const dim3 eg((unsigned)((groups + 63) / 64), 1u);
#define WQ_AE(BI, SY) awq_error_kernel<BI, SY><<<eg, 256, 0, st>>>(lc, (int)K, S, j, 1, E)
      if (bits == 4) { if (sym) WQ_AE(4, true); else WQ_AE(4, false); }
      else { if (sym) WQ_AE(3, true); else WQ_AE(3, false); }
#undef WQ_AE
      CUtensorMap tmE;
      {
        cuuint64_t dims[3] = {(cuuint64_t)K, (cuuint64_t)(r1 - r0), 1};
        cuuint64_t strides[2] = {(cuuint64_t)K * 2, (cuuint64_t)(r1 - r0) * (cuuint64_t)K * 2};
        cuuint32_t box[3] = {64, 128, 1};
        cuuint32_t es[3] = {1, 1, 1};
        if (enc(&tmE, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, E, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
          return cudaErrorInvalidValue;
      }
      // Tiles of this chunk land at their place in the full [alpha][n_tile][t_tile] array.
      LossArgs la;
      la.partial = partial + (size_t)(r0 / 128) * p.t_tiles;
      la.alpha0 = j;
      la.K = (int)K;
      la.t_tiles = p.t_tiles;
      la.n_tiles = p.n_tiles;
      la.stages = stages;
      la.err = err;
      awq_loss_kernel<<<dim3((unsigned)p.t_tiles, (unsigned)((r1 - r0 + 127) / 128), 1u), kLossThreads, smem, st>>>(
          tmE, tmX, la);
      e = cudaGetLastError();
      if (e != cudaSuccess) return e;
    }
  }
  awq_finalize_kernel<<<1, 256, 0, st>>>(partial, p.tiles, n_alpha, S, (int)K, loss_out, best_out,
                                          static_cast<__half*>(s_out), err);
  return cudaGetLastError();
}

}  // namespace wq
