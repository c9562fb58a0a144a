// GPTQ into the group-wise packed format ("CMU 11-868 L19-L20 Model
// Quantization", sections "The algorithm in four steps" and "Why it can
// actually run: from OBS to GPTQ"), in fp64 on the GPU:
//
//   1. H = 2 X^T X + lambda I (lambda = damp * mean diag H; an input channel
//      that is zero on every token gets H_kk = 1 and zero weights), then
//      G = Cholesky(H^-1)^T, the upper factor with H^-1 = G^T G. It comes
//      from one "UL" factorization H = U U^T (U upper, computed from the
//      bottom-right corner) and one triangular inverse: G = U^-1, since
//      H^-1 = U^-T U^-1 = (U^-1)^T U^-1.
//   2.-4. Column blocks of 128: per block one kernel quantizes the columns in
//      order for all rows (each thread one row: group step and zero from the
//      row's current weights when a group starts, the code, the error divided
//      by G_ii, the in-block update), then a GEMM moves every column to the
//      right by Err * G[block, right] (the lazy batch update).
//
// Rows are independent once G is known, so the column loop runs row-parallel
// with no grid-wide synchronisation; the dense steps are tiled fp64 kernels
// (64 x 64 tiles, 256 threads, 4 x 4 outputs per thread). Quantization
// decisions follow the library's quantizer on the fp32 value of each running
// weight (fp16 step rounded up, integer zero point, rint ties to even).
#include <math.h>

#include "wq_quant_core.cuh"
#include "wq_launch.h"

namespace wq {

constexpr int kTb = 64;   // dense tile
constexpr int kGb = 128;  // GPTQ column block

// ------------------------------------------------------------------ dense tiles
// C[64x64] += A[64 x kk] * B[kk x 64] for fp64 row-major operands given by
// (pointer, leading dimension), either transposed; 256 threads, each 4 x 4
// outputs; K in chunks of 32 through shared memory (sbuf: kTileBuf doubles).
constexpr int kKc = 32;
constexpr int kTileBuf = kTb * (kKc + 1) + kKc * (kTb + 1);  // 4192 doubles, 33.5 KB
struct TileAcc {
  double c[4][4];
};

__device__ __forceinline__ void tile_mma(TileAcc& acc, const double* __restrict__ A, int lda, bool a_trans,
                                         const double* __restrict__ B, int ldb, bool b_trans, int kk, double* sbuf) {
  double (*As)[kKc + 1] = reinterpret_cast<double (*)[kKc + 1]>(sbuf);                 // [64][33]: As[r][k]
  double (*Bs)[kTb + 1] = reinterpret_cast<double (*)[kTb + 1]>(sbuf + kTb * (kKc + 1));  // [32][65]: Bs[k][c]
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  for (int k0 = 0; k0 < kk; k0 += kKc) {
    const int kc = kk - k0 < kKc ? kk - k0 : kKc;
    for (int e = threadIdx.x; e < kTb * kKc; e += blockDim.x) {
      const int r = e / kKc, k = e % kKc;  // As[r][k]
      As[r][k] = k < kc ? (a_trans ? A[(size_t)(k0 + k) * lda + r] : A[(size_t)r * lda + k0 + k]) : 0.0;
      const int kb = e / kTb, c = e % kTb;  // Bs[kb][c]
      Bs[kb][c] = kb < kc ? (b_trans ? B[(size_t)c * ldb + k0 + kb] : B[(size_t)(k0 + kb) * ldb + c]) : 0.0;
    }
    __syncthreads();
#pragma unroll 4
    for (int k = 0; k < kc; ++k) {
      double a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[ty + 16 * i][k];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[k][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc.c[i][j] = fma(a[i], b[j], acc.c[i][j]);
    }
    __syncthreads();
  }
}

// ------------------------------------------------------------------ step 1: H
// H[a][b] = 2 sum_t X[t][a] X[t][b] for the upper tiles (a-tile <= b-tile),
// mirrored into the lower ones; fp16 products are exact in fp64.
__global__ void __launch_bounds__(256) gptq_hessian_kernel(const __half* __restrict__ X, int T, int K,
                                                           double* __restrict__ H) {
  const int ta = blockIdx.y, tb = blockIdx.x;
  if (ta > tb) return;
  __shared__ double Xa[32][kTb + 1], Xb[32][kTb + 1];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  double c[4][4] = {};
  for (int t0 = 0; t0 < T; t0 += 32) {
    for (int e = threadIdx.x; e < 32 * kTb; e += blockDim.x) {
      const int t = e / kTb, j = e % kTb;
      const bool in = t0 + t < T;
      const int a = ta * kTb + j, b = tb * kTb + j;
      Xa[t][j] = in && a < K ? (double)__half2float(X[(size_t)(t0 + t) * K + a]) : 0.0;
      Xb[t][j] = in && b < K ? (double)__half2float(X[(size_t)(t0 + t) * K + b]) : 0.0;
    }
    __syncthreads();
#pragma unroll 4
    for (int t = 0; t < 32; ++t) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) c[i][j] = fma(Xa[t][ty + 16 * i], Xb[t][tx + 16 * j], c[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int a = ta * kTb + ty + 16 * i, b = tb * kTb + tx + 16 * j;
      if (a < K && b < K) {
        H[(size_t)a * K + b] = 2.0 * c[i][j];
        H[(size_t)b * K + a] = 2.0 * c[i][j];
      }
    }
}

// Dead channels (H_kk == 0) -> H_kk = 1 and a flag; then lambda = damp *
// mean(diag) is added to the diagonal. One CTA (a fixed-order sum).
__global__ void __launch_bounds__(1024) gptq_damp_kernel(double* __restrict__ H, int K, double damp,
                                                         uint8_t* __restrict__ dead) {
  __shared__ double part[1024];
  double s = 0.0;
  for (int k = threadIdx.x; k < K; k += blockDim.x) {
    double d = H[(size_t)k * K + k];
    dead[k] = d == 0.0;
    if (d == 0.0) d = H[(size_t)k * K + k] = 1.0;
    s += d;
  }
  part[threadIdx.x] = s;
  __syncthreads();
  for (int o = 512; o > 0; o >>= 1) {
    if ((int)threadIdx.x < o) part[threadIdx.x] += part[threadIdx.x + o];
    __syncthreads();
  }
  const double lam = damp * part[0] / K;
  for (int k = threadIdx.x; k < K; k += blockDim.x) H[(size_t)k * K + k] += lam;
}

// ------------------------------------------------------------------ step 1: H = U U^T
// Blocked from the bottom-right: for the tile column kb (descending),
// (i) U_kk from the diagonal tile (one CTA, in shared memory), (ii) the panel
// above it, U[ib][kb] = A[ib][kb] U_kk^-T, (iii) the trailing update
// A[ib][jb] -= U[ib][kb] U[jb][kb]^T for ib <= jb < kb. A (= H, in place)
// keeps U in its upper triangle.
__global__ void __launch_bounds__(256) ul_diag_kernel(double* __restrict__ A, int K, int kb, int* err) {
  __shared__ double S[kTb][kTb + 1];
  const int base = kb * kTb, n = K - base < kTb ? K - base : kTb;
  for (int e = threadIdx.x; e < kTb * kTb; e += blockDim.x) {
    const int r = e / kTb, c = e % kTb;
    S[r][c] = r < n && c < n ? A[(size_t)(base + r) * K + base + c] : (r == c ? 1.0 : 0.0);
  }
  __syncthreads();
  // columns j = n-1 .. 0: U_jj = sqrt(S_jj), U_ij = S_ij / U_jj (i < j), then
  // S_il -= U_ij U_lj for i <= l < j (upper triangle only)
  for (int j = n - 1; j >= 0; --j) {
    if (threadIdx.x == 0) {
      const double d = S[j][j];
      if (!(d > 0.0)) latch_error(err, WQ_ERR_RANGE);  // not positive definite
      S[j][j] = sqrt(d > 0.0 ? d : 1.0);
    }
    __syncthreads();
    const double ujj = S[j][j];
    for (int i = threadIdx.x; i < j; i += blockDim.x) S[i][j] /= ujj;
    __syncthreads();
    for (int e = threadIdx.x; e < j * j; e += blockDim.x) {
      const int i = e / j, l = e % j;
      if (i <= l) S[i][l] -= S[i][j] * S[l][j];
    }
    __syncthreads();
  }
  for (int e = threadIdx.x; e < n * n; e += blockDim.x) {
    const int r = e / n, c = e % n;
    A[(size_t)(base + r) * K + base + c] = r <= c ? S[r][c] : 0.0;
  }
}

// Panel: X = A[ib][kb] solves X U_kk^T = A, i.e. for each row x of the tile,
// x_j = (a_j - sum_{l > j} x_l U_jl) / U_jj for j = n-1 .. 0 (U_kk upper).
// One CTA per tile ib < kb, one thread per row.
__global__ void __launch_bounds__(kTb) ul_panel_kernel(double* __restrict__ A, int K, int kb) {
  __shared__ double U[kTb][kTb + 1];
  const int base = kb * kTb, n = K - base < kTb ? K - base : kTb;
  const int ib = blockIdx.x;
  for (int e = threadIdx.x; e < kTb * kTb; e += blockDim.x) {
    const int r = e / kTb, c = e % kTb;
    U[r][c] = r < n && c < n ? A[(size_t)(base + r) * K + base + c] : 0.0;
  }
  __syncthreads();
  const int row = ib * kTb + threadIdx.x;
  double* x = A + (size_t)row * K + base;
  for (int j = n - 1; j >= 0; --j) {
    double v = x[j];
    for (int l = j + 1; l < n; ++l) v -= x[l] * U[j][l];
    x[j] = v / U[j][j];
  }
}

// Trailing update of the upper tiles left of the panel: A[ib][jb] -=
// P[ib] P[jb]^T with P[t] = A[t][kb] (the new panel), ib <= jb < kb.
__global__ void __launch_bounds__(256) ul_update_kernel(double* __restrict__ A, int K, int kb) {
  const int ib = blockIdx.y, jb = blockIdx.x;
  if (ib > jb) return;
  __shared__ double sbuf[kTileBuf];
  const int base = kb * kTb, n = K - base < kTb ? K - base : kTb;
  TileAcc acc = {};
  // C = P[ib] (64 x n) * P[jb]^T (n x 64)
  tile_mma(acc, A + (size_t)ib * kTb * K + base, K, false, A + (size_t)jb * kTb * K + base, K, true, n, sbuf);
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j)
      A[(size_t)(ib * kTb + ty + 16 * i) * K + jb * kTb + tx + 16 * j] -= acc.c[i][j];
}

// ------------------------------------------------------------------ step 1: G = U^-1
// Row blocks from the bottom: G[ib][ib] = U_ii^-1 (one CTA, back
// substitution), and for jb > ib: G[ib][jb] = -U_ii^-1 sum_{k=ib+1..jb}
// U[ib][k] G[k][jb]. U is read from the upper triangle of A; G (upper) is
// written into its own buffer.
__global__ void __launch_bounds__(256) trinv_diag_kernel(const double* __restrict__ A, int K, int ib,
                                                         double* __restrict__ G) {
  __shared__ double U[kTb][kTb + 1];
  const int base = ib * kTb, n = K - base < kTb ? K - base : kTb;
  for (int e = threadIdx.x; e < kTb * kTb; e += blockDim.x) {
    const int r = e / kTb, c = e % kTb;
    U[r][c] = r < n && c < n && r <= c ? A[(size_t)(base + r) * K + base + c] : (r == c ? 1.0 : 0.0);
  }
  __syncthreads();
  // column c of U^-1 by back substitution (thread c), written to G; the
  // entries below the diagonal stay 0 (G was cleared)
  if ((int)threadIdx.x < n) {
    const int c = threadIdx.x;
    double* gc = G + (size_t)base * K + base + c;  // G[base + r][base + c] = gc[r * K]
    for (int r = c; r >= 0; --r) {
      double v = r == c ? 1.0 : 0.0;
      for (int l = r + 1; l <= c; ++l) v -= U[r][l] * gc[(size_t)l * K];
      gc[(size_t)r * K] = v / U[r][r];
    }
  }
}

// The off-diagonal tiles of row block ib: one CTA per jb > ib.
__global__ void __launch_bounds__(256) trinv_row_kernel(const double* __restrict__ A, int K, int ib,
                                                        double* __restrict__ G) {
  const int jb = ib + 1 + blockIdx.x;
  __shared__ double sbuf[kTileBuf];
  const int base = ib * kTb;
  // T = U[ib][ib+1 .. jb] * G[ib+1 .. jb][jb]  (64 x span) * (span x 64)
  const int k_lo = (ib + 1) * kTb, k_hi = (jb + 1) * kTb;
  TileAcc acc = {};
  tile_mma(acc, A + (size_t)base * K + k_lo, K, false, G + (size_t)k_lo * K + jb * kTb, K, false, k_hi - k_lo, sbuf);
  // G[ib][jb] = -G_ii T with G_ii = G[ib][ib] (upper, already written)
  double (*Ts)[kTb + 1] = reinterpret_cast<double (*)[kTb + 1]>(sbuf);  // 64 x 65 <= kTileBuf
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) Ts[ty + 16 * i][tx + 16 * j] = acc.c[i][j];
  __syncthreads();
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int r = ty + 16 * i, c = tx + 16 * j;
      const double* gi = G + (size_t)(base + r) * K + base;
      double v = 0.0;
      for (int l = r; l < kTb; ++l) v = fma(gi[l], Ts[l][c], v);
      G[(size_t)(base + r) * K + jb * kTb + c] = -v;
    }
}

// ------------------------------------------------------------------ steps 2-4
__global__ void __launch_bounds__(256) gptq_init_kernel(const __half* __restrict__ W, int64_t n_el, int K,
                                                        const uint8_t* __restrict__ dead, double* __restrict__ Wd) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_el; i += (int64_t)gridDim.x * blockDim.x)
    Wd[i] = dead[i % K] ? 0.0 : (double)__half2float(W[i]);
}

// One column block [b0, b0 + 128) for 64 rows per CTA (thread r: row r):
// the rows' block of W and G[block][block] in shared memory; codes are packed
// into the row's words as the group's 32-channel units complete.
template <int BITS, bool SYM, int GS>
__global__ void __launch_bounds__(64) gptq_block_kernel(double* __restrict__ Wd, const double* __restrict__ G, int N,
                                                        int K, int b0, double* __restrict__ Err,
                                                        uint32_t* __restrict__ packed, __half* __restrict__ steps,
                                                        __half* __restrict__ zeros, int* err) {
  extern __shared__ double sm[];
  double* Gs = sm;                         // [128][129]
  double* Ws = sm + kGb * (kGb + 1);       // [64][129]
  const int nb = K - b0 < kGb ? K - b0 : kGb;
  for (int e = threadIdx.x; e < kGb * kGb; e += blockDim.x) {
    const int r = e / kGb, c = e % kGb;
    Gs[r * (kGb + 1) + c] = r < nb && c < nb ? G[(size_t)(b0 + r) * K + b0 + c] : 0.0;
  }
  const int row0 = blockIdx.x * 64;
  for (int e = threadIdx.x; e < 64 * kGb; e += blockDim.x) {
    const int r = e / kGb, c = e % kGb;
    Ws[r * (kGb + 1) + c] = row0 + r < N && c < nb ? Wd[(size_t)(row0 + r) * K + b0 + c] : 0.0;
  }
  __syncthreads();
  const int r = threadIdx.x, n = row0 + r;
  double* w = Ws + r * (kGb + 1);
  constexpr int Q = (1 << BITS) - 1;
  GroupQuant gq{};
  uint8_t codes[32];
  for (int i = 0; i < nb; ++i) {
    if (i % GS == 0) {  // a group starts: step and zero from its current weights (fp32 values)
      float lo = (float)w[i], hi = SYM ? fabsf((float)w[i]) : (float)w[i];
      for (int j = i + 1; j < i + GS; ++j) {
        const float v = (float)w[j];
        if (SYM) {
          hi = max_nan(hi, fabsf(v));
        } else {
          lo = min_nan(lo, v);
          hi = max_nan(hi, v);
        }
      }
      gq = group_quant_from_range<BITS, SYM>(lo, hi);
      if (n < N) {
        if (!isfinite(gq.sf)) latch_error(err, WQ_ERR_RANGE);
        const size_t gi = (size_t)n * (K / GS) + (b0 + i) / GS;
        steps[gi] = gq.step_h;
        zeros[gi] = __int2half_rn(gq.zero);
      }
    }
    const float qf = rintf(__fdiv_rn((float)w[i], gq.sf));  // the quantizer's rounding of the fp32 quotient
    int q;
    if (SYM) {
      constexpr int qmax = (1 << (BITS - 1)) - 1;
      q = (int)fminf(fmaxf(qf, (float)(-qmax - 1)), (float)qmax) + (1 << (BITS - 1));
    } else {
      q = (int)qf + gq.zero;
      q = q < 0 ? 0 : (q > Q ? Q : q);
    }
    codes[i & 31] = (uint8_t)q;
    const double deq = (double)(q - gq.zero) * (double)gq.sf;
    const double e = (w[i] - deq) / Gs[i * (kGb + 1) + i];
    for (int j = i + 1; j < nb; ++j) w[j] -= e * Gs[i * (kGb + 1) + j];
    if (n < N) Err[(size_t)n * kGb + i] = e;
    if ((i & 31) == 31 && n < N) {  // pack the 32-channel unit
      const size_t unit = ((size_t)n * K + b0 + i - 31) / 32;
      if (BITS == 4) {
        uint32_t o[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t wd = 0;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            wd |= (uint32_t)codes[8 * c + 2 * j] << (4 * j);
            wd |= (uint32_t)codes[8 * c + 2 * j + 1] << (4 * (j + 4));
          }
          o[c] = wd;
        }
        reinterpret_cast<uint4*>(packed)[unit] = make_uint4(o[0], o[1], o[2], o[3]);
      } else {
        uint32_t t3[3] = {0, 0, 0};
#pragma unroll
        for (int t = 0; t < 3; ++t)
#pragma unroll
          for (int j = 0; j < 5; ++j) {
            t3[t] |= (uint32_t)codes[10 * t + 2 * j] << (3 * j);
            t3[t] |= (uint32_t)codes[10 * t + 2 * j + 1] << (16 + 3 * j);
          }
#pragma unroll
        for (int b = 0; b < 3; ++b) {
          t3[b] |= ((uint32_t)(codes[30] >> b) & 1u) << 15;
          t3[b] |= ((uint32_t)(codes[31] >> b) & 1u) << 31;
        }
        packed[3 * unit] = t3[0];
        packed[3 * unit + 1] = t3[1];
        packed[3 * unit + 2] = t3[2];
      }
    }
  }
}

// Lazy batch update: Wd[:, b1:] -= Err[:, 0:128] * G[b0:b1, b1:], 64 x 64
// output tiles.
__global__ void __launch_bounds__(256) gptq_update_kernel(double* __restrict__ Wd, const double* __restrict__ Err,
                                                          const double* __restrict__ G, int N, int K, int b0,
                                                          int b1) {
  __shared__ double sbuf[kTileBuf];
  const int r0 = blockIdx.y * kTb, c0 = b1 + blockIdx.x * kTb;
  TileAcc acc = {};
  // Err has whole 64-row tiles (rows past N are 0); K is a multiple of 64
  tile_mma(acc, Err + (size_t)r0 * kGb, kGb, false, G + (size_t)b0 * K + c0, K, false, b1 - b0, sbuf);
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int r = r0 + ty + 16 * i, c = c0 + tx + 16 * j;
      if (r < N && c < K) Wd[(size_t)r * K + c] -= acc.c[i][j];
    }
}

// ------------------------------------------------------------------ host
// Workspace: H (then U in its upper triangle) and G, K x K fp64 each; the
// running weights, N x K fp64; the block errors, ceil(N/64)*64 x 128 fp64;
// the dead-channel flags. K is a multiple of 128, so every 64-tile is whole.
GptqPlan plan_gptq(int64_t N, int64_t K) {
  GptqPlan p;
  auto a256 = [](size_t x) { return (x + 255) & ~size_t(255); };
  const int64_t Np = (N + kTb - 1) / kTb * kTb;
  size_t off = 0;
  p.off_H = off;
  off = a256(off + (size_t)K * K * 8);
  p.off_G = off;
  off = a256(off + (size_t)K * K * 8);
  p.off_W = off;
  off = a256(off + (size_t)N * K * 8);
  p.off_Err = off;
  off = a256(off + (size_t)Np * kGb * 8);
  p.off_dead = off;
  off = a256(off + (size_t)K);
  p.total = off;
  return p;
}

cudaError_t launch_gptq(const void* X, int64_t T, const void* W, int64_t N, int64_t K, int bits, int group, bool sym,
                        double damp, uint32_t* packed, void* steps, void* zeros, void* workspace, int* err,
                        cudaStream_t st) {
  const GptqPlan p = plan_gptq(N, K);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  double* H = reinterpret_cast<double*>(ws + p.off_H);
  double* G = reinterpret_cast<double*>(ws + p.off_G);
  double* Wd = reinterpret_cast<double*>(ws + p.off_W);
  double* Err = reinterpret_cast<double*>(ws + p.off_Err);
  uint8_t* dead = ws + p.off_dead;
  const int Ki = (int)K, Ni = (int)N, KB = Ki / kTb;
  cudaError_t e;
  if ((e = cudaMemsetAsync(G, 0, (size_t)K * K * 8, st)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(Err, 0, (size_t)((N + kTb - 1) / kTb * kTb) * kGb * 8, st)) != cudaSuccess) return e;
  // step 1: H, damping, H = U U^T, G = U^-1
  gptq_hessian_kernel<<<dim3(KB, KB), 256, 0, st>>>(static_cast<const __half*>(X), (int)T, Ki, H);
  gptq_damp_kernel<<<1, 1024, 0, st>>>(H, Ki, damp, dead);
  for (int kb = KB - 1; kb >= 0; --kb) {
    ul_diag_kernel<<<1, 256, 0, st>>>(H, Ki, kb, err);
    if (kb > 0) {
      ul_panel_kernel<<<kb, kTb, 0, st>>>(H, Ki, kb);
      ul_update_kernel<<<dim3(kb, kb), 256, 0, st>>>(H, Ki, kb);
    }
  }
  for (int ib = KB - 1; ib >= 0; --ib) {
    trinv_diag_kernel<<<1, 256, 0, st>>>(H, Ki, ib, G);
    if (ib < KB - 1) trinv_row_kernel<<<KB - 1 - ib, 256, 0, st>>>(H, Ki, ib, G);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // steps 2-4 over column blocks of 128
  gptq_init_kernel<<<1184, 256, 0, st>>>(static_cast<const __half*>(W), N * K, Ki, dead, Wd);
  const size_t smem = (size_t)(kGb * (kGb + 1) + 64 * (kGb + 1)) * 8;
  auto run = [&](auto kern) -> cudaError_t {
    cudaError_t e2 = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e2 != cudaSuccess) return e2;
    for (int b0 = 0; b0 < Ki; b0 += kGb) {
      const int b1 = b0 + kGb;
      kern<<<(unsigned)((N + 63) / 64), 64, smem, st>>>(Wd, G, Ni, Ki, b0, Err, packed,
                                                        static_cast<__half*>(steps), static_cast<__half*>(zeros),
                                                        err);
      if (b1 < Ki)
        gptq_update_kernel<<<dim3((unsigned)((Ki - b1) / kTb), (unsigned)((N + kTb - 1) / kTb)), 256, 0, st>>>(
            Wd, Err, G, Ni, Ki, b0, b1);
    }
    return cudaGetLastError();
  };
#define WQ_GP(B, S, GSZ) return run(gptq_block_kernel<B, S, GSZ>)
  if (bits == 4) {
    if (sym) {
      if (group == 32) WQ_GP(4, true, 32);
      if (group == 64) WQ_GP(4, true, 64);
      WQ_GP(4, true, 128);
    }
    if (group == 32) WQ_GP(4, false, 32);
    if (group == 64) WQ_GP(4, false, 64);
    WQ_GP(4, false, 128);
  }
  if (sym) {
    if (group == 32) WQ_GP(3, true, 32);
    if (group == 64) WQ_GP(3, true, 64);
    WQ_GP(3, true, 128);
  }
  if (group == 32) WQ_GP(3, false, 32);
  if (group == 64) WQ_GP(3, false, 64);
  WQ_GP(3, false, 128);
#undef WQ_GP
}

}  // namespace wq
