// S6: W4A16 / W3A16 matmul on the 5th-generation tensor cores for M = 3..256
// rows of X per launch (larger M in chunks of 256).
//
// When M grows the weight-only matmul stops being a pure weight stream and
// becomes a dense contraction ("Quantising Large Language Models for
// Efficient Inference", "Weight-only vs weight-and-activation quantisation":
// weights are dequantized inside the matmul; tensor cores pay off for larger
// batches). The weight is still read once, packed, and dequantized on chip.
//
// Tile: one CTA owns 128 output channels n and all M rows of X ("swap AB":
// the dequantized weight tile is the 128-row A operand, held in tensor
// memory; X is the B operand with N_mma = M rounded up to 16; D = W X^T lives
// in tensor memory as [128 lanes = n][M columns]). K advances in stages of
// BK = 128 (one quantization group) or 64 input channels:
//   warp 0    TMA producer into a ring of S shared-memory stages: the packed
//             tile (128 rows x BK/2 bytes for 4-bit, 64- or 32-byte swizzle;
//             128 rows x 48 bytes for 3-bit, unswizzled) and the X
//             tile (BK/64 128-byte-swizzled 64-channel boxes)
//   warp 1    TMEM owner and single-thread tcgen05.mma issuer (BK/16 MMAs
//             per stage)
//   warps 2.. NH quartets of 4 warps dequantize the packed tile into a ring
//             of tensor-memory A buffers (warp w: output channels
//             32*(w%4)..+31 -- the TMEM lane quarter it may access; quartet h
//             takes the stages kt = h mod NH, so NH stages are dequantized at
//             once), then run the epilogue (tcgen05.ld -> fp16 -> Y).
// The shared-memory ring and the TMEM A ring are separate, so the TMA runs as
// far ahead as shared memory allows while only two or three A buffers occupy
// TMEM.
// Schedules:
//   per tile  one CTA per 128-row tile; when the row tiles cannot fill the
//             GPU (N = 8192 gives 64 tiles for 148 SMs), the KS CTAs of a
//             thread-block cluster take consecutive K ranges of the same
//             tile; ranks 1.. send their fp32 partial tiles to rank 0's
//             shared memory (its idle ring) over distributed shared memory,
//             and rank 0 adds them in rank order (deterministic) and writes Y.
//   stream-K  (SK, with a caller workspace) a persistent grid; CTA c takes the
//             (tile, stage) units [c U / P, (c + 1) U / P), at most one
//             tile's worth: the end of one tile and the start of the next,
//             each accumulated in its own TMEM columns. Partial tiles go to
//             the workspace; per tile and lane quarter, the warp that arrives
//             last at a counter adds all contributors' tiles in CTA order
//             (deterministic), writes Y and zeroes the counter. No CTA waits
//             for another.
// Every mbarrier wait is bounded; on a timeout the kernel latches
// WQ_ERR_TIMEOUT, drains its own copies, frees its tensor memory and returns.
#include <cooperative_groups.h>
#include <type_traits>

#include "wq_sm100.cuh"
#include "wq_launch.h"

namespace wq {

using namespace sm100;

constexpr int kTcRows = 128;             // output channels per CTA
constexpr int kTcMaxABufs = 3;           // TMEM A buffers at most (barrier space)

struct TcArgs {
  const __half* steps;
  const __half* zeros;
  __half* Y;
  int M, N, K;
  int BN;          // MMA N (M rounded up to 16)
  int stages;      // shared-memory ring depth
  uint32_t tmem_cols;
  int* err;
  long long spin_limit;  // SM clock cycles a bounded wait may last
  int stall;             // test hook: issue no loads, so every consumer wait runs out
  int ksplit;            // CTAs of a cluster sharing one row tile along K (grid.y)
  int streamk;           // 1: CTA c takes stage units [c U / P, (c + 1) U / P) of all tiles, at most
                         // one tile's worth, so at most two segments; segment j accumulates in TMEM
                         // columns [j BN, (j + 1) BN)
  long long units;       // U = row tiles * stages per row
  float* part;           // stream-K: fp32 partial tiles, two slots per CTA [P][2][128][BN]
  unsigned* cnt;         // stream-K: arrivals per tile and TMEM lane quarter [tiles][4]; zero before
                         // a launch, and zero again after it (the last arrival resets its counter)
};

__device__ __forceinline__ __half2 u2h(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }
__device__ __forceinline__ uint32_t h2u(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }

// Eight 4-bit codes (one packed word: k0..k7) -> four fp16 pairs
// fp16_rn((q - zero) * step), in k order. (1024+q) - (1024+zero) and
// (1024+16q)/16 - (64+zero) are exact, so the only rounding is the product.
__device__ __forceinline__ uint4 dequant_word4(uint32_t w, __half2 zz, __half2 zz16n, __half2 s2) {
  const __half2 one16 = __float2half2_rn(0.0625f);
  const uint32_t w8 = w >> 8;
  const uint32_t p0 = and_or(w, 0x000F000Fu, kHalf2Magic);
  const uint32_t p1 = and_or(w, 0x00F000F0u, kHalf2Magic);
  const uint32_t p2 = and_or(w8, 0x000F000Fu, kHalf2Magic);
  const uint32_t p3 = and_or(w8, 0x00F000F0u, kHalf2Magic);
  uint4 r;
  r.x = h2u(__hmul2(__hsub2(u2h(p0), zz), s2));
  r.y = h2u(__hmul2(__hfma2(u2h(p1), one16, zz16n), s2));
  r.z = h2u(__hmul2(__hsub2(u2h(p2), zz), s2));
  r.w = h2u(__hmul2(__hfma2(u2h(p3), one16, zz16n), s2));
  return r;
}

// 32 3-bit codes (three packed words: k0..k31) -> sixteen fp16 pairs
// fp16_rn((q - zero) * step), in k order. One LOP3 leaves a pair as
// 1024 + c q with c = 1, 8 or 64 (the code's bit offset in its 16-bit lane);
// (1024 + c q) / c - (1024 / c + zero) is exact, so again the only rounding
// is the product. Pair j of word t holds k = 10t + 2j, 10t + 2j + 1; bit b of
// k = 30 and 31 sits in bit 15 and 31 of word b.
__device__ __forceinline__ void dequant_chunk3(const uint32_t* w3, __half2 zz, __half2 zz8n, __half2 zz64n, __half2 s2,
                                               uint32_t (&o)[16]) {
  const __half2 i8 = __float2half2_rn(0.125f), i64 = __float2half2_rn(0.015625f);
#pragma unroll
  for (int t = 0; t < 3; ++t) {
    const uint32_t w = w3[t], w9 = w >> 9;
    o[5 * t + 0] = h2u(__hmul2(__hsub2(u2h(and_or(w, 0x00070007u, kHalf2Magic)), zz), s2));
    o[5 * t + 1] = h2u(__hmul2(__hfma2(u2h(and_or(w, 0x00380038u, kHalf2Magic)), i8, zz8n), s2));
    o[5 * t + 2] = h2u(__hmul2(__hfma2(u2h(and_or(w, 0x01C001C0u, kHalf2Magic)), i64, zz64n), s2));
    o[5 * t + 3] = h2u(__hmul2(__hsub2(u2h(and_or(w9, 0x00070007u, kHalf2Magic)), zz), s2));
    o[5 * t + 4] = h2u(__hmul2(__hfma2(u2h(and_or(w9, 0x00380038u, kHalf2Magic)), i8, zz8n), s2));
  }
  uint32_t hb = and_or(w3[0] >> 15, 0x00010001u, kHalf2Magic);
  hb = and_or(w3[1] >> 14, 0x00020002u, hb);
  hb = and_or(w3[2] >> 13, 0x00040004u, hb);
  o[15] = h2u(__hmul2(__hsub2(u2h(hb), zz), s2));
}

// BITS: 4 (packed words of 8 codes) or 3 (chunks of three words per 32 codes;
// 128-channel stages, rows of 48 bytes, no swizzle needed: a quarter warp's
// 16-byte reads at a 48-byte row pitch already fall on distinct banks).
// BK: input channels per stage, 128 (one group) or 64 (half a group; shallower
// shared-memory stages, so a deeper ring fits when M is large; 4-bit only).
// NH: dequantizing warp quartets; quartet h owns the stages kt = h mod NH
// whole (every row, every channel), so the per-stage chain of one quartet
// (wait for the tile, dequantize, store to tensor memory, publish) overlaps
// with the other quartets' stages.
// NA: depth of the TMEM A ring (2, or 3 when the tile leaves room).
// GS: quantization group (128, or 32 / 64 channels: then every stage holds
// BK / GS groups, and each dequantizing thread applies the step and zero of
// the NGT groups of its part of the stage).
template <int BITS, int BK, int NH, int NA, int GS, bool SK>
__global__ void __launch_bounds__(64 + 128 * NH, 1)
w4a16_gemm_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmP,
                     TcArgs a) {
  static_assert(BITS == 4 || (BITS == 3 && BK == 128), "3-bit tiles: 128-channel stages");
  static_assert(!SK || NH == 1, "stream-K: one dequantizing quartet");
  constexpr int NGT = GS < BK ? BK / GS : 1;      // groups in one stage
  constexpr int kRowBytes = BK * BITS / 8;        // packed bytes of one row and stage
  constexpr int kPackedStage = kTcRows * kRowBytes;  // bytes of the packed tile
  constexpr int kACols = BK / 2;                  // TMEM columns per A buffer
  constexpr int kXBoxes = BK / 64;                // 64-channel X boxes per stage
  constexpr int kWords = BK * BITS / 32;          // packed words per dequant thread and stage
  constexpr int kChunks = kWords / 4;             // 16-byte chunks per dequant thread and stage
  constexpr int kRegs = BK / 2;                   // fp16 pairs per dequant thread and stage
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int S = a.stages;
  const int xbox = a.BN * 128;                       // one 64-channel X box
  const int stage_bytes = kXBoxes * xbox + kPackedStage;  // X boxes + packed
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)S * stage_bytes);
  uint64_t* sempty = full + S;
  uint64_t* afull = sempty + S;
  uint64_t* aempty = afull + kTcMaxABufs;
  uint64_t* accum = aempty + kTcMaxABufs;  // accum[j]: segment j's accumulator is complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  auto stageX = [&](int s) { return smem + (size_t)s * stage_bytes; };
  auto stageP = [&](int s) { return smem + (size_t)s * stage_bytes + kXBoxes * xbox; };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // This CTA's stages are the units [u0, u1) of the (row tile, stage) space,
  // tile-major: unit u is stage u % KT_all of row tile u / KT_all. Per-tile
  // schedule: one tile (blockIdx.x), and with split K the y-th of ksplit
  // consecutive stage ranges. Stream-K: CTA c takes [c U / P, (c + 1) U / P)
  // of all U units (P = gridDim.x), so every CTA gets the same number of
  // stages; a maximal run of one tile's stages is a segment.
  const int KT_all = a.K / BK;
  long long u0, u1;
  if constexpr (SK) {
    u0 = (long long)blockIdx.x * a.units / gridDim.x;
    u1 = (long long)(blockIdx.x + 1) * a.units / gridDim.x;
  } else {
    const long long base = (long long)blockIdx.x * KT_all;
    u0 = base + ((long long)KT_all * blockIdx.y) / a.ksplit;
    u1 = base + ((long long)KT_all * (blockIdx.y + 1)) / a.ksplit;
  }
  const int KT = (int)(u1 - u0);  // stages of this CTA
  const int tile0 = (int)(u0 / KT_all), kg0 = (int)(u0 % KT_all);
  // segments: j = 0 (row tile tile0, stages [kg0, ke0)), and with stream-K
  // possibly j = 1 (row tile tile0 + 1, stages [0, ke1))
  const int nseg = SK && KT > 0 && (int)((u1 - 1) / KT_all) != tile0 ? 2 : 1;
  const int ke0 = nseg == 2 ? KT_all : kg0 + KT;
  const int ke1 = nseg == 2 ? (int)((u1 - 1) % KT_all) + 1 : 0;
  const int G = a.K / GS;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&sempty[s], 1);
    }
    for (int b = 0; b < NA; ++b) {
      mbar_init(&afull[b], 128);
      mbar_init(&aempty[b], 1);
    }
    mbar_init(&accum[0], 1);
    mbar_init(&accum[1], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, a.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tmem_a = tmem + (uint32_t)(a.BN * (SK ? 2 : 1));  // A buffers follow the accumulator(s)

  if (warp == 0) {
    // ---------------------------------------------------------- TMA producer
    if (lane == 0) {
      prefetch_tensormap(&tmX);
      prefetch_tensormap(&tmP);
      int issued = 0;
      for (int j = 0, s = 0, u = 0; j < (a.stall ? 0 : nseg) && !*abort_flag; ++j) {  // s = kt % S, u = kt / S
        const int row0 = (tile0 + j) * kTcRows, kb = j == 0 ? kg0 : 0, ke = j == 0 ? ke0 : ke1;
        for (int kg = kb; kg < ke; ++kg) {
          if (*abort_flag) break;
          if (u > 0 && !mbar_wait(&sempty[s], (u - 1) & 1, a.err, a.spin_limit)) { *abort_flag = 1; break; }
          mbar_arrive_expect_tx(&full[s], (uint32_t)stage_bytes);
#pragma unroll
          for (int i = 0; i < kXBoxes; ++i) tma_load_2d(stageX(s) + i * xbox, &tmX, kg * BK + 64 * i, 0, &full[s]);
          tma_load_2d(stageP(s), &tmP, kg * (kRowBytes / 4), row0, &full[s]);
          ++issued;
          if (++s == S) { s = 0; ++u; }
        }
      }
      // Drain: every copy this thread issued has landed before the CTA exits.
      for (int kt = issued > S ? issued - S : 0; kt < issued; ++kt)
        mbar_wait(&full[kt % S], (kt / S) & 1, a.err, a.spin_limit);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_f16_f32(kTcRows, a.BN);
      int committed = -1;  // stages whose MMAs were issued, minus one
      for (int j = 0, s = 0, b = 0, ub = 0; j < nseg && !*abort_flag; ++j) {
        const int kb = j == 0 ? kg0 : 0, ke = j == 0 ? ke0 : ke1;
        const uint32_t d = tmem + (uint32_t)(j * a.BN);  // segment j's accumulator
        for (int kg = kb; kg < ke; ++kg) {
          if (*abort_flag) break;
          if (!mbar_wait(&afull[b], ub & 1, a.err, a.spin_limit)) { *abort_flag = 1; break; }
          tc_fence_after();
          const uint32_t xaddr = smem_u32(stageX(s));
#pragma unroll
          for (int jj = 0; jj < BK / 16; ++jj) {
            const uint64_t bd = desc_kmajor_sw128(xaddr + (uint32_t)((jj >> 2) * xbox + (jj & 3) * 32));
            mma_f16_ts(d, tmem_a + (uint32_t)(b * kACols + 8 * jj), bd, idesc, (kg > kb || jj > 0) ? 1u : 0u);
          }
          mma_commit(&aempty[b]);
          mma_commit(&sempty[s]);
          ++committed;
          if (++s == S) s = 0;
          if (++b == NA) { b = 0; ++ub; }
        }
        if (!*abort_flag) mma_commit(&accum[j]);  // the segment's accumulator is complete
      }
      if (*abort_flag && committed >= 0)  // let issued MMAs finish before teardown
        mbar_wait(&aempty[committed % NA], (committed / NA) & 1, a.err, a.spin_limit);
    }
  } else {
    // ---------------------------------------------------------- dequant + epilogue
    const int q = warp & 3;             // TMEM lane quarter this warp may access
    const int h = (warp - 2) >> 2;      // quartet: stages kt = h mod NH
    const int r = 32 * q + lane;        // output channel within the tile
    // Stream-K bookkeeping: the CTA that holds unit u, the first unit of CTA c
    const long long P = gridDim.x;
    auto owner = [&](long long u) { return (int)(((u + 1) * P - 1) / a.units); };
    auto first_unit = [&](int c) { return (long long)c * a.units / P; };

    // Epilogue of segment `seg` (row tile `tile`, accumulator columns seg * BN):
    // a whole tile goes to Y; a partial one (stream-K) goes to this CTA's slot
    // `seg`, and the warp that arrives last at the tile's lane-quarter counter
    // adds all contributors' slots in CTA order (deterministic) and writes Y.
    // Returns false on abort.
    auto epilogue = [&](int tile, int seg, bool whole) -> bool {
      const uint32_t dcol = (uint32_t)(seg * a.BN);
      bool done = !__any_sync(0xffffffffu, *abort_flag != 0);
      if (done) done = __all_sync(0xffffffffu, mbar_wait(&accum[seg], 0, a.err, a.spin_limit));
      if (!done) { *abort_flag = 1; return false; }
      tc_fence_after();
      const int n = tile * kTcRows + r;
      if (whole) {
        if (a.ksplit == 1) {
          for (int c0 = 16 * h; c0 < a.BN; c0 += 16 * NH) {
            uint32_t v[16];
            tmem_ld16(tmem + dcol + ((uint32_t)(32 * q) << 16) + (uint32_t)c0, v);
            tmem_ld_wait();
            if (n < a.N) {
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const int m = c0 + i;
                if (m < a.M) a.Y[(size_t)m * a.N + n] = __float2half_rn(__uint_as_float(v[i]));
              }
            }
          }
        }
        return true;
      }
      if constexpr (SK) {
        float* slot = a.part + ((size_t)(2 * blockIdx.x + seg) * kTcRows + r) * a.BN;
        for (int c0 = 0; c0 < a.BN; c0 += 16) {
          uint32_t v[16];
          tmem_ld16(tmem + dcol + ((uint32_t)(32 * q) << 16) + (uint32_t)c0, v);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; i += 4)
            *reinterpret_cast<float4*>(slot + c0 + i) = make_float4(__uint_as_float(v[i]), __uint_as_float(v[i + 1]),
                                                                    __uint_as_float(v[i + 2]), __uint_as_float(v[i + 3]));
        }
        __threadfence();
        __syncwarp();
        const long long tu0 = (long long)tile * KT_all;
        const int cfirst = owner(tu0), clast = owner(tu0 + KT_all - 1);
        unsigned arrived = 0;
        if (lane == 0) arrived = atomicAdd(&a.cnt[4 * tile + q], 1u);
        arrived = __shfl_sync(0xffffffffu, arrived, 0);
        if (arrived == (unsigned)(clast - cfirst)) {  // every other contributor's slot is written
          if (lane == 0) a.cnt[4 * tile + q] = 0u;   // zero again for the next launch
          __threadfence();
          for (int c0 = 0; c0 < a.BN; c0 += 16) {
            float t[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) t[i] = 0.f;
            for (int c = cfirst; c <= clast; ++c) {
              const int wc = first_unit(c) / KT_all == tile ? 0 : 1;
              const float* src = a.part + ((size_t)(2 * c + wc) * kTcRows + r) * a.BN + c0;
#pragma unroll
              for (int i = 0; i < 16; i += 4) {
                const float4 f = __ldcg(reinterpret_cast<const float4*>(src + i));
                t[i] += f.x; t[i + 1] += f.y; t[i + 2] += f.z; t[i + 3] += f.w;
              }
            }
            if (n < a.N) {
#pragma unroll
              for (int i = 0; i < 16; ++i)
                if (c0 + i < a.M) a.Y[(size_t)(c0 + i) * a.N + n] = __float2half_rn(t[i]);
            }
          }
        }
      }
      return true;
    };

    // step and zero of the NGT groups of this quartet's current stage, and of
    // its next stage, fetched one stage ahead of their use
    __half st_cur[NGT], zr_cur[NGT], st_next[NGT], zr_next[NGT];
    const __half hzero = __float2half(0.f);
    // this thread's row of steps and zeros in segment j's tile (row 0 past N:
    // its values are never stored)
    auto row_of = [&](int j) {
      const int row = (tile0 + j) * kTcRows + r;
      return (size_t)(row < a.N ? row : 0) * G;
    };
    auto fetch = [&](size_t rowg, int kg) {
#pragma unroll
      for (int i = 0; i < NGT; ++i) {
        st_next[i] = a.steps[rowg + (kg * BK) / GS + i];
        zr_next[i] = a.zeros[rowg + (kg * BK) / GS + i];
      }
    };
#pragma unroll
    for (int i = 0; i < NGT; ++i) st_cur[i] = zr_cur[i] = st_next[i] = zr_next[i] = hzero;
    // Software pipeline: stage kt is dequantized into registers while the
    // tensor-memory stores of this quartet's previous stage complete; then that
    // stage is published to the MMA issuer and kt's stores are issued
    // (tcgen05.st reads its source registers when it issues, so they need no
    // copy).
    int pend_b = -1;  // A buffer whose stores are in flight (-1: none)
    bool ok_all = true;
    // the quartet's first stage: kt = h (segment 0 unless it is shorter)
    if (h < ke0 - kg0) fetch(row_of(0), kg0 + h);
    else if (h < KT) fetch(row_of(1), h - (ke0 - kg0));
    // kt: this CTA's stage index; s = kt mod S, u = kt / S, b = kt mod NA,
    // ub = kt / NA (NH <= S, NA). Two segments only with one quartet.
    int kt = h, s = h, u = 0, b = h, ub = 0;
    for (int j = 0; j < nseg && ok_all; ++j) {
      const int kb = j == 0 ? kg0 : 0, ke = j == 0 ? ke0 : ke1;
      const int off = j == 0 ? 0 : ke0 - kg0;  // kt of the segment's first stage
      const size_t rowg = row_of(j);
      const size_t rowg_next = j + 1 < nseg ? row_of(j + 1) : rowg;
      for (; kt < off + (ke - kb); kt += NH) {
        if (__any_sync(0xffffffffu, *abort_flag != 0)) { ok_all = false; break; }
        const int kg = kb + (kt - off);
        const int kn = kg + NH;  // this quartet's next stage, if in this segment
#pragma unroll
        for (int i = 0; i < NGT; ++i) {
          st_cur[i] = st_next[i];
          zr_cur[i] = zr_next[i];
        }
        // (the next stage's group may be this one: half-group stages)
        if (kn < ke) {
          if (GS < BK || (kn * BK) / GS != (kg * BK) / GS) fetch(rowg, kn);
        } else if (j + 1 < nseg) {
          fetch(rowg_next, 0);
        }
        __half2 s2[NGT], zz[NGT], zz16n[NGT];
#pragma unroll
        for (int i = 0; i < NGT; ++i) {
          s2[i] = __halves2half2(st_cur[i], st_cur[i]);
          const __half z1024 = __hadd(zr_cur[i], __float2half(1024.f));
          const __half z64n = __hneg(__hadd(zr_cur[i], __float2half(64.f)));
          zz[i] = __halves2half2(z1024, z1024);
          zz16n[i] = __halves2half2(z64n, z64n);
        }
        const bool landed = mbar_wait(&full[s], u & 1, a.err, a.spin_limit);
        if (!__all_sync(0xffffffffu, landed)) { *abort_flag = 1; ok_all = false; break; }
        // The 4-bit packed tile is swizzled by the TMA: with 64-byte rows (BK =
        // 128) 16-byte chunk c of row r sits at chunk c ^ ((r >> 1) & 3), with
        // 32-byte rows (BK = 64) at c ^ ((r >> 2) & 1); both keep a warp's loads
        // conflict-free. 3-bit rows (48 bytes) are not swizzled.
        uint32_t words[kWords];
        const uint8_t* prow = stageP(s) + r * kRowBytes;
        const int sw = BITS == 3 ? 0 : BK == 128 ? (r >> 1) & 3 : (r >> 2) & 1;
#pragma unroll
        for (int i = 0; i < kChunks; ++i) {
          const uint4 v = *reinterpret_cast<const uint4*>(prow + ((i ^ sw) << 4));
          words[4 * i] = v.x; words[4 * i + 1] = v.y; words[4 * i + 2] = v.z; words[4 * i + 3] = v.w;
        }
        uint32_t nv[kRegs / 16][16];
        if constexpr (BITS == 4) {
#pragma unroll
          for (int j = 0; j < kWords; ++j) {
            const int gi = 8 * j / (GS < BK ? GS : BK);  // word j's group within the stage
            const uint4 d = dequant_word4(words[j], zz[gi], zz16n[gi], s2[gi]);
            nv[j >> 2][4 * (j & 3)] = d.x; nv[j >> 2][4 * (j & 3) + 1] = d.y;
            nv[j >> 2][4 * (j & 3) + 2] = d.z; nv[j >> 2][4 * (j & 3) + 3] = d.w;
          }
        } else {
#pragma unroll
          for (int c = 0; c < kRegs / 16; ++c) {  // 32 channels from three words
            const int gi = 32 * c / (GS < BK ? GS : BK);
            const __half z128n = __hneg(__hadd(zr_cur[gi], __float2half(128.f)));
            const __half z16n = __hneg(__hadd(zr_cur[gi], __float2half(16.f)));
            dequant_chunk3(&words[3 * c], zz[gi], __halves2half2(z128n, z128n), __halves2half2(z16n, z16n), s2[gi],
                           nv[c]);
          }
        }
        if (pend_b >= 0) {  // publish this quartet's previous stage
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(&afull[pend_b]);
          pend_b = -1;
        }
        bool ok = true;
        if (kt >= NA) ok = mbar_wait(&aempty[b], (ub - 1) & 1, a.err, a.spin_limit);
        if (!__all_sync(0xffffffffu, ok)) { *abort_flag = 1; ok_all = false; break; }
        const uint32_t ta = tmem_a + ((uint32_t)(32 * q) << 16) + (uint32_t)(b * kACols);
#pragma unroll
        for (int i = 0; i < kRegs / 16; ++i) tmem_st16(ta + 16 * i, nv[i]);
        pend_b = b;
        if ((s += NH) >= S) { s -= S; ++u; }
        if ((b += NH) >= NA) { b -= NA; ++ub; }
      }
    }
    if (pend_b >= 0) {
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&afull[pend_b]);
    }
    // Epilogues: segment 0 (tile0, from stage kg0) and, when the CTA's stages
    // cross a tile boundary (stream-K), segment 1 (the next tile, up to stage
    // kg1).
    if (ok_all && KT > 0) {
      const int kg1 = (int)((u1 - 1) % KT_all);
      const bool two = (u1 - 1) / KT_all != tile0;
      if constexpr (!SK) {
        epilogue(tile0, 0, true);
      } else if (epilogue(tile0, 0, kg0 == 0 && (two || kg1 == KT_all - 1)) && two) {
        epilogue(tile0 + 1, 1, kg1 == KT_all - 1);
      }
    } else if (!ok_all) {
      *abort_flag = 1;
    }
  }

  if (a.ksplit > 1) {
    // Split K: every CTA of the cluster is past its K loop (rank 0's ring is
    // idle) before rank r > 0 writes its partial tile [row][m] (fp32) into
    // slot r - 1 of rank 0's ring; after the second cluster barrier rank 0 adds
    // them to its own accumulator in rank order. All threads of every CTA
    // reach both barriers, on every path.
    namespace cg = cooperative_groups;
    cg::cluster_group cl = cg::this_cluster();
    const unsigned rank = cl.block_rank();
    const bool epi = warp >= 2 && warp < 2 + 4 * NH;
    const int q = warp & 3, h = (warp - 2) >> 2;
    const int r = 32 * q + (int)(threadIdx.x & 31);
    const int n = (int)blockIdx.x * kTcRows + r;
    tc_fence_before();
    cl.sync();
    tc_fence_after();
    const bool ok = !*abort_flag;  // read after the barrier: one value per CTA
    float* part = reinterpret_cast<float*>(smem);  // rank 0's ring: [ksplit - 1][128][BN]
    if (epi && rank > 0 && ok) {
      float* dst = cl.map_shared_rank(part, 0) + ((size_t)(rank - 1) * kTcRows + r) * a.BN;
      for (int c0 = 16 * h; c0 < a.BN; c0 += 16 * NH) {
        uint32_t v[16];
        tmem_ld16(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)c0, v);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) dst[c0 + i] = __uint_as_float(v[i]);
      }
    }
    tc_fence_before();
    cl.sync();
    tc_fence_after();
    if (epi && rank == 0 && ok) {
      for (int c0 = 16 * h; c0 < a.BN; c0 += 16 * NH) {
        uint32_t v[16];
        tmem_ld16(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)c0, v);
        tmem_ld_wait();
        if (n < a.N) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int m = c0 + i;
            float t = __uint_as_float(v[i]);
            for (int k = 1; k < a.ksplit; ++k) t += part[((size_t)(k - 1) * kTcRows + r) * a.BN + m];
            if (m < a.M) a.Y[(size_t)m * a.N + n] = __float2half_rn(t);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, a.tmem_cols);
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

static int tc_num_sms() {
  static int sms = 0;
  if (sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms <= 0) sms = 148;
  }
  return sms;
}

static uint32_t pow2_cols(uint32_t c) {
  uint32_t p = 32;
  while (p < c) p <<= 1;
  return p;
}

// Shape of one launch for a chunk of mc <= 256 rows of X.
struct TcShape {
  int BN, BK, NA, cps, S, stage;
  uint32_t tmem_cols;
  size_t smem;
};

// stages_opt: 0 = library choice; otherwise the shared-memory ring depth (two
// CTAs per SM when that ring and the tile's TMEM fit half an SM).
// bk_opt: 0 = library choice, else 64 or 128 input channels per stage.
static bool tc_shape(int mc, int bits, int stages_opt, int bk_opt, TcShape& t) {
  t.BN = ((mc + 15) / 16) * 16;
  // Half-group stages for wide X tiles (BN >= 96: a 5-deep ring still fits
  // two CTAs per SM), whole-group stages otherwise (fewer waits per weight).
  // 3-bit tiles always take 128-channel stages (a 64-channel row would be
  // 24 bytes, not a whole number of 16-byte TMA units).
  t.BK = bits == 3 ? 128 : bk_opt != 0 ? bk_opt : (t.BN >= 96 ? 64 : 128);
  // A third A buffer when it still fits the same TMEM allocation
  t.NA = pow2_cols((uint32_t)(t.BN + 3 * t.BK / 2)) == pow2_cols((uint32_t)(t.BN + 2 * t.BK / 2)) ? 3 : 2;
  t.tmem_cols = pow2_cols((uint32_t)(t.BN + t.NA * t.BK / 2));
  // CTAs per SM: as many as the 512 TMEM columns hold (1, 2 or 4), fewer
  // while their share of shared memory cannot hold a ring of three stages.
  // The ring then takes that share (at most 16 stages).
  t.stage = (t.BK / 64) * t.BN * 128 + kTcRows * t.BK * bits / 8;
  auto share = [](int c) { return (size_t)(225 * 1024) / (size_t)c - 3 * 1024; };
  t.cps = 512 / (int)t.tmem_cols;
  if (stages_opt > 0) {
    t.S = stages_opt;
    while (t.cps > 1 && (size_t)t.S * t.stage + 2048 > share(t.cps)) t.cps /= 2;
    if ((size_t)t.S * t.stage + 2048 > share(1)) return false;
  } else {
    while (t.cps > 1 && 3 * (size_t)t.stage + 2048 > share(t.cps)) t.cps /= 2;
    t.S = (int)((share(t.cps) - 2048) / t.stage);
    if (t.S > 16) t.S = 16;
    if (t.S < 2) t.S = 2;
  }
  t.smem = 1024 + (size_t)t.S * t.stage + (2 * t.S + 2 * kTcMaxABufs + 2) * 8 + 16;
  // At most cps CTAs per SM (their TMEM must fit at once): ask for more than
  // 1/(cps+1) of the SM's shared memory.
  const size_t smem_floor = (size_t)(228 * 1024) / (size_t)(t.cps + 1) + 1024;
  if (t.smem < smem_floor) t.smem = smem_floor;
  return true;
}

// Stream-K: CTAs of the persistent grid (every resident slot, at least two
// stages each) and the workspace they need: the arrival counters (one per row
// tile and TMEM lane quarter) in a fixed first region, so that calls of any
// shape that share a workspace find them where they left them (zero), then
// two fp32 partial tiles per CTA.
constexpr size_t kTcCounterBytes = 64 * 1024;  // row tiles <= 4096
static long long tc_streamk_ctas(const TcShape& t, int tiles, int KT_all) {
  const long long units = (long long)tiles * KT_all;
  long long P = (long long)t.cps * tc_num_sms();
  if (P > units / 2) P = units / 2;
  return P < 1 ? 1 : P;
}
static size_t tc_streamk_bytes(const TcShape& t, long long P) {
  return kTcCounterBytes + (size_t)P * 2 * kTcRows * t.BN * 4;
}

size_t gemm_tc_workspace_bytes(int64_t M, int64_t N, int64_t K, int bits) {
  TcShape t;
  const int mc = (int)(M < 256 ? M : 256);
  if (M < 1 || !tc_shape(mc, bits, 0, 0, t)) return 0;
  const int tiles = (int)((N + kTcRows - 1) / kTcRows);
  return tc_streamk_bytes(t, tc_streamk_ctas(t, tiles, (int)(K / t.BK)));
}

// dw_opt: 0 = library choice (4), else 4 or 8 dequantizing warps.
// ksplit_opt: 0 = library choice, else 1, 2, 4 or 8 CTAs of a cluster along K.
// streamk_opt: 0 = library choice (stream-K when a large enough workspace is
// given and X has at most 16 rows: measured faster or equal on every weight
// shape of the bench there, slower from 32 rows on, where the partial tiles
// grow), 1 = off, 2 = on whenever the workspace is large enough.
// wait_ms: how long a bounded mbarrier wait may last; stall: test hook (the
// producer issues no loads, so the kernel's waits run out and it returns with
// WQ_ERR_TIMEOUT latched).
cudaError_t launch_gemm_tc(const void* X, const uint32_t* packed, const void* steps, const void* zeros, int64_t M,
                           int64_t N, int64_t K, int bits, int group, void* Y, int* err, cudaStream_t st,
                           int stages_opt, int bk_opt, int dw_opt, int ksplit_opt, int streamk_opt, void* workspace,
                           size_t workspace_bytes, int wait_ms, bool stall) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  for (int64_t m0 = 0; m0 < M; m0 += 256) {
    const int mc = (int)((M - m0) < 256 ? (M - m0) : 256);
    TcShape t;
    if (!tc_shape(mc, bits, stages_opt, bk_opt, t)) return cudaErrorInvalidValue;
    const int BN = t.BN, BK = t.BK, NA = t.NA, S = t.S;
    CUtensorMap tmX, tmP;
    {
      cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)mc};
      cuuint64_t strides[1] = {(cuuint64_t)K * 2};
      cuuint32_t box[2] = {64, (cuuint32_t)BN};
      cuuint32_t es[2] = {1, 1};
      void* base = const_cast<__half*>(static_cast<const __half*>(X) + m0 * K);
      if (enc(&tmX, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, base, dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    }
    {
      // [N][K * bits / 32] words; a box is 128 rows of one stage's words
      // (64 or 32 bytes, swizzled, for 4-bit; 48 bytes, unswizzled, for 3-bit)
      cuuint64_t dims[2] = {(cuuint64_t)(K * bits / 32), (cuuint64_t)N};
      cuuint64_t strides[1] = {(cuuint64_t)(K * bits / 8)};
      cuuint32_t box[2] = {(cuuint32_t)(BK * bits / 32), 128};
      cuuint32_t es[2] = {1, 1};
      const CUtensorMapSwizzle swz = bits == 3 ? CU_TENSOR_MAP_SWIZZLE_NONE
                                     : BK == 128 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
      if (enc(&tmP, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t*>(packed), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    }
    TcArgs a;
    a.steps = static_cast<const __half*>(steps);
    a.zeros = static_cast<const __half*>(zeros);
    a.Y = static_cast<__half*>(Y) + m0 * N;
    a.M = mc;
    a.N = (int)N;
    a.K = (int)K;
    a.BN = BN;
    a.err = err;
    a.spin_limit = (long long)wait_ms * 2000000LL;  // cycles at <= 2 GHz: at least wait_ms
    a.stall = stall ? 1 : 0;
    a.tmem_cols = t.tmem_cols;
    a.stages = S;
    // Dequantizing warp quartets: 1, or 2 when asked for 8 warps (stages
    // alternate between them; measured no faster) and the ring has at least 3
    // stages. A quartet publishes stage kt only once it holds stage kt + NH,
    // which needs the shared-memory slot that stage kt - S + NH frees: the ring
    // must be deeper than NH.
    const int NH = (dw_opt != 8 || S < 3) ? 1 : 2;
    const int tiles = (int)((N + kTcRows - 1) / kTcRows);
    const int KT_all = (int)(K / BK);
    a.units = (long long)tiles * KT_all;
    // Stream-K (one quartet, no cluster split): every CTA of a persistent grid
    // takes the same number of stages, whole tiles or not; at most one tile's
    // worth, so at most two segments, each with its own accumulator (with two
    // A buffers when three do not fit the same TMEM allocation beside them).
    const long long P = tc_streamk_ctas(t, tiles, KT_all);
    int NAk = NA;
    bool streamk = workspace != nullptr && workspace_bytes >= tc_streamk_bytes(t, P) && NH == 1 &&
                   ksplit_opt <= 1 && tiles <= (int)(kTcCounterBytes / 16) && (a.units + P - 1) / P <= KT_all &&
                   (streamk_opt == 2 || (streamk_opt == 0 && BN <= 16));
    if (streamk && pow2_cols((uint32_t)(2 * BN + NA * BK / 2)) > t.tmem_cols) {
      if (NA == 3 && pow2_cols((uint32_t)(2 * BN + 2 * BK / 2)) <= t.tmem_cols) NAk = 2;
      else streamk = false;
    }
    a.streamk = streamk ? 1 : 0;
    a.cnt = streamk ? static_cast<unsigned*>(workspace) : nullptr;
    a.part = streamk ? reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kTcCounterBytes) : nullptr;
    using I1 = std::integral_constant<int, 1>;
    using I2 = std::integral_constant<int, 2>;
    using I32 = std::integral_constant<int, 32>;
    using I64 = std::integral_constant<int, 64>;
    using I128 = std::integral_constant<int, 128>;
    auto pick_na = [&](auto bits_c, auto bk, auto nh, auto gs, auto sk) {
      constexpr int B = decltype(bits_c)::value, K_ = decltype(bk)::value, H = decltype(nh)::value,
                    S_ = decltype(gs)::value;
      constexpr bool SK_ = decltype(sk)::value;
      return NAk == 3 ? w4a16_gemm_tc_kernel<B, K_, H, 3, S_, SK_> : w4a16_gemm_tc_kernel<B, K_, H, 2, S_, SK_>;
    };
    using SKon = std::integral_constant<bool, true>;
    using SKoff = std::integral_constant<bool, false>;
    auto pick = [&](auto bits_c, auto bk, auto gs) {
      return streamk ? pick_na(bits_c, bk, I1{}, gs, SKon{})
                     : NH == 1 ? pick_na(bits_c, bk, I1{}, gs, SKoff{}) : pick_na(bits_c, bk, I2{}, gs, SKoff{});
    };
    using B3 = std::integral_constant<int, 3>;
    using B4 = std::integral_constant<int, 4>;
    decltype(pick(B4{}, I128{}, I128{})) kern;
    if (bits == 3)
      kern = group == 32 ? pick(B3{}, I128{}, I32{}) : group == 64 ? pick(B3{}, I128{}, I64{})
                                                                   : pick(B3{}, I128{}, I128{});
    else if (group == 32)
      kern = BK == 128 ? pick(B4{}, I128{}, I32{}) : pick(B4{}, I64{}, I32{});
    else if (group == 64)
      kern = BK == 128 ? pick(B4{}, I128{}, I64{}) : pick(B4{}, I64{}, I64{});
    else
      kern = BK == 128 ? pick(B4{}, I128{}, I128{}) : pick(B4{}, I64{}, I128{});
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)t.smem);
    if (e != cudaSuccess) return e;
    // Split K over a cluster while the row tiles leave SMs idle: double it
    // while twice the CTAs still fit one per SM (two CTAs sharing an SM run
    // no faster than one: 8192 x 8192 at M = 16 measured 31 us at 128 CTAs,
    // 34 us at 256), every CTA keeps at least 4 stages, and rank 0's ring
    // holds the other ranks' fp32 partial tiles.
    const size_t ring = (size_t)S * t.stage, part = (size_t)kTcRows * BN * 4;
    int ks = 1;
    if (!streamk) {
      if (ksplit_opt > 0) {
        ks = ksplit_opt;
        if ((size_t)(ks - 1) * part > ring || KT_all < ks) return cudaErrorInvalidValue;
      } else {
        const long slots = tc_num_sms();
        while (ks < 8 && (long)tiles * ks * 2 <= slots && KT_all / (ks * 2) >= 4 &&
               (size_t)(2 * ks - 1) * part <= ring)
          ks *= 2;
      }
    }
    a.ksplit = ks;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = streamk ? dim3((unsigned)P, 1, 1) : dim3((unsigned)tiles, (unsigned)ks, 1);
    cfg.blockDim = dim3(64 + 128 * NH, 1, 1);
    cfg.dynamicSmemBytes = t.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = (unsigned)ks;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = ks > 1 ? 1 : 0;
    e = cudaLaunchKernelEx(&cfg, kern, tmX, tmP, a);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace wq
