// Kernel 3: AWQ-style W4A16 linear, int4 weights with a bf16 scale and an
// integer zero point per (output row, group of 64 along K):
//
//   y[m, n] = sum_g s[n, g] * sum_{k in g} (q[n, k] - z[n, g]) x[m, k]  (+ b[n])
//
// Method: "Nunchaku Lite" docs, "Supported quantization types" (awq_w4a16 /
// int4 / group 64, an AWQ-style INT4 weight-only kernel); the Nunchaku Lite
// article: used for the adaptive-normalisation layers, activations stay 16-bit.
//
// Design (sm_100a, memory-bound at small M).  A CTA owns 128 output rows and all
// M <= 64 tokens and streams its 128 x K/2 bytes of packed weights exactly once.
// Warp 8 is the TMA producer: per 256-K stage one 128-row x 128-byte weight tile
// (128-byte swizzle) and the tokens' activations as four 64-column sub-tiles
// (128-byte swizzle, rows past M read as zeros), into a deep ring of stages (the
// activations are shared by every CTA and come from L2).  Warps 0-7 own 16
// weight rows each; per stage they wait on the stage's barrier, and release it
// with one arrival per warp -- no block-wide barrier.  The weights are the A
// operand of mma.sync m16n8k16 (16 weight rows x 8 tokens), dequantized in
// registers: a nibble q becomes the bf16 128 + q by bit placement (exact).
// Inside every 32-K step the K order is permuted (the same permutation for A and
// B): lane quad position p takes real K elements 8p..8p+7, i.e. one 32-bit word
// of nibbles per weight row and one 16-byte load of activations per token tile.
// The zero point:
//   * M <= 8: sum_k (128 + q) x is accumulated as is and corrected per group,
//       s (sum (128 + q) x - (128 + z) sum x); sum x comes from a second MMA with
//       an all-ones A operand on the same activation fragment, so no per-weight
//       subtraction is needed.
//   * M > 8: one packed bf16 subtraction of 128 + z gives q - z exactly.
// Either way every product is exact and each group's fp32 partial sum is scaled
// by s once.  Scales and zeros are read from global memory one stage ahead.
// Every mbarrier wait is bounded.
#pragma once

#include "ptx.cuh"

namespace svdq {
namespace k3 {

constexpr int kRows = 128;                 // output rows (weight rows) per CTA
constexpr int kComputeWarps = 8;           // 16 weight rows each
constexpr int kThreads = (kComputeWarps + 1) * 32;
constexpr int kChunk = 256;                // K per stage
constexpr int kGroup = 64;
constexpr int kWBytes = kRows * 128;       // 16 KB of packed weights per stage

template <int NT>
struct Cfg {
  static constexpr int XSUB = NT * 8 * 128;                 // one 64-column activation sub-tile
  static constexpr int STAGE = kWBytes + 4 * XSUB;
  static constexpr int STAGES = NT == 1 ? 10 : (NT == 2 ? 8 : (NT == 4 ? 6 : 4));
  static constexpr int OFF_BAR = STAGES * STAGE;
  static constexpr int SMEM = OFF_BAR + 8 * 2 * STAGES + 16 + 1024;
  static_assert(STAGE % 1024 == 0, "1 KB alignment of swizzled tiles");
  static_assert(SMEM <= 227 * 1024, "shared memory");
};

struct Params {
  const __nv_bfloat16* scales;     // [N, K/64]
  const __nv_bfloat16* zeros;      // [N, K/64]
  const __nv_bfloat16* bias;       // [N] or null
  __nv_bfloat16* Y;                // [M, N]
  int M, N, K;
};

// bf16x2 {128 + low nibble of byte b of w, 128 + high nibble of byte b of w};
// sel picks byte b of w into byte 0 and byte b of w >> 4 into byte 2.
__device__ __forceinline__ uint32_t nib_pair(uint32_t w, uint32_t w4, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(w), "r"(w4), "r"(sel));
  return (r & 0x000F000Fu) | 0x43004300u;
}

__device__ __forceinline__ uint32_t bf16x2_sub(uint32_t a, uint32_t b) {
  __nv_bfloat162 r = __hsub2(*reinterpret_cast<__nv_bfloat162*>(&a), *reinterpret_cast<__nv_bfloat162*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}

template <int NT>
__global__ void __launch_bounds__(kThreads, 1)
awq_gemm_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX, const Params p) {
  using C = Cfg<NT>;
  constexpr int S = C::STAGES;
  constexpr bool kSumX = NT == 1;                  // zero point through sum x (see above)
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t bars = base + C::OFF_BAR;
  auto full = [&](int s) { return bars + 8u * s; };
  auto empty = [&](int s) { return bars + 8u * (S + s); };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + C::OFF_BAR + 16 * S);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int n0 = blockIdx.x * kRows;
  const int nkb = p.K / kChunk;

  if (warp == kComputeWarps && lane == 0) {
    for (int s = 0; s < S; ++s) { mbar_init(full(s), 1); mbar_init(empty(s), kComputeWarps); }
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmW);
    prefetch_tmap(&tmX);
  }
  __syncthreads();
  grid_dependency_wait();                          // X may belong to the previous kernel
  grid_launch_dependents();

  if (warp == kComputeWarps) {
    // ---------------------------------------------------------------- TMA producer
    for (int kb = 0; kb < nkb; ++kb) {
      const int s = kb % S;
      const uint32_t ph = (kb / S) & 1u;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(empty(s), ph ^ 1u, abort_flag, 21))) break;
      if (elect_one()) {
        const uint32_t sb = base + s * C::STAGE;
        mbar_arrive_expect_tx(full(s), C::STAGE);
        tma_load_2d(sb, &tmW, kb * (kChunk / 2), n0, full(s));
#pragma unroll
        for (int j = 0; j < 4; ++j) tma_load_2d(sb + kWBytes + j * C::XSUB, &tmX, kb * kChunk + j * 64, 0, full(s));
      }
      __syncwarp();
    }
  } else {
    // ---------------------------------------------------------------- dequantize + mma.sync
    const int g = lane >> 2, q = lane & 3;
    const int rg = warp * 16 + g;                  // this lane's weight rows: rg and rg + 8
    const uint32_t sw = static_cast<uint32_t>(rg & 7);   // (rg + 8) & 7 is the same
    const int gpr = p.K / kGroup;                  // groups per weight row
    const int na = min(n0 + rg, p.N - 1), nb = min(n0 + rg + 8, p.N - 1);   // clamped for the loads
    const uint2* sa = reinterpret_cast<const uint2*>(p.scales + static_cast<size_t>(na) * gpr);
    const uint2* sb_ = reinterpret_cast<const uint2*>(p.scales + static_cast<size_t>(nb) * gpr);
    const uint2* za = reinterpret_cast<const uint2*>(p.zeros + static_cast<size_t>(na) * gpr);
    const uint2* zb = reinterpret_cast<const uint2*>(p.zeros + static_cast<size_t>(nb) * gpr);
    constexpr uint32_t kOnes = 0x3F803F80u;        // bf16x2 {1, 1}

    float tot[NT][4];
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
      for (int t = 0; t < 4; ++t) tot[j][t] = 0.f;

    // scales and zeros of the 4 groups of a stage: 8 bytes per row, one stage ahead
    uint2 s_a = __ldg(sa), s_b = __ldg(sb_), z_a = __ldg(za), z_b = __ldg(zb);
    for (int kb = 0; kb < nkb; ++kb) {
      const int s = kb % S;
      const uint32_t ph = (kb / S) & 1u;
      const uint2 cs_a = s_a, cs_b = s_b, cz_a = z_a, cz_b = z_b;
      if (kb + 1 < nkb) {
        s_a = __ldg(sa + kb + 1); s_b = __ldg(sb_ + kb + 1);
        z_a = __ldg(za + kb + 1); z_b = __ldg(zb + kb + 1);
      }
      if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(full(s), ph, abort_flag, 22))) break;
      const uint32_t wst = base + s * C::STAGE;
      const uint32_t xst = wst + kWBytes;
      const uint32_t wrow_g = wst + rg * 128 + 4 * q;
      const uint32_t wrow_h = wrow_g + 8 * 128;
#pragma unroll
      for (int grp = 0; grp < 4; ++grp) {
        const uint32_t sw2a = grp < 2 ? cs_a.x : cs_a.y, sw2b = grp < 2 ? cs_b.x : cs_b.y;
        const uint32_t zw2a = grp < 2 ? cz_a.x : cz_a.y, zw2b = grp < 2 ? cz_b.x : cz_b.y;
        const float sg = (grp & 1) ? bf16hi_to_f32(sw2a) : bf16lo_to_f32(sw2a);
        const float sh = (grp & 1) ? bf16hi_to_f32(sw2b) : bf16lo_to_f32(sw2b);
        const float zg = ((grp & 1) ? bf16hi_to_f32(zw2a) : bf16lo_to_f32(zw2a)) + 128.f;
        const float zh = ((grp & 1) ? bf16hi_to_f32(zw2b) : bf16lo_to_f32(zw2b)) + 128.f;

        float ga[NT][4];
        float sx[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int j = 0; j < NT; ++j)
#pragma unroll
          for (int t = 0; t < 4; ++t) ga[j][t] = 0.f;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const uint32_t t32 = static_cast<uint32_t>(grp * 2 + half);   // 32-K step: 16-byte unit of a row
          uint32_t wg, wh;
          asm volatile("ld.shared.b32 %0, [%1];" : "=r"(wg) : "r"(wrow_g + ((t32 ^ sw) << 4)));
          asm volatile("ld.shared.b32 %0, [%1];" : "=r"(wh) : "r"(wrow_h + ((t32 ^ sw) << 4)));
          const uint32_t wg4 = wg >> 4, wh4 = wh >> 4;
          // pair b (real K elements 8q + 2b, 8q + 2b + 1) = byte b of w (low and high nibble)
          uint32_t A[2][4];
#pragma unroll
          for (int ks = 0; ks < 2; ++ks) {
            const uint32_t sel0 = static_cast<uint32_t>(2 * ks) | (static_cast<uint32_t>(4 + 2 * ks) << 8);
            const uint32_t sel1 = static_cast<uint32_t>(2 * ks + 1) | (static_cast<uint32_t>(5 + 2 * ks) << 8);
            A[ks][0] = nib_pair(wg, wg4, sel0);   // row g,   logical k 2q, 2q+1
            A[ks][1] = nib_pair(wh, wh4, sel0);   // row g+8
            A[ks][2] = nib_pair(wg, wg4, sel1);   // row g,   logical k 2q+8, 2q+9
            A[ks][3] = nib_pair(wh, wh4, sel1);
            if (!kSumX) {
              const uint32_t zzg = pack_bf16x2(zg, zg), zzh = pack_bf16x2(zh, zh);
              A[ks][0] = bf16x2_sub(A[ks][0], zzg);
              A[ks][1] = bf16x2_sub(A[ks][1], zzh);
              A[ks][2] = bf16x2_sub(A[ks][2], zzg);
              A[ks][3] = bf16x2_sub(A[ks][3], zzh);
            }
          }
          const uint32_t xsub = xst + (t32 >> 1) * C::XSUB;          // 64-column sub-tile
          const uint32_t unit = (t32 & 1u) * 4u + static_cast<uint32_t>(q);
#pragma unroll
          for (int j = 0; j < NT; ++j) {
            const int tr = 8 * j + g;                                 // token row
            uint32_t x0, x1, x2, x3;
            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(x0), "=r"(x1), "=r"(x2), "=r"(x3)
                         : "r"(xsub + tr * 128 + ((unit ^ static_cast<uint32_t>(tr & 7)) << 4)));
            mma_bf16_16816(ga[j], A[0][0], A[0][1], A[0][2], A[0][3], x0, x1);
            mma_bf16_16816(ga[j], A[1][0], A[1][1], A[1][2], A[1][3], x2, x3);
            if (kSumX) {
              mma_bf16_16816(sx, kOnes, kOnes, kOnes, kOnes, x0, x1);
              mma_bf16_16816(sx, kOnes, kOnes, kOnes, kOnes, x2, x3);
            }
          }
        }
        // D fragment: c0 (row g, token 2q), c1 (row g, token 2q+1), c2/c3 the same for row g+8
#pragma unroll
        for (int j = 0; j < NT; ++j) {
          if (kSumX) {
            tot[j][0] = fmaf(sg, fmaf(-zg, sx[0], ga[j][0]), tot[j][0]);
            tot[j][1] = fmaf(sg, fmaf(-zg, sx[1], ga[j][1]), tot[j][1]);
            tot[j][2] = fmaf(sh, fmaf(-zh, sx[2], ga[j][2]), tot[j][2]);
            tot[j][3] = fmaf(sh, fmaf(-zh, sx[3], ga[j][3]), tot[j][3]);
          } else {
            tot[j][0] = fmaf(sg, ga[j][0], tot[j][0]);
            tot[j][1] = fmaf(sg, ga[j][1], tot[j][1]);
            tot[j][2] = fmaf(sh, ga[j][2], tot[j][2]);
            tot[j][3] = fmaf(sh, ga[j][3], tot[j][3]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive_relaxed(empty(s));   // this warp is done with the stage
    }

    const int ra = n0 + rg, rb = ra + 8;
    const float ba = (p.bias && ra < p.N) ? __bfloat162float(p.bias[ra]) : 0.f;
    const float bb = (p.bias && rb < p.N) ? __bfloat162float(p.bias[rb]) : 0.f;
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      const int t0 = 8 * j + 2 * q, t1 = t0 + 1;
      if (t0 < p.M) {
        if (ra < p.N) p.Y[static_cast<size_t>(t0) * p.N + ra] = __float2bfloat16_rn(tot[j][0] + ba);
        if (rb < p.N) p.Y[static_cast<size_t>(t0) * p.N + rb] = __float2bfloat16_rn(tot[j][2] + bb);
      }
      if (t1 < p.M) {
        if (ra < p.N) p.Y[static_cast<size_t>(t1) * p.N + ra] = __float2bfloat16_rn(tot[j][1] + ba);
        if (rb < p.N) p.Y[static_cast<size_t>(t1) * p.N + rb] = __float2bfloat16_rn(tot[j][3] + bb);
      }
    }
  }
  __syncthreads();
  if (*abort_flag && warp == kComputeWarps && lane == 0) {
    // a wait ran out: let the copies already issued land before shared memory goes away
    const uint64_t t0 = global_timer_ns();
    while (global_timer_ns() - t0 < 2000000ull) { }
  }
}

}  // namespace k3
}  // namespace svdq
