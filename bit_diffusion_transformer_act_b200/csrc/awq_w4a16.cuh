// Kernel 3: AWQ-style W4A16 linear, int4 weights with a bf16 scale and an
// integer zero point per (output row, group of 64 along K):
//
//   y[m, n] = sum_g s[n, g] * sum_{k in g} (q[n, k] - z[n, g]) x[m, k]  (+ b[n])
//
// Method: "Nunchaku Lite" docs, "Supported quantization types" (awq_w4a16 /
// int4 / group 64, an AWQ-style INT4 weight-only kernel); the Nunchaku Lite
// article: used for the adaptive-normalisation layers, activations stay 16-bit.
//
// Design (sm_100a, memory-bound).  Used for M <= 8 tokens (9..64 go to the tcgen05
// kernel, awq_umma.cuh).  A CTA owns 128 output rows and all tokens and streams its
// 128 x K/2 bytes of packed weights exactly once.  Warp 8 is the TMA producer: per
// 256-K stage one 128-row x 128-byte weight tile (128-byte swizzle) and the tokens'
// activations as four 64-column sub-tiles (128-byte swizzle, rows past M read as
// zeros), into a deep ring of stages (the activations are shared by every CTA and come
// from L2).  Warp 9 prepares each stage before the consumers see it: it reorders every
// 8-element activation unit to (k0,k4) (k1,k5) (k2,k6) (k3,k7) and sums each token's
// 64 activations of each group.  Warps 0-7 own 16 weight rows each and release a stage
// with one relaxed arrival per warp -- no block-wide barrier in the loop.  The weights
// are the A operand of mma.sync m16n8k16 (16 weight rows x 8 tokens), dequantized in
// registers: a nibble q becomes the bf16 128 + q by bit placement (exact).  A lane's
// 32-bit word of nibbles (one ldmatrix fetches the four words of a group) covers real K
// elements 8p..8p+7 of a 32-K step (p = lane % 4); with the reordered activations a pair
// of nibbles (p, p + 4) becomes a bf16x2 operand with one shift and one logic operation,
// the same K-slot permutation on both operands.  The zero point enters once per group:
// s (sum (128 + q) x - (128 + z) sum x).  Every product is exact and each group's fp32
// partial sum is scaled by s once.  Scales and zeros are read from global memory two
// stages ahead.  Every mbarrier wait is bounded.
#pragma once

#include "ptx.cuh"

namespace svdq {
namespace k3 {

constexpr int kRows = 128;                 // output rows (weight rows) per CTA
constexpr int kComputeWarps = 8;           // 16 weight rows each
constexpr int kChunk = 256;                // K per stage
constexpr int kGroup = 64;
constexpr int kWBytes = kRows * 128;       // 16 KB of packed weights per stage

constexpr int kXSub = 8 * 128;             // one 64-column activation sub-tile (8 tokens)
constexpr int kOffSx = kWBytes + 4 * kXSub;    // group sums: [4 groups][8 tokens] fp32
constexpr int kStage = (kOffSx + 4 * 8 * 4 + 1023) / 1024 * 1024;
constexpr int kStages = 5;                 // about 100 KB: two CTAs fit an SM (this launch's and the next's)
constexpr int kOffBar = kStages * kStage;
constexpr int kSmem = kOffBar + 8 * 3 * kStages + 16 + 1024;
constexpr int kProducer = kComputeWarps, kPrepWarp = kComputeWarps + 1;
constexpr int kThreads = (kComputeWarps + 2) * 32;
static_assert(kStage % 1024 == 0, "1 KB alignment of swizzled tiles");
static_assert(kSmem <= 113 * 1024, "two CTAs per SM");

struct Params {
  const __nv_bfloat16* scales;     // [N, K/64]
  const __nv_bfloat16* zeros;      // [N, K/64]
  const __nv_bfloat16* bias;       // [N] or null
  __nv_bfloat16* Y;                // [M, N]
  int M, N, K;
};

// bf16x2 {128 + nibble 0 of v, 128 + nibble 4 of v}: one three-input logic operation,
// (v & 0x000F000F) | magic, with magic = 0x43004300 held in a register (an instruction takes
// one immediate; with both constants immediate the compiler spends two operations).
__device__ __forceinline__ uint32_t nib04(uint32_t v, uint32_t magic) {
  uint32_t r;
  asm("lop3.b32 %0, %1, 0x000F000F, %2, 0xEA;" : "=r"(r) : "r"(v), "r"(magic));
  return r;
}

// D (16x8 fp32) = A (16x16 bf16, row) x B (16x8 bf16, col) + D, or + 0.  Not volatile:
// pure functions of their registers, so independent MMAs and loads may be interleaved.
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma16816_zero_c(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                                uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%10, %10, %10, %10};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.f));
}

// kVec: the scale and zero rows take 8-byte loads of four groups (K % 256 == 0, aligned rows)
template <bool kVec>
__global__ void __launch_bounds__(kThreads, 2)
awq_gemm_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX, const Params p) {
  constexpr int S = kStages;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t bars = base + kOffBar;
  auto full = [&](int s) { return bars + 8u * s; };
  auto empty = [&](int s) { return bars + 8u * (S + s); };
  auto ready = [&](int s) { return bars + 8u * (2 * S + s); };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + kOffBar + 24 * S);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int n0 = blockIdx.x * kRows;
  const int nkb = (p.K + kChunk - 1) / kChunk;     // the last stage may hold 1-3 groups (K % 64 == 0)

  if (warp == kProducer && lane == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), kComputeWarps);
      mbar_init(ready(s), 32);
    }
    *abort_flag = 0;
    abort_flag[1] = 0x43004300;                    // the dequantization constant, read back as a register
    fence_mbar_init();
    prefetch_tmap(&tmW);
    prefetch_tmap(&tmX);
  }
  __syncthreads();
  const int npre = min(S, nkb);                    // stages whose weight tiles load before the wait
  if (warp == kProducer && lane == 0) {
    // The weights, scales and zeros never come from the previous kernel: the first stages'
    // weight tiles are loaded while it finishes (with the kernel small enough for two CTAs per
    // SM, this CTA can be resident next to the previous kernel's), and this CTA's scale and
    // zero rows are pulled toward L2 (hints; L2 is coherent, so nothing stale can be read).
    for (int kb = 0; kb < npre; ++kb) {
      mbar_arrive_expect_tx(full(kb), kWBytes + 4 * kXSub);
      tma_load_2d(base + kb * kStage, &tmW, kb * (kChunk / 2), n0, full(kb));
    }
    const size_t rb = static_cast<size_t>(n0) * (p.K / kGroup) * 2;
    const uint32_t bytes = static_cast<uint32_t>(min(kRows, p.N - n0) * (p.K / kGroup) * 2);
    bulk_prefetch_l2_any(reinterpret_cast<const uint8_t*>(p.scales) + rb, bytes);
    bulk_prefetch_l2_any(reinterpret_cast<const uint8_t*>(p.zeros) + rb, bytes);
  }
  grid_dependency_wait();                          // X may belong to the previous kernel
  grid_launch_dependents();

  if (warp == kProducer) {
    // ---------------------------------------------------------------- TMA producer
    if (elect_one()) {
      // the activations of the stages whose weights are already on their way
      for (int kb = 0; kb < npre; ++kb)
#pragma unroll
        for (int j = 0; j < 4; ++j)
          tma_load_2d(base + kb * kStage + kWBytes + j * kXSub, &tmX, kb * kChunk + j * 64, 0, full(kb));
    }
    __syncwarp();
    for (int kb = npre; kb < nkb; ++kb) {
      const int s = kb % S;
      const uint32_t ph = (kb / S) & 1u;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(empty(s), ph ^ 1u, abort_flag, 21))) break;
      if (elect_one()) {
        const uint32_t sb = base + s * kStage;
        mbar_arrive_expect_tx(full(s), kWBytes + 4 * kXSub);
        tma_load_2d(sb, &tmW, kb * (kChunk / 2), n0, full(s));
#pragma unroll
        for (int j = 0; j < 4; ++j) tma_load_2d(sb + kWBytes + j * kXSub, &tmX, kb * kChunk + j * 64, 0, full(s));
      }
      __syncwarp();
    }
  } else if (warp == kPrepWarp) {
    // ---------------------------------------------------------------- activation reorder + group sums
    const int tok = lane & 7, grp = lane >> 3;     // this lane: token lane % 8 of group lane / 8
    for (int kb = 0; kb < nkb; ++kb) {
      const int s = kb % S;
      const uint32_t ph = (kb / S) & 1u;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(full(s), ph, abort_flag, 23))) break;
      uint8_t* st = gbase + s * kStage;
      uint8_t* row = st + kWBytes + grp * kXSub + tok * 128;
      // all eight units are loaded before the first store, so the loads overlap
      uint4 vu[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) vu[u] = *reinterpret_cast<const uint4*>(row + ((u ^ tok) << 4));
      float sum = 0.f;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const uint4 v = vu[u];
        const float a0 = bf16lo_to_f32(v.x) + bf16hi_to_f32(v.x), a1 = bf16lo_to_f32(v.y) + bf16hi_to_f32(v.y);
        const float a2 = bf16lo_to_f32(v.z) + bf16hi_to_f32(v.z), a3 = bf16lo_to_f32(v.w) + bf16hi_to_f32(v.w);
        sum += (a0 + a1) + (a2 + a3);
        uint4 n;
        asm("prmt.b32 %0, %1, %2, 0x5410;" : "=r"(n.x) : "r"(v.x), "r"(v.z));   // (k0, k4)
        asm("prmt.b32 %0, %1, %2, 0x7632;" : "=r"(n.y) : "r"(v.x), "r"(v.z));   // (k1, k5)
        asm("prmt.b32 %0, %1, %2, 0x5410;" : "=r"(n.z) : "r"(v.y), "r"(v.w));   // (k2, k6)
        asm("prmt.b32 %0, %1, %2, 0x7632;" : "=r"(n.w) : "r"(v.y), "r"(v.w));   // (k3, k7)
        *reinterpret_cast<uint4*>(row + ((u ^ tok) << 4)) = n;
      }
      reinterpret_cast<float*>(st + kOffSx)[grp * 8 + tok] = sum;
      fence_proxy_async_smem();                    // the next TMA into this stage comes after these stores
      mbar_arrive(ready(s));                       // release: this lane's stores are visible to the consumers
    }
  } else {
    // ---------------------------------------------------------------- dequantize + mma.sync
    const int g = lane >> 2, q = lane & 3;
    const uint32_t magic = static_cast<uint32_t>(abort_flag[1]);   // 0x43004300, opaque to the compiler
    float tot[4] = {0.f, 0.f, 0.f, 0.f};           // this lane's sums (D fragment layout)
    const int rg = warp * 16 + g;                  // this lane's weight rows: rg and rg + 8
    const int gpr = p.K / kGroup;                  // groups per weight row
    const int na = min(n0 + rg, p.N - 1), nb = min(n0 + rg + 8, p.N - 1);   // clamped for the loads
    // rows of scales and zero points; groups past K (a partial last stage) read as 0, and their
    // codes and activations are zero-filled by the copies, so they add nothing
    const uint16_t* sa = reinterpret_cast<const uint16_t*>(p.scales) + static_cast<size_t>(na) * gpr;
    const uint16_t* sb_ = reinterpret_cast<const uint16_t*>(p.scales) + static_cast<size_t>(nb) * gpr;
    const uint16_t* za = reinterpret_cast<const uint16_t*>(p.zeros) + static_cast<size_t>(na) * gpr;
    const uint16_t* zb = reinterpret_cast<const uint16_t*>(p.zeros) + static_cast<size_t>(nb) * gpr;
    constexpr bool vec = kVec;
    // ldmatrix: this lane's row address (matrices: rows 0-7 / 8-15 of the slice, 32-K steps 2 grp / 2 grp + 1)
    const int lrow = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
    uint32_t woff[4];
#pragma unroll
    for (int grp = 0; grp < 4; ++grp)
      woff[grp] = static_cast<uint32_t>(lrow * 128) +
                  ((static_cast<uint32_t>(2 * grp + (lane >> 4)) ^ static_cast<uint32_t>(lane & 7)) << 4);
    // activation unit of this lane in a sub-tile (token row g), per 32-K step
    const uint32_t xoff0 = static_cast<uint32_t>(g * 128) + ((static_cast<uint32_t>(q) ^ static_cast<uint32_t>(g)) << 4);
    const uint32_t xoff1 = static_cast<uint32_t>(g * 128) + ((static_cast<uint32_t>(4 + q) ^ static_cast<uint32_t>(g)) << 4);

    // scales and zeros of the 4 groups of a stage (8 bytes per row), two stages ahead
    uint2 pa[4], pb[4];
    {
      const int k1 = min(1, nkb - 1);
      pa[0] = ld_groups4(sa, 0, gpr, vec); pa[1] = ld_groups4(sb_, 0, gpr, vec);
      pa[2] = ld_groups4(za, 0, gpr, vec); pa[3] = ld_groups4(zb, 0, gpr, vec);
      pb[0] = ld_groups4(sa, k1, gpr, vec); pb[1] = ld_groups4(sb_, k1, gpr, vec);
      pb[2] = ld_groups4(za, k1, gpr, vec); pb[3] = ld_groups4(zb, k1, gpr, vec);
    }
    for (int kb = 0; kb < nkb; ++kb) {
      const int s = kb % S;
      const uint32_t ph = (kb / S) & 1u;
      const uint2 cur[4] = {pa[0], pa[1], pa[2], pa[3]};
#pragma unroll
      for (int t = 0; t < 4; ++t) pa[t] = pb[t];
      {
        const int kk = min(kb + 2, nkb - 1);
        pb[0] = ld_groups4(sa, kk, gpr, vec); pb[1] = ld_groups4(sb_, kk, gpr, vec);
        pb[2] = ld_groups4(za, kk, gpr, vec); pb[3] = ld_groups4(zb, kk, gpr, vec);
      }
      if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(ready(s), ph, abort_flag, 22))) break;
      const uint32_t wst = base + s * kStage;
      const float* sxs = reinterpret_cast<const float*>(gbase + s * kStage + kOffSx);
      // every shared-memory operand of the stage first (the loads are issued back to back), then
      // the four groups' MMAs as eight independent two-MMA chains, so that their latencies overlap
      uint32_t wq[4][4];                           // per group: {row g, row g+8} x {32-K step 0, 1}
      uint32_t xv[4][2][4];                        // per group and 32-K step: this lane's activation unit
#pragma unroll
      for (int grp = 0; grp < 4; ++grp) {
        ldmatrix_x4(wst + woff[grp], wq[grp][0], wq[grp][1], wq[grp][2], wq[grp][3]);
#pragma unroll
        for (int half = 0; half < 2; ++half)
          asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(xv[grp][half][0]), "=r"(xv[grp][half][1]), "=r"(xv[grp][half][2]), "=r"(xv[grp][half][3])
                       : "r"(wst + kWBytes + grp * kXSub + (half ? xoff1 : xoff0)));
      }
      float gp[4][2][4];
#pragma unroll
      for (int grp = 0; grp < 4; ++grp) {
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          // nibbles (p, p + 4) -> K slot pairs; the activations were reordered to match
          const uint32_t wg = wq[grp][2 * half], wh = wq[grp][2 * half + 1];
          const uint32_t wg4 = wg >> 4, wh4 = wh >> 4;
          const uint32_t(&x)[4] = xv[grp][half];
          mma16816_zero_c(gp[grp][half], nib04(wg, magic), nib04(wh, magic), nib04(wg4, magic), nib04(wh4, magic),
                          x[0], x[1]);
          mma16816(gp[grp][half], nib04(wg >> 8, magic), nib04(wh >> 8, magic), nib04(wg4 >> 8, magic),
                   nib04(wh4 >> 8, magic), x[2], x[3]);
        }
      }
#pragma unroll
      for (int grp = 0; grp < 4; ++grp) {
        const uint32_t w0 = grp < 2 ? cur[0].x : cur[0].y, w1 = grp < 2 ? cur[1].x : cur[1].y;
        const uint32_t w2 = grp < 2 ? cur[2].x : cur[2].y, w3 = grp < 2 ? cur[3].x : cur[3].y;
        const float sg = (grp & 1) ? bf16hi_to_f32(w0) : bf16lo_to_f32(w0);
        const float sh = (grp & 1) ? bf16hi_to_f32(w1) : bf16lo_to_f32(w1);
        const float zg = ((grp & 1) ? bf16hi_to_f32(w2) : bf16lo_to_f32(w2)) + 128.f;
        const float zh = ((grp & 1) ? bf16hi_to_f32(w3) : bf16lo_to_f32(w3)) + 128.f;
        // the group's exact integer-weighted sums (each half's fp32 sum of 32 exact products)
        float ga[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) ga[e] = gp[grp][0][e] + gp[grp][1][e];
        // D fragment: c0 (row g, token 2q), c1 (row g, token 2q+1), c2/c3 the same for row g+8
        const float2 sx = *reinterpret_cast<const float2*>(sxs + grp * 8 + 2 * q);
        tot[0] = fmaf(sg, fmaf(-zg, sx.x, ga[0]), tot[0]);
        tot[1] = fmaf(sg, fmaf(-zg, sx.y, ga[1]), tot[1]);
        tot[2] = fmaf(sh, fmaf(-zh, sx.x, ga[2]), tot[2]);
        tot[3] = fmaf(sh, fmaf(-zh, sx.y, ga[3]), tot[3]);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive_relaxed(empty(s));   // this warp is done with the stage
    }

    const int ra = n0 + rg, rb = ra + 8;
    const float ba = (p.bias && ra < p.N) ? __bfloat162float(p.bias[ra]) : 0.f;
    const float bb = (p.bias && rb < p.N) ? __bfloat162float(p.bias[rb]) : 0.f;
    const int t0 = 2 * q, t1 = t0 + 1;
    if (t0 < p.M) {
      if (ra < p.N) p.Y[static_cast<size_t>(t0) * p.N + ra] = __float2bfloat16_rn(tot[0] + ba);
      if (rb < p.N) p.Y[static_cast<size_t>(t0) * p.N + rb] = __float2bfloat16_rn(tot[2] + bb);
    }
    if (t1 < p.M) {
      if (ra < p.N) p.Y[static_cast<size_t>(t1) * p.N + ra] = __float2bfloat16_rn(tot[1] + ba);
      if (rb < p.N) p.Y[static_cast<size_t>(t1) * p.N + rb] = __float2bfloat16_rn(tot[3] + bb);
    }
  }
  __syncthreads();
  if (*abort_flag && warp == kProducer && lane == 0) {
    // a wait ran out: let the copies already issued land before shared memory goes away
    const uint64_t t0 = global_timer_ns();
    while (global_timer_ns() - t0 < 2000000ull) { }
  }
}

}  // namespace k3
}  // namespace svdq
