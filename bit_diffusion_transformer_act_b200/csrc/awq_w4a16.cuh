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
// kernel, awq_umma.cuh).  A CTA (one per SM) owns 128 output rows and all tokens and
// streams its 128 x K/2 bytes of packed weights exactly once.  Warp 16 is the TMA producer:
// after the first weight tile, the CTA's scale and zero rows into shared memory (when
// K % 512 == 0 and K <= 4096; else the consumers read them from global memory), then per
// 256-K stage one 128-row x
// 128-byte weight tile (128-byte swizzle) and the tokens' activations as four 64-column
// sub-tiles (128-byte swizzle, rows past M read as zeros; the activations are shared by every
// CTA and come from L2), paced: stage kb is requested once stage kb - 3 has landed (with every
// CTA's whole ring requested at once, the memory system serves them all interleaved and a
// CTA's first tile lands late).  Warps 17 and 18 prepare the even and odd stages before the
// consumers see them: they reorder every 8-element activation unit to (k0,k4) (k1,k5) (k2,k6)
// (k3,k7) and sum each token's 64 activations of each group.  Warps 0-15 are the consumers,
// two per 16 weight rows: warp w takes the even stages and w + 8 the odd ones, each releasing
// a stage with one relaxed arrival (no block-wide barrier in the loop), and at the end the odd
// warp's sums are added to the even warp's (a fixed order).  The weights are the A operand of
// mma.sync m16n8k16 (16 weight rows x 8 tokens), dequantized in registers: a nibble q becomes
// the bf16 128 + q by bit placement (exact).  A lane's 32-bit word of nibbles (one ldmatrix
// fetches the four words of a group) covers real K elements 8p..8p+7 of a 32-K step
// (p = lane % 4); with the reordered activations a pair of nibbles (p, p + 4) becomes a
// bf16x2 operand with one shift and one logic operation, the same K-slot permutation on both
// operands.  The zero point enters once per group: s (sum (128 + q) x - (128 + z) sum x).
// Every product is exact and each group's fp32 partial sum is scaled by s once.  Every
// mbarrier wait is bounded.
#pragma once

#include "ptx.cuh"

namespace svdq {
namespace k3 {

constexpr int kRows = 128;                 // output rows (weight rows) per CTA
constexpr int kSlices = 8;                 // 16 weight rows each
constexpr int kComputeWarps = 2 * kSlices; // two per row slice: even and odd stages
constexpr int kChunk = 256;                // K per stage
constexpr int kGroup = 64;
constexpr int kWBytes = kRows * 128;       // 16 KB of packed weights per stage

constexpr int kXSub = 8 * 128;             // one 64-column activation sub-tile (8 tokens)
constexpr int kOffSx = kWBytes + 4 * kXSub;    // group sums: [4 groups][8 tokens] fp32
constexpr int kStage = (kOffSx + 4 * 8 * 4 + 1023) / 1024 * 1024;
constexpr int kStages = 9;
constexpr int kPace = 3;                   // stage kb is requested once stage kb - kPace has landed
static_assert(kPace >= 1 && kPace < kStages, "pacing distance within the ring");
constexpr int kMaxSzGroups = 64;           // K <= 4096: the CTA's scale and zero rows held in shared memory
constexpr int kOffSz = kStages * kStage;   // [scales, zeros][128 rows][K / 64 groups] bf16
constexpr int kOffRed = kOffSz + 2 * kRows * kMaxSzGroups * 2;   // odd-stage sums: [8 slices][32 lanes][4] fp32
constexpr int kOffBar = kOffRed + kSlices * 32 * 16;
constexpr int kSmem = kOffBar + 8 * (3 * kStages + 1) + 16 + 1024;
constexpr int kProducer = kComputeWarps, kPrepWarp = kComputeWarps + 1;   // prep warps: even and odd stages
constexpr int kThreads = (kComputeWarps + 3) * 32;
static_assert(kStage % 1024 == 0, "1 KB alignment of swizzled tiles");
static_assert(kSmem <= 227 * 1024, "one CTA per SM");


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

// kSz: the CTA's scale and zero rows are copied into shared memory once, before the grid-dependency
// wait (tmS / tmZ: [N, K/64] bf16, box K/64 x 128; K % 512 == 0, K <= 4096, 16-byte aligned);
// otherwise the consumers read them from global memory two of their stages ahead, with 8-byte
// loads of four groups when kVec (K % 256 == 0, aligned rows).
template <bool kVec, bool kSz>
__global__ void __launch_bounds__(kThreads, 1)
awq_gemm_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                const __grid_constant__ CUtensorMap tmS, const __grid_constant__ CUtensorMap tmZ, const Params p) {
  constexpr int S = kStages;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t bars = base + kOffBar;
  auto full = [&](int s) { return bars + 8u * s; };
  auto empty = [&](int s) { return bars + 8u * (S + s); };
  auto ready = [&](int s) { return bars + 8u * (2 * S + s); };
  const uint32_t sz_bar = bars + 8u * (3 * S);     // the scale and zero rows have landed
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + kOffBar + 8 * (3 * S + 1));

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int n0 = blockIdx.x * kRows;
  const int nkb = (p.K + kChunk - 1) / kChunk;     // the last stage may hold 1-3 groups (K % 64 == 0)

  if (warp == kProducer && lane == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), kSlices);
      mbar_init(ready(s), 32);
    }
    mbar_init(sz_bar, 1);
    *abort_flag = 0;
    abort_flag[1] = 0x43004300;                    // the dequantization constant, read back as a register
    fence_mbar_init();
    prefetch_tmap(&tmW);
    prefetch_tmap(&tmX);
    if (kSz) {
      prefetch_tmap(&tmS);
      prefetch_tmap(&tmZ);
    }
  }
  __syncthreads();
  const int npre = min(kPace, nkb);                // stages whose weight tiles load before the wait
  if (warp == kProducer && lane == 0) {
    // The weights, scales and zeros never come from the previous kernel: they are requested
    // before the grid-dependency wait -- the first weight tile, the CTA's scale and zero rows
    // (every stage's epilogue needs them), copied into shared memory or pulled toward L2 (hints;
    // L2 is coherent, so nothing stale can be read), then the next weight tiles.
    auto load_w = [&](int kb) {
      mbar_arrive_expect_tx(full(kb), kWBytes + 4 * kXSub);
      tma_load_2d(base + kb * kStage, &tmW, kb * (kChunk / 2), n0, full(kb));
    };
    if (npre > 0) load_w(0);
    if (kSz) {
      const int gpr = p.K / kGroup;
      mbar_arrive_expect_tx(sz_bar, 2u * kRows * gpr * 2);
      tma_load_2d(base + kOffSz, &tmS, 0, n0, sz_bar);
      tma_load_2d(base + kOffSz + kRows * kMaxSzGroups * 2, &tmZ, 0, n0, sz_bar);
    } else {
      const size_t rb = static_cast<size_t>(n0) * (p.K / kGroup) * 2;
      const uint32_t bytes = static_cast<uint32_t>(min(kRows, p.N - n0) * (p.K / kGroup) * 2);
      bulk_prefetch_l2_any(reinterpret_cast<const uint8_t*>(p.scales) + rb, bytes);
      bulk_prefetch_l2_any(reinterpret_cast<const uint8_t*>(p.zeros) + rb, bytes);
    }
    for (int kb = 1; kb < npre; ++kb) load_w(kb);
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
      // paced: with every CTA's whole ring requested at once the memory system serves all of
      // them interleaved and each CTA's first tile lands late; kPace tiles ahead per CTA keep
      // the stream at full rate and let the consumers start early
      const int kp = kb - kPace;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(full(kp % S), (kp / S) & 1u, abort_flag, 25))) break;
      if (elect_one()) {
        const uint32_t sb = base + s * kStage;
        mbar_arrive_expect_tx(full(s), kWBytes + 4 * kXSub);
        tma_load_2d(sb, &tmW, kb * (kChunk / 2), n0, full(s));
#pragma unroll
        for (int j = 0; j < 4; ++j) tma_load_2d(sb + kWBytes + j * kXSub, &tmX, kb * kChunk + j * 64, 0, full(s));
      }
      __syncwarp();
    }
  } else if (warp >= kPrepWarp) {
    // ---------------------------------------------------------------- activation reorder + group sums
    const int tok = lane & 7, grp = lane >> 3;     // this lane: token lane % 8 of group lane / 8
    for (int kb = warp - kPrepWarp; kb < nkb; kb += 2) {
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
    const int slice = warp % kSlices, par = warp / kSlices;   // this warp: row slice, stage parity
    const uint32_t magic = static_cast<uint32_t>(abort_flag[1]);   // 0x43004300, opaque to the compiler
    float tot[4] = {0.f, 0.f, 0.f, 0.f};           // this lane's sums (D fragment layout)
    const int rg = slice * 16 + g;                 // this lane's weight rows: rg and rg + 8
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
    const int lrow = slice * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
    uint32_t woff[4];
#pragma unroll
    for (int grp = 0; grp < 4; ++grp)
      woff[grp] = static_cast<uint32_t>(lrow * 128) +
                  ((static_cast<uint32_t>(2 * grp + (lane >> 4)) ^ static_cast<uint32_t>(lane & 7)) << 4);
    // activation unit of this lane in a sub-tile (token row g), per 32-K step
    const uint32_t xoff0 = static_cast<uint32_t>(g * 128) + ((static_cast<uint32_t>(q) ^ static_cast<uint32_t>(g)) << 4);
    const uint32_t xoff1 = static_cast<uint32_t>(g * 128) + ((static_cast<uint32_t>(4 + q) ^ static_cast<uint32_t>(g)) << 4);

    // scales and zeros of the 4 groups of a stage (8 bytes per row): from shared memory, or from
    // global memory two of this warp's stages ahead
    uint2 pa[4], pb[4];
    if constexpr (!kSz) {
      const int k0 = min(par, nkb - 1), k1 = min(par + 2, nkb - 1);
      pa[0] = ld_groups4(sa, k0, gpr, vec); pa[1] = ld_groups4(sb_, k0, gpr, vec);
      pa[2] = ld_groups4(za, k0, gpr, vec); pa[3] = ld_groups4(zb, k0, gpr, vec);
      pb[0] = ld_groups4(sa, k1, gpr, vec); pb[1] = ld_groups4(sb_, k1, gpr, vec);
      pb[2] = ld_groups4(za, k1, gpr, vec); pb[3] = ld_groups4(zb, k1, gpr, vec);
    }
    bool sz_ok = true;
    if constexpr (kSz) sz_ok = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(sz_bar, 0, abort_flag, 24));
    const uint8_t* sz_s = gbase + kOffSz + static_cast<size_t>(rg) * gpr * 2;   // row rg; rg + 8 at + 8 gpr
    const uint8_t* sz_z = sz_s + kRows * kMaxSzGroups * 2;
    for (int kb = par; sz_ok && kb < nkb; kb += 2) {
      const int s = kb % S;
      const uint32_t ph = (kb / S) & 1u;
      uint2 cur[4];
      if constexpr (kSz) {
        cur[0] = *reinterpret_cast<const uint2*>(sz_s + kb * 8);
        cur[1] = *reinterpret_cast<const uint2*>(sz_s + 16 * gpr + kb * 8);
        cur[2] = *reinterpret_cast<const uint2*>(sz_z + kb * 8);
        cur[3] = *reinterpret_cast<const uint2*>(sz_z + 16 * gpr + kb * 8);
      } else {
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          cur[t] = pa[t];
          pa[t] = pb[t];
        }
        const int kk = min(kb + 4, nkb - 1);
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
      float gp[4][4];                              // per group: one chain of four MMAs
#pragma unroll
      for (int half = 0; half < 2; ++half) {
#pragma unroll
        for (int grp = 0; grp < 4; ++grp) {
          // nibbles (p, p + 4) -> K slot pairs; the activations were reordered to match
          const uint32_t wg = wq[grp][2 * half], wh = wq[grp][2 * half + 1];
          const uint32_t wg4 = wg >> 4, wh4 = wh >> 4;
          const uint32_t(&x)[4] = xv[grp][half];
          if (half == 0)
            mma16816_zero_c(gp[grp], nib04(wg, magic), nib04(wh, magic), nib04(wg4, magic), nib04(wh4, magic),
                            x[0], x[1]);
          else
            mma16816(gp[grp], nib04(wg, magic), nib04(wh, magic), nib04(wg4, magic), nib04(wh4, magic), x[0], x[1]);
          mma16816(gp[grp], nib04(wg >> 8, magic), nib04(wh >> 8, magic), nib04(wg4 >> 8, magic),
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
        // the group's integer-weighted sums (fp32 sums of 64 exact products)
        const float(&ga)[4] = gp[grp];
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

    // the odd-stage warp hands its sums to the even-stage warp of its slice, which adds them
    // (even + odd: a fixed order) and stores
    float4* red = reinterpret_cast<float4*>(gbase + kOffRed) + slice * 32 + lane;
    if (par == 1) *red = make_float4(tot[0], tot[1], tot[2], tot[3]);
    asm volatile("bar.sync 1, %0;" ::"n"(kComputeWarps * 32) : "memory");   // consumer warps only
    if (par == 0) {
      const float4 o = *red;
      tot[0] += o.x;
      tot[1] += o.y;
      tot[2] += o.z;
      tot[3] += o.w;
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
