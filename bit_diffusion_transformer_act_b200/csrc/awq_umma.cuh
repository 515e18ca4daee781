// Kernel 4: AWQ-style W4A16 linear for 9 <= M <= 64 tokens on the tcgen05 tensor
// cores.  Same arithmetic as kernel 3 (awq_w4a16.cuh):
//
//   y[m, n] = sum_g s[n, g] * sum_{k in g} (q[n, k] - z[n, g]) x[m, k]  (+ b[n])
//
// Method: "Nunchaku Lite" docs, "Supported quantization types" (awq_w4a16 /
// int4 / group 64).
//
// Design (sm_100a).  At M = 64 the product has as many tensor-core flops as there
// are weight bytes to stream, more than mma.sync sustains; here a CTA owns 128
// weight rows and all T (16, 32 or 64) token columns, and the dequantized weights are
// the A operand of tcgen05.mma (kind::f16, M = 128, N = T, K = 16), held in tensor
// memory (row n in lane n, two consecutive K per 32-bit column), with the fp32
// accumulators in tensor memory too.  Keeping A out of shared memory matters: a bf16 A
// written to and read back from shared memory costs four times the packed weight bytes
// twice, more shared-memory bandwidth than the MMAs' own B reads.  480 threads:
//   warp 0     TMA producer: before the grid-dependency wait the CTA's scale and zero rows
//              into shared memory (when K % 512 == 0, K <= 4096 and both are 16-byte
//              aligned; else the dequantizers and the epilogue read them from global memory a
//              stage ahead); then per 256-K stage the 128 x 128-byte weight-code tile and the
//              tokens' activations as four 64-column sub-tiles (128-byte swizzle, rows past
//              M read as zeros) -- the MMA's B operand as they land -- paced: stage kb is
//              requested once stage kb - 3 has landed.
//   warps 2-9  dequantizers, two per tensor-memory lane quarter: a thread owns one weight
//              row (its lane) and half of every group; it turns its 16 code bytes of a
//              group into bf16 q - z (128 + q by bit placement, one packed subtraction of
//              128 + z: exact) and writes them as 16 columns of its lane (tcgen05.st);
//              units of four groups (two at T = 64), two units in rotation.
//   warps 1, 14  the MMA issue (warp 1 also owns the tensor-memory allocation), even and
//              odd units in alternation: per unit four MMAs per group, each group into its
//              own T-column accumulator; one tcgen05.commit frees the A unit, one publishes
//              the unit's accumulators, one releases the unit's reads of the stage.  A single
//              issuing thread -- its barrier waits and 8-16 MMAs per unit -- was the limit.
//   warps 10-13 epilogue: a thread owns one accumulator row; per group it reads the
//              T partial sums (tcgen05.ld) and adds s[n, g] times them to fp32
//              registers, handing accumulators back four at a time; at the end + b, bf16
//              stores.
// Every product is exact and each group's fp32 partial sum is scaled by s once, as in
// kernel 3.  Every mbarrier wait is bounded.
#pragma once

#include "ptx.cuh"

namespace svdq {
namespace k4 {

constexpr int kRows = 128;                 // weight rows per CTA = MMA M
constexpr int kChunk = 256;                // K per stage
constexpr int kGroup = 64;
constexpr int kWBytes = kRows * 128;       // packed weight codes of one stage
constexpr int kACols = kGroup / 2;         // tensor-memory columns of one dequantized group (bf16 pairs)
constexpr int kABufs = 2;
constexpr int kDeqWarps = 8;               // two per lane quarter (half a group each)
constexpr int kEpiWarp0 = 2 + kDeqWarps;
constexpr int kMmaWarp2 = kEpiWarp0 + 4;   // the second MMA-issuing warp (odd units)
constexpr int kThreads = (kMmaWarp2 + 1) * 32;
constexpr int kMaxSzGroups = 64;           // K <= 4096: the CTA's scale and zero rows held in shared memory
constexpr int kPace = 3;                   // stage kb is requested once stage kb - kPace has landed

template <int T>
struct Cfg {
  static_assert(T == 16 || T == 32 || T == 64, "token columns");
  static constexpr int XSUB = T * 128;                      // one 64-K activation sub-tile
  static constexpr int STAGE = kWBytes + 4 * XSUB;
  // groups per A unit (the MMA warp's step): a whole stage, or half of one at T = 64 where
  // the accumulators take more tensor memory
  static constexpr int UG = T == 64 ? 2 : 4;
  static constexpr int STAGES = T == 64 ? 4 : (T == 32 ? 6 : 8);
  static constexpr int OFF_SZ = STAGES * STAGE;             // [scales, zeros][128 rows][K / 64 <= 64 groups] bf16
  static constexpr int OFF_BAR = OFF_SZ + 2 * kRows * kMaxSzGroups * 2;
  static constexpr int DBUFS = T == 64 ? 4 : 8;             // accumulators in tensor memory (T columns each)
  static constexpr int DPAIRS = DBUFS / UG;                 // handed over a unit at a time
  static constexpr int NUM_BARS = 2 * STAGES + 2 * kABufs + 2 * DPAIRS + 2;   // + drain, scale rows
  static constexpr int OFF_MISC = OFF_BAR + 8 * NUM_BARS;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;
  static constexpr int A_COL0 = DBUFS * T;                  // tensor memory: accumulators, then the A units
  static constexpr int TMEM_COLS = 512;
  static_assert(A_COL0 + kABufs * UG * kACols <= TMEM_COLS, "tensor memory");
  static_assert(DPAIRS >= 2, "accumulators double-buffered per unit");
  static_assert(STAGE % 1024 == 0, "1 KB alignment of swizzled tiles");
  static_assert(SMEM <= 227 * 1024 && SMEM > 116 * 1024, "shared memory: one CTA (and one 512-column allocation) per SM");
};

struct Params {
  const __nv_bfloat16* scales;     // [N, K/64]
  const __nv_bfloat16* zeros;      // [N, K/64]
  const __nv_bfloat16* bias;       // [N] or null
  __nv_bfloat16* Y;                // [M, N]
  int M, N, K;
};

// kind::f16 instruction descriptor: D f32, A and B bf16, both K-major, M = 128, N = T.
template <int T>
__device__ __forceinline__ uint32_t idesc_awq() {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(T >> 3) << 17) |
         (static_cast<uint32_t>(128 >> 4) << 24);
}

// bf16x2 {128 + low nibble, 128 + high nibble} of byte b of w, minus (128 + z) in both halves.
// magic = 0x43004300 comes in a register, so that the mask-and-place is one three-input logic
// operation (an instruction takes one immediate).
__device__ __forceinline__ uint32_t deq_pair(uint32_t w, uint32_t w4, uint32_t sel, uint32_t zz, uint32_t magic) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(w), "r"(w4), "r"(sel));
  asm("lop3.b32 %0, %0, 0x000F000F, %1, 0xEA;" : "+r"(r) : "r"(magic));
  __nv_bfloat162 d = __hsub2(*reinterpret_cast<__nv_bfloat162*>(&r), *reinterpret_cast<__nv_bfloat162*>(&zz));
  return *reinterpret_cast<uint32_t*>(&d);
}

// Reads N consecutive 32-bit TMEM columns of this thread's lane (N = 16 or 32) and waits.
template <int N>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[N]) {
  if constexpr (N == 32) {
    tmem_ld_32x32b_x32(taddr, r);
    tmem_wait_ld_regs(r);
  } else {
    static_assert(N == 16, "16 or 32 columns");
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile(
        "tcgen05.wait::ld.sync.aligned;"
        : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
          "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15])
        :
        : "memory");
  }
}

// kSz: the CTA's scale and zero rows are copied into shared memory once, before the grid-dependency
// wait (tmS / tmZ: [N, K/64] bf16, box K/64 x 128; K % 512 == 0, K <= 4096, 16-byte aligned);
// otherwise they are read from global memory a stage ahead, with 8-byte loads of four groups when
// kVec (K % 256 == 0, aligned rows).
template <int T, bool kVec, bool kSz>
__global__ void __launch_bounds__(kThreads, 1)
awq_umma_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                const __grid_constant__ CUtensorMap tmS, const __grid_constant__ CUtensorMap tmZ, const Params p) {
  using C = Cfg<T>;
  constexpr int S = C::STAGES;
  static_assert(4 % C::UG == 0, "units divide a stage");
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t bars = base + C::OFF_BAR;
  auto full = [&](int s) { return bars + 8u * s; };
  auto empty = [&](int s) { return bars + 8u * (S + s); };
  auto afull = [&](int a) { return bars + 8u * (2 * S + a); };
  auto afree = [&](int a) { return bars + 8u * (2 * S + kABufs + a); };
  constexpr int DP = C::DPAIRS;
  auto dfull = [&](int d) { return bars + 8u * (2 * S + 2 * kABufs + d); };
  auto dfree = [&](int d) { return bars + 8u * (2 * S + 2 * kABufs + DP + d); };
  const uint32_t drain = bars + 8u * (2 * S + 2 * kABufs + 2 * DP);
  const uint32_t sz_bar = drain + 8u;              // the scale and zero rows have landed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + C::OFF_MISC + 4);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int n0 = blockIdx.x * kRows;
  const int t0 = blockIdx.y * T;                   // this CTA's first token (M > 64: one CTA row per 64 tokens)
  const int nkb = (p.K + kChunk - 1) / kChunk;     // the last stage may hold 1-3 groups (K % 64 == 0)
  const int nunits = nkb * 4 / C::UG;                // C::UG groups per unit
  const int gpr = p.K / kGroup;                    // groups per weight row

  if (warp == 0 && lane == 0) {
    // a stage is free once the dequantizers have its code bytes and every unit's MMAs are done
    for (int s = 0; s < S; ++s) { mbar_init(full(s), 1); mbar_init(empty(s), kDeqWarps + 4 / C::UG); }
    for (int a = 0; a < kABufs; ++a) { mbar_init(afull(a), kDeqWarps); mbar_init(afree(a), 1); }
    for (int d = 0; d < DP; ++d) { mbar_init(dfull(d), 1); mbar_init(dfree(d), 4); }
    mbar_init(drain, 2);                           // both MMA-issuing warps
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
  if (warp == 1) tmem_alloc<C::TMEM_COLS>(smem_addr(tmem_slot));
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (warp == 0 && lane == 0) {
    // The weights, scales and zeros never come from the previous kernel: this CTA's scale and
    // zero rows are copied into shared memory (or pulled toward L2) and the first stages' tiles
    // toward L2 while it finishes (hints; L2 is coherent, so nothing stale can be read).
    if (kSz) {
      mbar_arrive_expect_tx(sz_bar, 2u * kRows * gpr * 2);
      tma_load_2d(base + C::OFF_SZ, &tmS, 0, n0, sz_bar);
      tma_load_2d(base + C::OFF_SZ + kRows * kMaxSzGroups * 2, &tmZ, 0, n0, sz_bar);
    } else {
      const size_t rb = static_cast<size_t>(n0) * (p.K / kGroup) * 2;
      const uint32_t bytes = static_cast<uint32_t>(min(kRows, p.N - n0) * (p.K / kGroup) * 2);
      bulk_prefetch_l2_any(reinterpret_cast<const uint8_t*>(p.scales) + rb, bytes);
      bulk_prefetch_l2_any(reinterpret_cast<const uint8_t*>(p.zeros) + rb, bytes);
    }
    for (int kb = 0; kb < min(kPace, nkb); ++kb) tma_prefetch_l2_2d(&tmW, kb * (kChunk / 2), n0);
  }
  grid_dependency_wait();                          // X may belong to the previous kernel
  grid_launch_dependents();

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    for (int kb = 0; kb < nkb; ++kb) {
      const int s = kb % S;
      const uint32_t ph = (kb / S) & 1u;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(empty(s), ph ^ 1u, abort_flag, 31))) break;
      if (kb >= kPace) {
        // paced: with every CTA's whole ring requested at once the memory system serves all of
        // them interleaved and each CTA's first tile lands late
        const int kp = kb - kPace;
        if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(full(kp % S), (kp / S) & 1u, abort_flag, 41))) break;
      }
      if (elect_one()) {
        const uint32_t sb = base + s * C::STAGE;
        mbar_arrive_expect_tx(full(s), C::STAGE);
        tma_load_2d(sb, &tmW, kb * (kChunk / 2), n0, full(s));
#pragma unroll
        for (int j = 0; j < 4; ++j) tma_load_2d(sb + kWBytes + j * C::XSUB, &tmX, kb * kChunk + j * 64, t0, full(s));
      }
      __syncwarp();
    }
  } else if (warp == 1 || warp == kMmaWarp2) {
    // ---------------------------------------------------------------- MMA issue (one elected lane)
    constexpr uint32_t kHiSw128 = smem_desc_hi(1024, 2);      // K-major, 128-byte swizzle, 8-row groups
    constexpr uint32_t kLbo = 1u << 16;
    const uint32_t idesc = idesc_awq<T>();
    for (int u = warp == 1 ? 0 : 1; u < nunits; u += 2) {   // two issuing warps, alternate units
      const int kb = u * C::UG / 4;
      const int s = kb % S, a = u % kABufs, dp = u % DP;
      bool ok = mbar_wait_bounded(full(s), (kb / S) & 1u, abort_flag, 32);
      ok = ok && mbar_wait_bounded(afull(a), (u / kABufs) & 1u, abort_flag, 33);
      ok = ok && mbar_wait_bounded(dfree(dp), ((u / DP) & 1u) ^ 1u, abort_flag, 34);
      if (!__all_sync(0xFFFFFFFFu, ok)) break;
      tc_fence_after();
      if (elect_one()) {
#pragma unroll
        for (int gi = 0; gi < C::UG; ++gi) {
          const int grp = (u * C::UG + gi) & 3;
          const uint32_t a_t = tmem + static_cast<uint32_t>(C::A_COL0 + (a * C::UG + gi) * kACols);
          const uint32_t b_lo = ((base + s * C::STAGE + kWBytes + grp * C::XSUB) >> 4) | kLbo;
          const uint32_t dacc = tmem + static_cast<uint32_t>((C::UG * dp + gi) * T);
#pragma unroll
          for (int j = 0; j < kGroup / 16; ++j)       // K = 16: 8 columns of A, 32 bytes of B
            umma_bf16_ta(dacc, a_t + j * 8, make_desc(b_lo + j * 2, kHiSw128), idesc, j != 0 ? 1u : 0u);
        }
        tc_commit(afree(a));
        tc_commit(dfull(dp));
        tc_commit(empty(s));                       // this unit's reads of the stage
      }
      __syncwarp();
    }
  } else if (warp < kEpiWarp0) {
    // ---------------------------------------------------------------- dequantizers
    const int dq = warp & 3;                       // tensor-memory lane quarter of this warp
    const int r = dq * 32 + lane;                  // weight row of the tile = tensor-memory lane
    const int h = (warp - 2) >> 2;                 // half of each group: code bytes 16 h .. 16 h + 15
    const uint32_t rsw = static_cast<uint32_t>(r & 7);
    const uint32_t tlane = tmem + (static_cast<uint32_t>(dq * 32) << 16) + static_cast<uint32_t>(C::A_COL0 + h * 16);
    const uint32_t magic = static_cast<uint32_t>(abort_flag[1]);   // 0x43004300, opaque to the compiler
    // groups past K (a partial last stage) read as zero points 0 and their codes as 0 (zero-filled
    // copies): their A columns are 0
    const uint16_t* zrow = reinterpret_cast<const uint16_t*>(p.zeros) + static_cast<size_t>(min(n0 + r, p.N - 1)) * gpr;
    const uint8_t* zsm = gbase + C::OFF_SZ + kRows * kMaxSzGroups * 2 + static_cast<size_t>(r) * gpr * 2;
    constexpr bool vec = kVec;
    uint2 zn = make_uint2(0u, 0u);                 // zeros of the 4 groups of the next stage
    bool sz_ok = true;
    if constexpr (kSz) sz_ok = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(sz_bar, 0, abort_flag, 39));
    else zn = ld_groups4(zrow, 0, gpr, vec);
    for (int kb = 0; sz_ok && kb < nkb; ++kb) {
      const int s = kb % S;
      uint2 zc;
      if constexpr (kSz) {
        zc = *reinterpret_cast<const uint2*>(zsm + kb * 8);
      } else {
        zc = zn;
        if (kb + 1 < nkb) zn = ld_groups4(zrow, kb + 1, gpr, vec);
      }
      if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(full(s), (kb / S) & 1u, abort_flag, 35))) break;
      const uint8_t* wrow = gbase + s * C::STAGE + r * 128;
      bool ok = true;
#pragma unroll 1
      for (int ul = 0; ul < 4 / C::UG; ++ul) {       // the stage's units
        const int u = kb * (4 / C::UG) + ul;
        const int a = u % kABufs;
        // this thread's 16 code bytes of each of the unit's groups (16-byte units 2 grp + h, swizzled)
        uint4 c[C::UG];
#pragma unroll
        for (int gi = 0; gi < C::UG; ++gi)
          c[gi] = *reinterpret_cast<const uint4*>(wrow + (((2 * (C::UG * ul + gi) + h) ^ rsw) << 4));
        if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(afree(a), ((u / kABufs) & 1u) ^ 1u, abort_flag, 36))) {
          ok = false;
          break;
        }
#pragma unroll
        for (int gi = 0; gi < C::UG; ++gi) {
          const int grp = C::UG * ul + gi;
          const uint32_t zw = grp < 2 ? zc.x : zc.y;
          const float z = ((grp & 1) ? bf16hi_to_f32(zw) : bf16lo_to_f32(zw)) + 128.f;
          const uint32_t zz = pack_bf16x2(z, z);
          const uint32_t cw[4] = {c[gi].x, c[gi].y, c[gi].z, c[gi].w};
          // column 4 v + t of this half: K elements 32 h + 8 v + 2 t and + 1 (code byte t of word v)
          uint32_t o[16];
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const uint32_t w = cw[v], w4 = w >> 4;
            o[4 * v + 0] = deq_pair(w, w4, 0x0400u, zz, magic);
            o[4 * v + 1] = deq_pair(w, w4, 0x0501u, zz, magic);
            o[4 * v + 2] = deq_pair(w, w4, 0x0602u, zz, magic);
            o[4 * v + 3] = deq_pair(w, w4, 0x0703u, zz, magic);
          }
          tmem_st_32x32b_x16(tlane + static_cast<uint32_t>((a * C::UG + gi) * kACols), o);
        }
        tmem_wait_st();                            // the stores are in tensor memory ...
        tc_fence_before();                         // ... and ordered before the arrival
        __syncwarp();
        if (lane == 0) mbar_arrive(afull(a));
      }
      if (!ok) break;
      __syncwarp();
      if (lane == 0) mbar_arrive_relaxed(empty(s));   // this warp's code bytes are in registers
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int quarter = warp & 3;                  // tensor-memory lanes 32 quarter .. + 31
    const int r = quarter * 32 + lane;
    const uint32_t trow = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const uint16_t* srow = reinterpret_cast<const uint16_t*>(p.scales) + static_cast<size_t>(min(n0 + r, p.N - 1)) * gpr;
    constexpr bool vec = kVec;
    float tot[T];
#pragma unroll
    for (int t = 0; t < T; ++t) tot[t] = 0.f;
    const uint8_t* ssm = gbase + C::OFF_SZ + static_cast<size_t>(r) * gpr * 2;
    uint2 sn = make_uint2(0u, 0u), sc = sn;
    bool sz_ok = true;
    if constexpr (kSz) sz_ok = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(sz_bar, 0, abort_flag, 40));
    else sn = sc = ld_groups4(srow, 0, gpr, vec);
    for (int u = 0; sz_ok && u < nunits; ++u) {
      const int dp = u % DP;
      if ((u * C::UG) % 4 == 0) {                   // first unit of a stage
        if constexpr (kSz) {
          sc = *reinterpret_cast<const uint2*>(ssm + (u * C::UG / 4) * 8);
        } else {
          sc = sn;
          if (u * C::UG / 4 + 1 < nkb) sn = ld_groups4(srow, u * C::UG / 4 + 1, gpr, vec);
        }
      }
      if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(dfull(dp), (u / DP) & 1u, abort_flag, 37))) break;
      tc_fence_after();
#pragma unroll
      for (int gi = 0; gi < C::UG; ++gi) {
        const int grp = (u * C::UG + gi) & 3;
        const uint32_t sw = grp < 2 ? sc.x : sc.y;
        const float sg = (grp & 1) ? bf16hi_to_f32(sw) : bf16lo_to_f32(sw);
        const uint32_t tcol = trow + static_cast<uint32_t>((C::UG * dp + gi) * T);
        if constexpr (T == 16) {
          uint32_t v[16];
          tmem_ld_cols<16>(tcol, v);
#pragma unroll
          for (int t = 0; t < 16; ++t) tot[t] = fmaf(sg, __uint_as_float(v[t]), tot[t]);
        } else {
#pragma unroll
          for (int hh = 0; hh < T / 32; ++hh) {
            uint32_t v[32];
            tmem_ld_cols<32>(tcol + hh * 32, v);
#pragma unroll
            for (int t = 0; t < 32; ++t) tot[hh * 32 + t] = fmaf(sg, __uint_as_float(v[t]), tot[hh * 32 + t]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_relaxed(dfree(dp));
    }
    if (n0 + r < p.N) {
      const float bb = p.bias ? __bfloat162float(p.bias[n0 + r]) : 0.f;
#pragma unroll
      for (int t = 0; t < T; ++t)
        if (t0 + t < p.M) p.Y[static_cast<size_t>(t0 + t) * p.N + n0 + r] = __float2bfloat16_rn(tot[t] + bb);
    }
  }

  __syncthreads();
  if (*abort_flag) {
    // a wait ran out: let the MMAs and copies already issued finish before the memory goes away
    if (warp == 1 || warp == kMmaWarp2) {
      if (elect_one()) tc_commit(drain);
      __syncwarp();
      mbar_wait_bounded(drain, 0, nullptr, 38);
    }
    if (warp == 0 && lane == 0) {
      const uint64_t t0 = global_timer_ns();
      while (global_timer_ns() - t0 < 2000000ull) { }
    }
    __syncthreads();
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc<C::TMEM_COLS>(tmem);
  }
}

}  // namespace k4
}  // namespace svdq
