// Kernel 8: the SVDQuant W4A4 linear layer of the int4 / group-64 row on tcgen05.
//
//   y[m, n] = sum_g s_a[m, g] s_w[n, g] sum_{k in g} c_a[m, k] c_w[n, k] + (U L2)[m, n] + b[n]
//
// Method: "Nunchaku Lite" docs, "Supported quantization types": svdq_w4a4 with int4 precision
// and group size 64 (the same low-rank correction as the nvfp4 row; the docs note that nvfp4 is
// the faster of the two on Blackwell).  c are signed 4-bit codes (-7..7 in practice), s bf16
// per-64 scales of both operands, U = X_hat L1 (as kernel 1 writes it, hi + lo, no per-tensor
// scale in this format).
//
// Design (sm_100a).  The tensor cores have no 4-bit integer MMA; the int4 codes travel as their
// E4M3 bytes (every integer -8..8 is exact in E4M3) and are multiplied by the fp8 MMA
// (tcgen05 kind::f8f6f4, E4M3 x E4M3, fp32 accumulation): each group's 64-term sum of integer
// products (at most 3136 in magnitude) is exact in the fp32 accumulator.  Because both
// operands carry their own scale per group, the scale product s_a s_w differs for every
// (row, column, group): each group gets its own accumulator, and the epilogue applies the
// scales.  Persistent CTAs over 128 x 128 output tiles, 576 threads:
//   warp 0     TMA producer: per tile the low-rank tiles ([U hi | U lo], L2^T) as one stage, then
//              per 128-K stage the 128 x 128-byte code tiles of A and B (128-byte swizzle).
//   warp 1     tensor memory and the MMA issue: the low-rank product (four bf16 MMAs, K = 16)
//              into its own 128-column accumulator, then per group two fp8 MMAs (K = 32) into
//              one of three rotating 128-column group accumulators.
//   warps 2-17 epilogue, four per tensor-memory lane quarter, 32 columns each: start from the
//              low-rank product, then per group read the group's accumulator, hand it back, and
//              add s_a[m, g] s_w[n, g] times it (packed fp32 pairs; both scales group-major --
//              s_w pre-widened to fp32 in the weights, s_a bf16 with rows padded to 128 -- and
//              brought in by the producer, per group a 512-byte and a 256-byte TMA row, into a
//              ring of eight slots, so the epilogue's loop reads no global memory);
//              at the end + b, bf16, TMA stores through a 64-byte-swizzled staging tile.
// Every mbarrier wait is bounded; a wait that runs out records SVDQ_ERR_TIMEOUT and the CTA
// winds down.
#pragma once

#include "gemm_nvfp4.cuh"
#include "ptx.cuh"

namespace svdq {
namespace k8 {

constexpr int BM = 128;
constexpr int BN = 128;
constexpr int BK = 128;                    // K per stage: two groups
constexpr int kGroup = 64;
constexpr int STAGES = 4;
constexpr int kEpiWarps = 16;              // four per tensor-memory lane quarter
constexpr int kCols = BN / (kEpiWarps / 4);  // accumulator columns per epilogue warp (32)
constexpr int kThreads = (2 + kEpiWarps) * 32;
constexpr int A_BYTES = BM * BK;           // E4M3 codes
constexpr int B_BYTES = BN * BK;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int UCAT_BYTES = BM * 64 * 2;    // [U hi | U lo] bf16, fits the A slot
constexpr int L2_BYTES = BN * 32 * 2;      // L2^T bf16, fits the B slot
constexpr int GBUF = 3;                    // group accumulators in tensor memory
constexpr uint32_t TM_LR = GBUF * BN;      // the low-rank accumulator's first column
constexpr int TMEM_COLS = 512;
constexpr int SB = 8;                      // scale slots: one group's 128 fp32 weight scales, then its
constexpr int WS_SLOT = BN * 4 + BM * 2;   // 128 bf16 activation scales
// barriers: full[S], empty[S], grp_full[3], grp_empty[3], lr_full, lr_empty, drain, ws_full[SB], ws_empty[SB]
constexpr int NUM_BARS = 2 * STAGES + 2 * GBUF + 3 + 2 * SB;
constexpr int OFF_BAR = STAGES * STAGE_BYTES;
constexpr int OFF_MISC = OFF_BAR + 8 * NUM_BARS;
constexpr int OFF_BIAS = (OFF_MISC + 64 + 127) / 128 * 128;        // per epilogue warp: kCols bias values (bf16)
constexpr int OFF_STAGE = (OFF_BIAS + kEpiWarps * kCols * 2 + 1023) / 1024 * 1024;   // per epilogue warp: 32 x 32 bf16
constexpr int OFF_WS = OFF_STAGE + kEpiWarps * 2048;                            // SB weight-scale slots
constexpr int SMEM_BYTES = OFF_WS + SB * WS_SLOT + 1024;
constexpr uint32_t TX_MAIN = STAGE_BYTES;
constexpr uint32_t TX_LOWRANK = UCAT_BYTES + L2_BYTES;
static_assert(TM_LR + BN <= TMEM_COLS, "tensor memory");
static_assert(STAGE_BYTES % 1024 == 0 && A_BYTES % 1024 == 0, "1 KB alignment of swizzled tiles");
static_assert(UCAT_BYTES <= A_BYTES && L2_BYTES <= B_BYTES, "low-rank tiles fit a stage");
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");

struct Params {
  const __nv_bfloat16* bias;       // [N]
  int M, N, K;
  int tiles_n, tiles;
};

// kind::f8f6f4: D f32 (bits 4-5 = 1), A and B E4M3 (format 0), K-major, N = 128, M = 128.
__device__ __forceinline__ uint32_t idesc_e4m3() {
  return (1u << 4) | (static_cast<uint32_t>(BN >> 3) << 17) | (static_cast<uint32_t>(BM >> 4) << 24);
}
// kind::f16: D f32, A and B bf16, K-major, N = 128, M = 128.
__device__ __forceinline__ uint32_t idesc_bf16() {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(BN >> 3) << 17) |
         (static_cast<uint32_t>(BM >> 4) << 24);
}

__device__ __forceinline__ void umma_e4m3(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{ .reg .pred p; setp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p; }"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
}

__global__ void __launch_bounds__(kThreads, 1)
int4_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const __grid_constant__ CUtensorMap tmU, const __grid_constant__ CUtensorMap tmL2,
                 const __grid_constant__ CUtensorMap tmY, const __grid_constant__ CUtensorMap tmWS,
                 const __grid_constant__ CUtensorMap tmAS, const Params p) {
  constexpr int S = STAGES;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t bars = base + OFF_BAR;
  auto full = [&](int s) { return bars + 8u * s; };
  auto empty = [&](int s) { return bars + 8u * (S + s); };
  auto grp_full = [&](int b) { return bars + 8u * (2 * S + b); };
  auto grp_empty = [&](int b) { return bars + 8u * (2 * S + GBUF + b); };
  const uint32_t lr_full = bars + 8u * (2 * S + 2 * GBUF);
  const uint32_t lr_empty = bars + 8u * (2 * S + 2 * GBUF + 1);
  const uint32_t drain = bars + 8u * (2 * S + 2 * GBUF + 2);
  auto ws_full = [&](int b) { return bars + 8u * (2 * S + 2 * GBUF + 3 + b); };
  auto ws_empty = [&](int b) { return bars + 8u * (2 * S + 2 * GBUF + 3 + SB + b); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + OFF_MISC + 4);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int ngroups = p.K / kGroup;
  const int nkb = (ngroups + 1) / 2;               // 128-K stages (the last may hold one group)

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < S; ++s) { mbar_init(full(s), 1); mbar_init(empty(s), 1); }
    for (int b = 0; b < GBUF; ++b) { mbar_init(grp_full(b), 1); mbar_init(grp_empty(b), kEpiWarps); }
    mbar_init(lr_full, 1);
    mbar_init(lr_empty, kEpiWarps);
    mbar_init(drain, 1);
    for (int b = 0; b < SB; ++b) { mbar_init(ws_full(b), 1); mbar_init(ws_empty(b), kEpiWarps); }
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmA); prefetch_tmap(&tmB); prefetch_tmap(&tmU); prefetch_tmap(&tmL2); prefetch_tmap(&tmY);
    prefetch_tmap(&tmWS); prefetch_tmap(&tmAS);
  }
  if (warp == 1) tmem_alloc<TMEM_COLS>(smem_addr(tmem_slot));
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  grid_dependency_wait();
  grid_launch_dependents();

  constexpr uint32_t kHiSw128 = smem_desc_hi(1024, 2);
  constexpr uint32_t kHiSw64 = smem_desc_hi(512, 4);
  constexpr uint32_t kLbo = 1u << 16;

  if (warp == 0) {
    // ------------------------------------------------------------------ producer
    uint32_t g = 0, gs = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < p.tiles; t += gridDim.x) {
      const int m0 = (t / p.tiles_n) * BM, n0 = (t % p.tiles_n) * BN;
      for (int kb = -1; ok && kb < nkb; ++kb, ++g) {   // kb == -1: the low-rank stage
        const int s = g % S;
        if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(empty(s), ((g / S) & 1u) ^ 1u, abort_flag, 51))) {
          ok = false;
          break;
        }
        if (elect_one()) {
          const uint32_t sb = base + s * STAGE_BYTES;
          if (kb < 0) {
            mbar_arrive_expect_tx(full(s), TX_LOWRANK);
            tma_load_2d(sb, &tmU, 0, m0, full(s));
            tma_load_2d(sb + A_BYTES, &tmL2, 0, n0, full(s));
          } else {
            mbar_arrive_expect_tx(full(s), TX_MAIN);
            tma_load_2d(sb, &tmA, kb * BK, m0, full(s));
            tma_load_2d(sb + A_BYTES, &tmB, kb * BK, n0, full(s));
          }
        }
        __syncwarp();
        // the scales of the stage's groups (weights, then activations), one slot each (the
        // epilogue frees them)
        for (int j = 0; kb >= 0 && j < min(2, ngroups - 2 * kb); ++j, ++gs) {
          const int b = gs % SB;
          if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(ws_empty(b), ((gs / SB) & 1u) ^ 1u, abort_flag, 58))) {
            ok = false;
            break;
          }
          if (elect_one()) {
            mbar_arrive_expect_tx(ws_full(b), WS_SLOT);
            tma_load_2d(base + OFF_WS + b * WS_SLOT, &tmWS, n0, 2 * kb + j, ws_full(b));
            tma_load_2d(base + OFF_WS + b * WS_SLOT + BN * 4, &tmAS, m0, 2 * kb + j, ws_full(b));
          }
          __syncwarp();
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issue
    const uint32_t id8 = idesc_e4m3(), idb = idesc_bf16();
    uint32_t g = 0, gc = 0;
    int i = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < p.tiles; t += gridDim.x, ++i) {
      for (int kb = -1; ok && kb < nkb; ++kb, ++g) {
        const int s = g % S;
        const uint32_t sb = base + s * STAGE_BYTES;
        const uint32_t a_lo = (sb >> 4) | kLbo, b_lo = ((sb + A_BYTES) >> 4) | kLbo;
        if (kb < 0) {
          // the low-rank accumulator must have been read by the previous tile's epilogue
          if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(lr_empty, (i & 1) ^ 1, abort_flag, 52))) { ok = false; break; }
        }
        if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(full(s), (g / S) & 1u, abort_flag, 53))) { ok = false; break; }
        tc_fence_after();
        if (kb < 0) {
          if (elect_one()) {
            // A [U hi | U lo] (K 0..63), B L2^T (K 0..31) twice: U hi L2 + U lo L2
#pragma unroll
            for (int j = 0; j < 4; ++j)
              umma_bf16(tmem + TM_LR, make_desc(a_lo + j * 2, kHiSw128), make_desc(b_lo + (j & 1) * 2, kHiSw64),
                        idb, j ? 1u : 0u);
            tc_commit(empty(s));
            tc_commit(lr_full);
          }
          __syncwarp();
          continue;
        }
        const int ng = min(2, ngroups - 2 * kb);
        for (int gi = 0; gi < ng; ++gi, ++gc) {
          const int b = gc % GBUF;
          if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(grp_empty(b), ((gc / GBUF) & 1u) ^ 1u, abort_flag, 54))) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < 2; ++kk)      // K = 32 bytes per MMA
              umma_e4m3(tmem + static_cast<uint32_t>(b * BN), make_desc(a_lo + gi * 4 + kk * 2, kHiSw128),
                        make_desc(b_lo + gi * 4 + kk * 2, kHiSw128), id8, kk ? 1u : 0u);
            tc_commit(grp_full(b));
          }
          __syncwarp();
        }
        if (!ok) break;
        if (elect_one()) tc_commit(empty(s));
        __syncwarp();
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    const int quarter = warp & 3;
    const int ew = warp - 2;
    const int eh = ew >> 2;                        // columns kCols eh .. kCols (eh + 1) - 1 of the tile
    const int r = quarter * 32 + lane;
    uint8_t* sbias = gbase + OFF_BIAS + ew * (kCols * 2);
    const uint32_t stage_tile = base + OFF_STAGE + ew * 2048;
    const uint32_t stage_row = stage_tile + lane * 64;
    const uint32_t sw = (static_cast<uint32_t>(lane) >> 1) & 3u;
    uint32_t gc = 0;
    int i = 0;
    bool ok = true;
    const uint8_t* ws_smem = gbase + OFF_WS;
    for (int t = blockIdx.x; ok && t < p.tiles; t += gridDim.x, ++i) {
      const int m0 = (t / p.tiles_n) * BM, n0 = (t % p.tiles_n) * BN;
      const int nc = n0 + kCols * eh;              // this warp's first column
      if (lane < kCols / 8)
        *reinterpret_cast<uint4*>(sbias + lane * 16) = __ldg(reinterpret_cast<const uint4*>(p.bias + nc) + lane);
      __syncwarp();
      const uint32_t trow = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(kCols * eh);
      // start from the low-rank product
      static_assert(kCols == 32, "one 32-column tensor-memory load per warp and group");
      float acc[kCols];
      if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(lr_full, i & 1, abort_flag, 55))) break;
      tc_fence_after();
      {
        uint32_t R0[32];
        tmem_ld_32x32b_x32(trow + TM_LR, R0);
        tmem_wait_ld_regs(R0);
#pragma unroll
        for (int j = 0; j < 32; ++j) acc[j] = __uint_as_float(R0[j]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(lr_empty);
      // the groups
      for (int gi = 0; gi < ngroups; ++gi, ++gc) {
        const int b = gc % GBUF;
        const int sbi = gc % SB;
        const uint8_t* slot = ws_smem + sbi * WS_SLOT;
        const float4* sw4 = reinterpret_cast<const float4*>(slot) + (kCols / 4) * eh;
        if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(grp_full(b), (gc / GBUF) & 1u, abort_flag, 56) &&
                                         mbar_wait_bounded(ws_full(sbi), (gc / SB) & 1u, abort_flag, 59))) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t D[32];
        tmem_ld_32x32b_x32(trow + static_cast<uint32_t>(b * BN), D);
        const float sa = bf16lo_to_f32(*reinterpret_cast<const uint16_t*>(slot + BN * 4 + 2 * r));
        tmem_wait_ld_regs(D);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(grp_empty(b));
        const uint64_t sa2 = f32x2_pack(sa, sa);
#pragma unroll
        for (int q = 0; q < kCols / 4; ++q) {
          const float4 wsv = sw4[q];               // one broadcast shared-memory load
          const int j = q * 4;
          const uint64_t s01 = f32x2_mul(sa2, f32x2_pack(wsv.x, wsv.y));
          const uint64_t s23 = f32x2_mul(sa2, f32x2_pack(wsv.z, wsv.w));
          const int a = q * 4;
          uint64_t v01 = f32x2_fma(s01, f32x2_pack(__uint_as_float(D[j]), __uint_as_float(D[j + 1])),
                                   f32x2_pack(acc[a], acc[a + 1]));
          uint64_t v23 = f32x2_fma(s23, f32x2_pack(__uint_as_float(D[j + 2]), __uint_as_float(D[j + 3])),
                                   f32x2_pack(acc[a + 2], acc[a + 3]));
          f32x2_unpack(v01, acc[a], acc[a + 1]);
          f32x2_unpack(v23, acc[a + 2], acc[a + 3]);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(ws_empty(sbi));
      }
      if (!ok) break;
      // + b, bf16, one 32-column TMA store through the staging tile
      if (m0 + quarter * 32 < p.M) {
#pragma unroll
        for (int c = 0; c < kCols / 32; ++c) {
          if (lane == 0) bulk_wait_group_read<0>();
          __syncwarp();
          uint32_t o[16];
          const uint32_t* bw = reinterpret_cast<const uint32_t*>(sbias + c * 64);
#pragma unroll
          for (int k = 0; k < 16; ++k)
            o[k] = pack_bf16x2(acc[32 * c + 2 * k] + bf16lo_to_f32(bw[k]), acc[32 * c + 2 * k + 1] + bf16hi_to_f32(bw[k]));
#pragma unroll
          for (int q = 0; q < 4; ++q)
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                         ::"r"(stage_row + ((static_cast<uint32_t>(q) ^ sw) << 4)), "r"(o[q * 4]), "r"(o[q * 4 + 1]),
                           "r"(o[q * 4 + 2]), "r"(o[q * 4 + 3])
                         : "memory");
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tmY, stage_tile, nc + 32 * c, m0 + quarter * 32);
            bulk_commit_group();
          }
        }
      }
    }
    if (lane == 0) bulk_wait_group<0>();
    __syncwarp();
  }

  __syncthreads();
  if (*abort_flag) {
    if (warp == 1) {
      if (elect_one()) tc_commit(drain);
      __syncwarp();
      mbar_wait_bounded(drain, 0, nullptr, 57);
    }
    if (warp == 0 && lane == 0) {
      const uint64_t t0 = global_timer_ns();
      while (global_timer_ns() - t0 < 2000000ull) { }
    }
    __syncthreads();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc<TMEM_COLS>(tmem);
  }
}

}  // namespace k8
}  // namespace svdq
