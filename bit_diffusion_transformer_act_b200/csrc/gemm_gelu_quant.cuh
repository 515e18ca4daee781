// Kernel 6: the MLP up-projection's NVFP4 GEMM with GELU and the down projection's activation
// pass fused into its epilogue; kernel 7: the reduction of its partial low-rank products.
//
// Method: "Nunchaku Lite" docs, section on fused kernels -- the original engine runs the MLP
// with a fused GELU kernel (its benchmark table gives the GELU-MLP fusion 1.06x).  What the
// fused epilogue computes is what the unfused pipeline computes (the reading of the pages):
//   y = bf16( g_a g_w (Q(X_hat) Q(R)^T) + U L2 + b )            the up projection (kernel 2)
//   h = bf16( GELU(y) ),  GELU(x) = x Phi(x) (erf form)           the hidden state
//   then kernel 1 on h with the down projection's smooth_inv, g_a and L1: NVFP4 codes and
//   swizzled E4M3 scales of h_hat = h smooth_inv, and U = h_hat L1 as bf16 hi + lo of U / g_a,
// without writing h (a 4608 x 12288 bf16 hidden state is 113 MB) or reading it back.
//
// Design (sm_100a).  The GEMM is kernel 2's pair-wide block-scaled tcgen05 mainloop with
// 256 x 128 output tiles (both accumulators and the low-rank product of the down projection
// fit in tensor memory next to each other), five 256-K stages, and a contiguous range of the
// row-major tile order per CTA pair, so that a pair walks consecutive N tiles of a row block.
// 384 threads per CTA:
//   warp 0     TMA producer of the mainloop (as kernel 2).
//   warp 1     tensor memory, block-scaled and low-rank MMAs of the up projection (leader).
//   warps 2-9  epilogue: a warp owns 32 rows (its tensor-memory lane quarter) and two of the
//              tile's four 32-column chunks.  Per element y = alpha acc + b, rounded to bf16;
//              h = bf16(GELU(y)) is one gather from a 64K-entry table of bf16(GELU(x)) for
//              every bf16 x (filled in double precision); h is written into a 128 x 64 shared-memory
//              slab (the A operand of the low-rank MMA, 128-byte swizzle) and quantized in
//              registers with the down projection's smoothing and scale (the quantizer of
//              kernel 1: codes and scale bytes stored straight to global memory).
//   warp 10    both CTAs: per tile, TMA loads of this CTA's half of the down projection's
//              packed low-rank factor (diag(smooth_inv) L1)^T (hi and lo, 16 of the 32 rank rows,
//              the tile's 128 columns) for the low-rank MMA.
//   warp 11    leader: per 64-column slab, eight tcgen05 MMAs (M = 256, N = 32, K = 16) adding
//              h_slab (hi + lo)^T into a 32-column fp32 accumulator that stays in tensor memory
//              over the pair's consecutive tiles of one row block; when the row block changes
//              (or the range ends), the epilogue reads it out as one partial per (pair, row block).
// Kernel 7 then sums, for every row, the partials of the pairs whose ranges cover its row block
// (in pair order: deterministic), and writes U / g_a as bf16 hi + lo.  Every mbarrier wait is
// bounded; a wait that runs out records SVDQ_ERR_TIMEOUT and the CTA winds down.
#pragma once

#include "act_amax.cuh"
#include "gemm_nvfp4.cuh"
#include "nvfp4_quant.cuh"
#include "ptx.cuh"

namespace svdq {
namespace k6 {

constexpr int BM = 128;                    // A rows per CTA (256 per pair)
constexpr int BN = 128;                    // output columns per tile (64 B rows per CTA)
constexpr int BN_HALF = BN / 2;
constexpr int BK = 256;
constexpr int STAGES = 5;
constexpr int kEpiWarps = 8;
constexpr int kLoadWarp = 2 + kEpiWarps;   // warp 10
constexpr int kUWarp = kLoadWarp + 1;      // warp 11
constexpr int kThreads = (kUWarp + 1) * 32;
constexpr int A_BYTES = BM * BK / 2;
constexpr int B_BYTES = BN_HALF * BK / 2;
constexpr int SFA_BYTES = (BK / 64) * 512;
constexpr int SFB_BYTES = (BK / 64) * 512;  // one 128-row scale block per tile
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
constexpr int UCAT_BYTES = BM * 64 * 2;
constexpr int L2_BYTES = BN_HALF * 32 * 2;
constexpr int SLAB_BYTES = BM * 64 * 2;    // 128 rows x 64 bf16, 128-byte swizzle
constexpr int L1T_BYTES = 16 * 64 * 2;     // 16 rank rows x 64 columns: one hi or lo slab half
constexpr int L1BUF_BYTES = 4 * L1T_BYTES; // hi slab 0, hi slab 1, lo slab 0, lo slab 1
constexpr int NBF = 8;
// barriers: full[NBF], empty[S], acc_full[2], acc_empty[2], drain, slab_ready[2], slab_free[2],
// l1_full[2], l1_free[2], u_full, u_empty
constexpr int NUM_BARS = NBF + STAGES + 2 + 2 + 1 + 2 + 2 + 2 + 2 + 1 + 1;
constexpr int OFF_SLAB = STAGES * STAGE_BYTES;
constexpr int OFF_L1 = OFF_SLAB + 2 * SLAB_BYTES;
constexpr int OFF_BAR = OFF_L1 + 2 * L1BUF_BYTES;
constexpr int OFF_MISC = OFF_BAR + 8 * NUM_BARS;
// per epilogue warp: the tile's bias (BN bf16), then its -smooth_inv (BN fp32)
constexpr int VEC_BYTES = BN * 2 + BN * 4;
constexpr int OFF_VEC = (OFF_MISC + 64 + 127) / 128 * 128;
// the GELU table's window |x| in [2^-31, 256) (bf16 magnitude patterns [0x3000, 0x4380)), both
// signs, copied into shared memory once per CTA: [sign][pattern - 0x3000]
constexpr uint32_t kGeluLo = 0x3000u;
constexpr uint32_t kGeluSpan = 0x4380u - kGeluLo;
constexpr int OFF_GELU = OFF_VEC + kEpiWarps * VEC_BYTES;
constexpr int SMEM_BYTES = OFF_GELU + 2 * kGeluSpan * 2 + 1024;
// tensor memory: accumulators [0, 128) and [128, 256), scale regions [256, 320), U [320, 352)
constexpr int SF_COLS = 4 * (BK / 64) + 4 * (BK / 64);
constexpr uint32_t TM_SF = 2 * BN;
constexpr uint32_t SFB_OFF = 4 * (BK / 64);
constexpr uint32_t TM_U = TM_SF + 2 * SF_COLS;
constexpr int TMEM_COLS = 512;
constexpr uint32_t TX_MAIN = 2u * STAGE_BYTES;
constexpr uint32_t TX_LOWRANK = 2u * (UCAT_BYTES + L2_BYTES);
constexpr uint32_t TX_L1 = 2u * L1BUF_BYTES;
static_assert(TM_U + 32 <= TMEM_COLS, "tensor memory");
static_assert(NBF > STAGES, "a full barrier is reused only after its group was consumed");
static_assert(STAGE_BYTES % 1024 == 0 && B_BYTES % 1024 == 0 && OFF_SLAB % 1024 == 0 && OFF_L1 % 1024 == 0,
              "1 KB alignment of swizzled tiles");
static_assert(UCAT_BYTES <= A_BYTES && L2_BYTES <= B_BYTES, "low-rank tiles fit the stage slots");
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");

struct Params {
  const __nv_bfloat16* bias;       // [N] (the up projection's)
  const __nv_bfloat16* smooth;     // [N] the down projection's smooth_inv
  uint8_t* codes;                  // [M, N/2] out
  uint8_t* scales;                 // swizzled [ceil(M/128) * 128, N/16] out
  float* ws;                       // partial U: [npairs][slots][256][32]
  __nv_bfloat16* h_out;            // [M, N] or null: the hidden state, for inspection
  const uint16_t* gelu;            // [65536]: bf16(GELU(x)) for every bf16 pattern x
  int M, N, K;
  int tiles_n, tiles;
  int slots;
  float alpha;                     // g_a g_w of the up projection
  float g, inv_g;                  // the down projection's g_a (a power of two) and its inverse
};

// First tile of pair p's contiguous range of the row-major tile order.
__host__ __device__ __forceinline__ int range_start(int p, int tiles, int npairs) {
  return static_cast<int>((static_cast<long long>(p) * tiles) / npairs);
}

// kind::f16, D f32, A and B bf16, K-major, M = 256 (pair), N = 32.
__device__ __forceinline__ uint32_t idesc_u() {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(32 >> 3) << 17) |
         (static_cast<uint32_t>(256 >> 4) << 24);
}

// bf16 nearest (ties to even) to a double, rounded once: 8 significant bits, the exponent range
// of fp32 (subnormal steps of 2^-133); overflow gives infinity.
__device__ __forceinline__ uint16_t bf16_rne_from_double(double v) {
  if (isnan(v)) return 0x7FC0;
  const uint16_t sign = signbit(v) ? 0x8000 : 0;
  const double a = fabs(v);
  if (a == 0.0) return sign;
  if (isinf(a)) return sign | 0x7F80;
  int e;
  (void)frexp(a, &e);                              // a in [2^(e-1), 2^e)
  const int step = max(e - 8, -133);               // weight of the last kept bit
  const double r = ldexp(rint(ldexp(a, -step)), step);   // rint: to nearest, ties to even
  return sign | static_cast<uint16_t>(__float_as_uint(static_cast<float>(r)) >> 16);   // exact (or inf)
}

// The GELU table: entry i (a bf16 bit pattern x) holds bf16(x Phi(x)), Phi(x) = erfc(-x / sqrt 2) / 2
// evaluated in double precision and rounded once.  h = bf16(GELU(y)) with y already rounded to
// bf16 is then one look-up.  Outside 2^-9 <= x < 4 and -16 < x <= -2^-9 the table has closed
// forms, which the epilogue uses outside its shared-memory window (below):
//   x >= 4: x Phi(x) rounds to x;   x <= -16: to -0;
//   2^-125 <= |x| < 2^-9: to x / 2 exactly (the pattern minus one exponent step), as
//     x^2 / sqrt(2 pi) is below half an ulp of x / 2;
//   |x| < 2^-125 (bf16 subnormals and the smallest normal binade): x / 2 rounded to nearest even
//     on the subnormal grid (the double evaluation carries no x^2 term there);
//   +inf: +inf; -inf: NaN (-inf times Phi(-inf) = 0); NaN: the quiet NaN of the same payload.
__global__ void __launch_bounds__(256) gelu_table_kernel(uint16_t* __restrict__ table) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= 65536) return;
  const double x = static_cast<double>(__uint_as_float(static_cast<uint32_t>(i) << 16));
  table[i] = bf16_rne_from_double(0.5 * x * erfc(-x / sqrt(2.0)));
}

// h for any bf16 pattern u: the shared-memory window where it holds u, else the closed forms
// listed with the table (equal to the table's entries; checked over every finite pattern).
__device__ __forceinline__ uint32_t gelu_bf16_rule(uint32_t u, const uint16_t* win) {
  const uint32_t w = u & 0x7FFFu, s = u >> 15;
  if (w - kGeluLo < kGeluSpan) return win[s * kGeluSpan + (w - kGeluLo)];
  if (w >= 0x7F80u) return u == 0xFF80u ? 0xFFC0u : (w == 0x7F80u ? u : (u | 0x40u));
  if (w >= kGeluLo + kGeluSpan) return s ? 0x8000u : u;
  if (w >= 0x100u) return u - 0x80u;
  return (u & 0x8000u) | ((w >> 1) + (w & (w >> 1) & 1u));
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
gemm_gelu_quant_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                       const __grid_constant__ CUtensorMap tmSFA, const __grid_constant__ CUtensorMap tmSFB,
                       const __grid_constant__ CUtensorMap tmU, const __grid_constant__ CUtensorMap tmL2,
                       const __grid_constant__ CUtensorMap tmL1, const Params p) {
  constexpr int S = STAGES;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);

  const uint32_t bars = base + OFF_BAR;
  auto full = [&](uint32_t it) { return bars + 8u * (it % NBF); };
  auto empty = [&](int s) { return bars + 8u * (NBF + s); };
  auto acc_full = [&](int b) { return bars + 8u * (NBF + S + b); };
  auto acc_empty = [&](int b) { return bars + 8u * (NBF + S + 2 + b); };
  const uint32_t drain = bars + 8u * (NBF + S + 4);
  auto slab_ready = [&](int b) { return bars + 8u * (NBF + S + 5 + b); };
  auto slab_free = [&](int b) { return bars + 8u * (NBF + S + 7 + b); };
  auto l1_full = [&](int b) { return bars + 8u * (NBF + S + 9 + b); };
  auto l1_free = [&](int b) { return bars + 8u * (NBF + S + 11 + b); };
  const uint32_t u_full = bars + 8u * (NBF + S + 13);
  const uint32_t u_empty = bars + 8u * (NBF + S + 14);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + OFF_MISC + 4);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const uint32_t cta = cluster_ctarank();
  const bool leader = cta == 0;
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;
  const int natoms = p.K / 64;
  const int nkb = (p.K + BK - 1) / BK;
  const int t_begin = range_start(pair, p.tiles, npairs);
  const int t_end = range_start(pair + 1, p.tiles, npairs);
  const int mt_first = t_begin / p.tiles_n;
  // a tile starts / ends a part (a run of the range's tiles within one row block)
  auto starts_part = [&](int t) { return t == t_begin || t % p.tiles_n == 0; };
  auto ends_part = [&](int t) { return t + 1 == t_end || (t + 1) % p.tiles_n == 0; };

  if (warp == 0 && lane == 0) {
    for (int i = 0; i < NBF; ++i) mbar_init(full(i), 2);
    for (int s = 0; s < S; ++s) mbar_init(empty(s), 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(acc_full(b), 1);
      mbar_init(acc_empty(b), 2 * kEpiWarps);
      mbar_init(slab_ready(b), 2 * kEpiWarps);
      mbar_init(slab_free(b), 1);
      mbar_init(l1_full(b), 1);
      mbar_init(l1_free(b), 1);
    }
    mbar_init(drain, 1);
    mbar_init(u_full, 1);
    mbar_init(u_empty, 2 * 4);                     // one warp per lane quarter, both CTAs
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmA); prefetch_tmap(&tmB); prefetch_tmap(&tmSFA);
    prefetch_tmap(&tmSFB); prefetch_tmap(&tmU); prefetch_tmap(&tmL2); prefetch_tmap(&tmL1);
  }
  if (warp == 1) tmem_alloc_pair<TMEM_COLS>(smem_addr(tmem_slot));
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (warp == 0 && lane == 0 && t_begin < t_end) {
    const int bn_first = (t_begin % p.tiles_n) * BN + static_cast<int>(cta) * BN_HALF;
    for (int kb = 0; kb < S && kb < nkb; ++kb) tma_prefetch_l2_2d(&tmB, kb * (BK / 2), bn_first);
  }
  grid_dependency_wait();
  grid_launch_dependents();
  uint16_t* gelu_win = reinterpret_cast<uint16_t*>(gbase + OFF_GELU);
  if (warp >= 2 && warp < 2 + kEpiWarps) {
    // the epilogue warps copy the table's window (no early exit precedes this barrier)
    for (int j = threadIdx.x - 64; j < static_cast<int>(2 * kGeluSpan); j += kEpiWarps * 32) {
      const uint32_t s = j >= static_cast<int>(kGeluSpan) ? 1u : 0u;
      gelu_win[j] = __ldg(p.gelu + ((s << 15) | (kGeluLo + static_cast<uint32_t>(j) - s * kGeluSpan)));
    }
    asm volatile("bar.sync 2, %0;" ::"n"(kEpiWarps * 32) : "memory");
  }

  constexpr uint32_t kHiSw128 = smem_desc_hi(1024, 2);
  constexpr uint32_t kHiSw64 = smem_desc_hi(512, 4);
  constexpr uint32_t kHiSf = smem_desc_hi(128, 0);
  constexpr uint32_t kLbo = 1u << 16;

  if (warp == 0) {
    // ------------------------------------------------------------------ producer (kernel 2's)
    uint32_t g = 0, it = 0;
    bool ok = true;
    for (int t = t_begin; ok && t < t_end; ++t) {
      const int mt = t / p.tiles_n, nt = t % p.tiles_n;
      const int m0 = mt * 256 + static_cast<int>(cta) * BM;
      const int n0 = nt * BN;
      const int bn0 = n0 + static_cast<int>(cta) * BN_HALF;
      const int rb = m0 / 128, nb = n0 / 128;
      for (int kb0 = 0; ok && kb0 <= nkb; ++it) {
        const int cnt = kb0 + 1 < nkb ? 2 : 1;
        const uint32_t fbar = full(it);
        const uint32_t fb = map_to_cta(fbar, 0);
        for (int c = 0; c < cnt; ++c) {
          const int kb = kb0 + c;
          const int s = g % S;
          const uint32_t ph = (g / S) & 1u;
          if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(empty(s), ph ^ 1u, abort_flag, 31))) { ok = false; break; }
          const uint32_t sb = base + s * STAGE_BYTES;
          if (elect_one()) {
            if (kb < nkb) {
              if (leader) mbar_arrive_expect_tx(fbar, TX_MAIN);
              tma_load_2d_pair(sb, &tmA, kb * (BK / 2), m0, fb);
              tma_load_2d_pair(sb + A_BYTES, &tmB, kb * (BK / 2), bn0, fb);
              tma_load_2d_pair(sb + A_BYTES + B_BYTES, &tmSFA, 0, rb * natoms + kb * (BK / 64), fb);
              tma_load_2d_pair(sb + A_BYTES + B_BYTES + SFA_BYTES, &tmSFB, 0, nb * natoms + kb * (BK / 64), fb);
            } else {
              if (leader) mbar_arrive_expect_tx(fbar, TX_LOWRANK);
              tma_load_2d_pair(sb, &tmU, 0, m0, fb);
              tma_load_2d_pair(sb + A_BYTES, &tmL2, 0, bn0, fb);
            }
            if (cnt == 1 && leader) mbar_arrive(fbar);
          }
          __syncwarp();
          ++g;
        }
        kb0 += cnt;
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (leader) {
      // ------------------------------------------------------------------ up-projection MMAs (kernel 2's)
      const uint32_t id4 = k2::idesc_nvfp4_m256<BN>();
      const uint32_t idb = k2::idesc_bf16_m256<BN>();
      uint32_t g = 0, it = 0;
      int i = 0;
      bool ok = true;
      for (int t = t_begin; ok && t < t_end; ++t, ++i) {
        const int b = i & 1;
        if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(acc_empty(b), ((i >> 1) & 1) ^ 1, abort_flag, 32))) break;
        tc_fence_after();
        const uint32_t dacc = tmem + static_cast<uint32_t>(b * BN);
        for (int kb = 0; kb <= nkb; ++it) {
          const int cnt = kb + 1 < nkb ? 2 : 1;
          if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(full(it), (it / NBF) & 1u, abort_flag, 33))) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (elect_one()) {
            for (int c = 0; c < cnt; ++c) {
              const uint32_t gg = g + c;
              const int kbb = kb + c;
              const int s = gg % S;
              const uint32_t sb = base + s * STAGE_BYTES;
              const uint32_t a_lo = (sb >> 4) | kLbo;
              const uint32_t b_lo = ((sb + A_BYTES) >> 4) | kLbo;
              if (kbb < nkb) {
                const int na = min(BK / 64, natoms - kbb * (BK / 64));
                const uint32_t sfa_lo = (sb + A_BYTES + B_BYTES) >> 4;
                const uint32_t sfb_lo = sfa_lo + SFA_BYTES / 16;
                const uint32_t tsf = tmem + TM_SF + (gg & 1u) * SF_COLS;
#pragma unroll
                for (int kk = 0; kk < BK / 64; ++kk) {
                  if (kk < na) {
                    tc_copy_32x128b_x4_pair(tsf + 4 * kk, make_desc(sfa_lo + kk * 32, kHiSf));
                    tc_copy_32x128b_x4_pair(tsf + SFB_OFF + kk * 4, make_desc(sfb_lo + kk * 32, kHiSf));
                  }
                }
#pragma unroll
                for (int kk = 0; kk < BK / 64; ++kk) {
                  if (kk < na)
                    umma_nvfp4_pair(dacc, make_desc(a_lo + kk * 2, kHiSw128), make_desc(b_lo + kk * 2, kHiSw128),
                                    id4, tsf + 4 * kk, tsf + SFB_OFF + kk * 4, (kbb | kk) != 0 ? 1u : 0u);
                }
              } else {
                const uint32_t l_lo = ((sb + A_BYTES) >> 4) | kLbo;
#pragma unroll
                for (int j = 0; j < 4; ++j)
                  umma_bf16_pair(dacc, make_desc(a_lo + j * 2, kHiSw128), make_desc(l_lo + (j & 1) * 2, kHiSw64),
                                 idb, 1u);
              }
              tc_commit_pair(empty(s), 0x3);
            }
            if (kb + cnt - 1 == nkb) tc_commit_pair(acc_full(b), 0x3);
          }
          __syncwarp();
          g += cnt;
          kb += cnt;
        }
      }
    }
    __syncwarp();
  } else if (warp == kLoadWarp) {
    // ------------------------------------------------------------------ low-rank factor tiles (both CTAs)
    // this CTA's 16 rank rows of (diag(smooth_inv) L1)^T, hi (rows 0-31 of the packed
    // section) and lo (rows 32-63), for the tile's two 64-column slabs
    int i = 0;
    for (int t = t_begin; t < t_end; ++t, ++i) {
      const int tb = i & 1;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(l1_free(tb), ((i >> 1) & 1) ^ 1, abort_flag, 34))) break;
      if (elect_one()) {
        const int n0 = (t % p.tiles_n) * BN;
        const uint32_t fb = map_to_cta(l1_full(tb), 0);
        const uint32_t dst = base + OFF_L1 + tb * L1BUF_BYTES;
        if (leader) mbar_arrive_expect_tx(l1_full(tb), TX_L1);
        const int r0 = static_cast<int>(cta) * 16;
#pragma unroll
        for (int s = 0; s < 2; ++s) {
          tma_load_2d_pair(dst + s * L1T_BYTES, &tmL1, n0 + 64 * s, r0, fb);
          tma_load_2d_pair(dst + (2 + s) * L1T_BYTES, &tmL1, n0 + 64 * s, 32 + r0, fb);
        }
      }
      __syncwarp();
    }
  } else if (warp == kUWarp) {
    if (leader) {
      // ------------------------------------------------------------------ low-rank MMAs of the down projection (leader)
      const uint32_t idu = idesc_u();
      int i = 0, parts = 0;
      bool ok = true;
      for (int t = t_begin; ok && t < t_end; ++t, ++i) {
        const int tb = i & 1;
        if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(l1_full(tb), (i >> 1) & 1, abort_flag, 35))) break;
        const uint32_t l1b = base + OFF_L1 + tb * L1BUF_BYTES;
        for (int s = 0; s < 2; ++s) {
          const int sn = 2 * i + s;
          const int buf = sn & 1;
          // the slab was written with generic stores by both CTAs: acquire at cluster scope
          if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded_cluster(slab_ready(buf), (sn >> 1) & 1, abort_flag, 36))) {
            ok = false;
            break;
          }
          const bool first = s == 0 && starts_part(t);
          if (first && parts > 0 &&
              !__all_sync(0xFFFFFFFFu, mbar_wait_bounded(u_empty, (parts - 1) & 1, abort_flag, 37))) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (elect_one()) {
            const uint32_t a_lo = ((base + OFF_SLAB + buf * SLAB_BYTES) >> 4) | kLbo;
            const uint32_t hi_lo = ((l1b + s * L1T_BYTES) >> 4) | kLbo;
            const uint32_t lo_lo = ((l1b + (2 + s) * L1T_BYTES) >> 4) | kLbo;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_bf16_pair(tmem + TM_U, make_desc(a_lo + kk * 2, kHiSw128), make_desc(hi_lo + kk * 2, kHiSw128),
                             idu, (first && kk == 0) ? 0u : 1u);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_bf16_pair(tmem + TM_U, make_desc(a_lo + kk * 2, kHiSw128), make_desc(lo_lo + kk * 2, kHiSw128),
                             idu, 1u);
            tc_commit_pair(slab_free(buf), 0x3);
            if (s == 1) {
              tc_commit_pair(l1_free(tb), 0x3);
              if (ends_part(t)) tc_commit_pair(u_full, 0x3);
            }
          }
          __syncwarp();
        }
        if (ends_part(t)) ++parts;
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ epilogue (both CTAs)
    const int quarter = warp & 3;
    const int ew = warp - 2;
    const int eh = ew >> 2;                        // chunks eh and eh + 2 of each tile
    const float alpha = p.alpha;
    uint8_t* svec = gbase + OFF_VEC + ew * VEC_BYTES;   // [0, 256): bias (bf16); [256, 768): -smooth_inv (fp32)
    const int r = quarter * 32 + lane;             // this thread's row within the CTA's 128
    int i = 0, parts = 0;
    for (int t = t_begin; t < t_end; ++t, ++i) {
      const int mt = t / p.tiles_n, nt = t % p.tiles_n;
      const int mblk = mt * 256 + static_cast<int>(cta) * BM;     // this CTA's first row
      const int m = mblk + r;
      const int n0 = nt * BN;
      const int b = i & 1;
      if (lane < 16)
        *reinterpret_cast<uint4*>(svec + lane * 16) = __ldg(reinterpret_cast<const uint4*>(p.bias + n0) + lane);
      {
        const uint2 sv = __ldg(reinterpret_cast<const uint2*>(p.smooth + n0) + lane);   // 4 factors per lane
        *reinterpret_cast<float4*>(svec + 256 + lane * 16) =
            make_float4(-bf16lo_to_f32(sv.x), -bf16hi_to_f32(sv.x), -bf16lo_to_f32(sv.y), -bf16hi_to_f32(sv.y));
      }
      __syncwarp();
      if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(acc_full(b), (i >> 1) & 1, abort_flag, 38))) break;
      tc_fence_after();
      const uint32_t trow = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(b * BN);
      uint32_t R[2][32];
      tmem_ld_32x32b_x32(trow + 32u * eh, R[0]);
      tmem_ld_32x32b_x32(trow + 32u * (eh + 2), R[1]);
      tmem_wait_ld_regs(R[0]);
      tmem_wait_ld_regs(R[1]);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(map_to_cta(acc_empty(b), 0));
      const bool block_live = mblk < p.M;          // the scale buffer holds this 128-row block
      bool ok = true;
      // First both chunks' h (table gathers) and their hand-over to the low-rank MMA, then the
      // quantization and the global stores: the slab's cluster-scope release arrival orders
      // every earlier write of the thread, and global stores still in flight would hold it up.
      uint32_t hw[2][16];
#pragma unroll
      for (int jj = 0; jj < 2; ++jj) {
        const int c = eh + 2 * jj;                 // chunk of the tile, in slab jj
        const uint4* bias4 = reinterpret_cast<const uint4*>(svec + c * 64);
        uint32_t yb[16];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint4 bv = bias4[q];
          const uint32_t bw[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            const int k = q * 8 + w * 2;
            const uint64_t y = f32x2_fma(f32x2_pack(alpha, alpha), f32x2_pack(__uint_as_float(R[jj][k]),
                                                                               __uint_as_float(R[jj][k + 1])),
                                         f32x2_pack(bf16lo_to_f32(bw[w]), bf16hi_to_f32(bw[w])));
            float y0, y1;
            f32x2_unpack(y, y0, y1);
            yb[q * 4 + w] = pack_bf16x2(y0, y1);
          }
        }
        // h = bf16(GELU(y)) for the 32 values from the shared-memory window; a warp with a
        // value outside it (|y| < 2^-31 or >= 256, or not finite) takes the full rule
        bool inside = true;
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const uint32_t tl = (yb[k] & 0x7FFFu) - kGeluLo, th = ((yb[k] >> 16) & 0x7FFFu) - kGeluLo;
          inside = inside && tl < kGeluSpan && th < kGeluSpan;
          const uint32_t il = ((yb[k] >> 15) & 1u) * kGeluSpan + min(tl, kGeluSpan - 1);
          const uint32_t ih = (yb[k] >> 31) * kGeluSpan + min(th, kGeluSpan - 1);
          hw[jj][k] = static_cast<uint32_t>(gelu_win[il]) | (static_cast<uint32_t>(gelu_win[ih]) << 16);
        }
        if (!__all_sync(0xFFFFFFFFu, inside)) {
#pragma unroll
          for (int k = 0; k < 16; ++k)
            hw[jj][k] = gelu_bf16_rule(yb[k] & 0xFFFFu, gelu_win) | (gelu_bf16_rule(yb[k] >> 16, gelu_win) << 16);
        }
      }
#pragma unroll
      for (int jj = 0; jj < 2; ++jj) {
        const int c = eh + 2 * jj;
        const int sn = 2 * i + jj;
        const int buf = sn & 1;
        // the slab must have been consumed by the low-rank MMAs two slabs back
        if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(slab_free(buf), ((sn >> 1) & 1) ^ 1, abort_flag, 39))) {
          ok = false;
          break;
        }
        const uint32_t row = base + OFF_SLAB + buf * SLAB_BYTES + static_cast<uint32_t>(r) * 128;
        const uint32_t sw = static_cast<uint32_t>(r & 7);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t u = static_cast<uint32_t>((c & 1) * 4 + q);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                       ::"r"(row + ((u ^ sw) << 4)), "r"(hw[jj][4 * q]), "r"(hw[jj][4 * q + 1]), "r"(hw[jj][4 * q + 2]),
                         "r"(hw[jj][4 * q + 3])
                       : "memory");
        }
        fence_proxy_async_smem();                  // the tensor core reads the slab through the async proxy
        __syncwarp();
        if (lane == 0) mbar_arrive_remote_cluster(map_to_cta(slab_ready(buf), 0));
      }
      if (!ok) break;
#pragma unroll
      for (int jj = 0; jj < 2; ++jj) {
        const int c = eh + 2 * jj;
        // the down projection's activation pass on h: -h smooth_inv in pairs, two 16-groups
        const uint64_t* sm2 = reinterpret_cast<const uint64_t*>(svec + 256 + c * 128);   // -smooth_inv pairs
        uint32_t sc2 = 0;
        uint2 cb[2];
#pragma unroll
        for (int gq = 0; gq < 2; ++gq) {
          uint64_t nx[8];
#pragma unroll
          for (int w = 0; w < 8; ++w) {
            const uint32_t hv = hw[jj][gq * 8 + w];
            nx[w] = f32x2_mul(f32x2_pack(bf16lo_to_f32(hv), bf16hi_to_f32(hv)), sm2[gq * 8 + w]);
          }
          sc2 |= quantize_group(nx, p.g, p.inv_g, cb[gq]) << (8 * gq);
        }
        const int col = n0 + 32 * c;
        if (m < p.M) {
          *reinterpret_cast<uint4*>(p.codes + static_cast<size_t>(m) * (p.N / 2) + col / 2) =
              make_uint4(cb[0].x, cb[0].y, cb[1].x, cb[1].y);
          if (p.h_out) {
            uint4* hd = reinterpret_cast<uint4*>(p.h_out + static_cast<size_t>(m) * p.N + col);
#pragma unroll
            for (int q = 0; q < 4; ++q)
              hd[q] = make_uint4(hw[jj][4 * q], hw[jj][4 * q + 1], hw[jj][4 * q + 2], hw[jj][4 * q + 3]);
          }
        }
        if (block_live) {                          // rows past M in the last block get zero scales
          uint8_t* sdst = p.scales + (static_cast<size_t>(mblk / 128) * (p.N / 64) + col / 64) * 512 +
                          (r % 32) * 16 + (r / 32) * 4 + (c & 1) * 2;
          *reinterpret_cast<uint16_t*>(sdst) = m < p.M ? static_cast<uint16_t>(sc2) : uint16_t(0);
        }
      }
      if (ends_part(t)) {
        // the pair's low-rank partial of this row block: one warp per lane quarter reads it out
        if (eh == 0) {
          if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(u_full, parts & 1, abort_flag, 40))) break;
          tc_fence_after();
          uint32_t u[32];
          tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(quarter * 32) << 16) + TM_U, u);
          tmem_wait_ld_regs(u);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_remote(map_to_cta(u_empty, 0));
          float4* dst = reinterpret_cast<float4*>(
              p.ws + ((static_cast<size_t>(pair) * p.slots + (mt - mt_first)) * 256 + cta * BM + r) * 32);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            dst[q] = make_float4(__uint_as_float(u[4 * q]), __uint_as_float(u[4 * q + 1]),
                                 __uint_as_float(u[4 * q + 2]), __uint_as_float(u[4 * q + 3]));
        }
        ++parts;
      }
    }
  }

  __syncthreads();
  if (*abort_flag) {
    if (warp == 1 && leader) {
      if (elect_one()) tc_commit_pair(drain, 0x1);
      __syncwarp();
      mbar_wait_bounded(drain, 0, nullptr, 41);
    }
    if (warp == 0 && lane == 0) {
      const uint64_t t0 = global_timer_ns();
      while (global_timer_ns() - t0 < 2000000ull) { }
    }
    __syncthreads();
  }
  tc_fence_before();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair<TMEM_COLS>(tmem);
  }
}

// Kernel 7: U[m] = sum of the partials of the pairs whose ranges cover row m's 256-row block, in
// pair order; written as U / g (exact: g a power of two) split into bf16 hi + lo.  One thread
// per (row, four ranks).
__global__ void __launch_bounds__(256)
u_reduce_kernel(const float* __restrict__ ws, int M, int tiles_n, int tiles, int npairs, int slots, float inv_g,
                __nv_bfloat16* __restrict__ ucat) {
  grid_dependency_wait();
  grid_launch_dependents();
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  const int m = idx >> 3;
  const int q = idx & 7;                           // ranks 4q .. 4q + 3
  if (m >= M) return;
  const int mt = m / 256, local = m % 256;
  const int t0 = mt * tiles_n, t1 = t0 + tiles_n - 1;
  auto pair_of = [&](int t) {
    int pp = static_cast<int>((static_cast<long long>(t) * npairs) / tiles);
    while (pp > 0 && range_start(pp, tiles, npairs) > t) --pp;
    while (pp + 1 < npairs && range_start(pp + 1, tiles, npairs) <= t) ++pp;
    return pp;
  };
  const int p0 = pair_of(t0), p1 = pair_of(t1);
  float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int pp = p0; pp <= p1; ++pp) {
    const int slot = mt - range_start(pp, tiles, npairs) / tiles_n;
    const float4 v = *reinterpret_cast<const float4*>(ws + ((static_cast<size_t>(pp) * slots + slot) * 256 + local) * 32 + 4 * q);
    s.x += v.x; s.y += v.y; s.z += v.z; s.w += v.w;
  }
  const float uu[4] = {s.x * inv_g, s.y * inv_g, s.z * inv_g, s.w * inv_g};
  uint32_t hw[2], lw[2];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const float h0 = __bfloat162float(__float2bfloat16_rn(uu[2 * j]));
    const float h1 = __bfloat162float(__float2bfloat16_rn(uu[2 * j + 1]));
    hw[j] = pack_bf16x2(h0, h1);
    lw[j] = pack_bf16x2(uu[2 * j] - h0, uu[2 * j + 1] - h1);
  }
  __nv_bfloat16* dst = ucat + static_cast<size_t>(m) * 64 + 4 * q;
  *reinterpret_cast<uint2*>(dst) = make_uint2(hw[0], hw[1]);
  *reinterpret_cast<uint2*>(dst + 32) = make_uint2(lw[0], lw[1]);
}

}  // namespace k6
}  // namespace svdq
