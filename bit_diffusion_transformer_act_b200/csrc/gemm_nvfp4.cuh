// Kernel 2: NVFP4 block-scaled GEMM on tcgen05 with the SVDQuant epilogue.
//
//   Y = bf16( alpha * (Q(X_hat) Q(R)^T) + U L2 + b ),  alpha = g_a g_w
//
// Method: "Nunchaku Lite" docs, "Supported quantization types" (svdq_w4a4,
// nvfp4, group 16: an NVFP4 runtime kernel with an SVDQ low-rank correction);
// the Nunchaku Lite article: the low-rank branch is 16-bit.
//
// Design (sm_100a, one 128 x BN output tile per CTA, 192 threads):
//   warp 0  TMA producer: E2M1 code tiles of A (activations) and B (weights)
//           through a 3-stage ring of 128-byte-swizzled shared-memory tiles
//           (256 K elements per stage), their E4M3 scale atoms by bulk copy,
//           and once per tile the low-rank activation tile [128 x 64] (bf16 hi | lo of
//           U / g_a) and the (L2 / g_w)^T tile [BN x 32].
//   warp 1  allocates tensor memory and issues, from one thread, the scale
//           copies (tcgen05.cp, shared -> tensor memory, 4 columns per 128 rows
//           per MMA) and the block-scaled MMAs
//           (kind::mxf4nvf4, block16 = one UE4M3 scale per 16 K, K = 64 per
//           instruction, fp32 accumulator in tensor memory); after the K loop,
//           four bf16 MMAs (K = 16 each) add [U_hi | U_lo] [L2 | L2]^T / (g_a g_w)
//           into the same accumulator (both operands were pre-scaled by powers of
//           two, so the accumulator ends as Acc + U L2 / alpha exactly).
//   warps 2-5  epilogue: read the accumulator from tensor memory (32 columns
//           per tcgen05.ld), apply alpha and the bias with one fma, round to
//           bf16 and store.
// Every mbarrier wait is bounded (about one second); a wait that runs out
// records SVDQ_ERR_TIMEOUT in the device status word, makes the other roles
// give up, drains the copies and MMAs in flight (bounded too), frees the
// tensor memory and returns.
#pragma once

#include "ptx.cuh"

namespace svdq {
namespace k2 {

constexpr int BM = 128;
constexpr int BK = 256;                    // K elements per pipeline stage
constexpr int kStages = 3;
constexpr int kThreads = 192;

template <int BN>
struct Cfg {
  static constexpr int A_BYTES = BM * BK / 2;
  static constexpr int B_BYTES = BN * BK / 2;
  static constexpr int SFA_BYTES = (BM / 128) * (BK / 64) * 512;
  static constexpr int SFB_BYTES = (BN / 128) * (BK / 64) * 512;
  static constexpr int UCAT_BYTES = BM * 64 * 2;       // bf16 [hi | lo] of U / g_a (rows of 128 B)
  static constexpr int L2_BYTES = BN * 32 * 2;
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + kStages * A_BYTES;
  static constexpr int OFF_SFA = OFF_B + kStages * B_BYTES;
  static constexpr int OFF_SFB = OFF_SFA + kStages * SFA_BYTES;
  static constexpr int OFF_UCAT = OFF_SFB + kStages * SFB_BYTES;
  static constexpr int OFF_L2 = OFF_UCAT + UCAT_BYTES;
  static constexpr int OFF_BAR = OFF_L2 + L2_BYTES;
  static constexpr int NUM_BARS = 2 * kStages + 4;   // full, empty, lr_loaded, lr_ready, acc_full, drain
  static constexpr int OFF_MISC = OFF_BAR + 8 * NUM_BARS;
  static constexpr int SMEM_BYTES = OFF_MISC + 64 + 1024;   // + slack to align the base to 1024
  // tensor memory columns: accumulator [0, BN), scale factors of A (4 per MMA), of B (4 per 128 rows per MMA)
  static constexpr uint32_t TM_SFA = BN;
  static constexpr uint32_t TM_SFB = BN + 4 * (BK / 64);
  static constexpr int TM_USED = BN + 4 * (BK / 64) + 4 * (BN / 128) * (BK / 64);
  static constexpr int TMEM_COLS = TM_USED <= 256 ? 256 : 512;
  static_assert(TM_USED <= 512, "tensor memory overflow");
  static_assert(OFF_UCAT % 1024 == 0 && OFF_L2 % 1024 == 0, "alignment");
};

struct Params {
  const uint8_t* sfa;              // activation scales, swizzled, rows padded to 128
  const uint8_t* sfb;              // weight scales, swizzled
  const __nv_bfloat16* bias;       // [N]
  __nv_bfloat16* Y;                // [M, N]
  int M, N, K;
  float alpha;
};

// Instruction descriptors (tcgen05 "instruction descriptor" bit fields).
// Block-scaled: bits 7-9 A type (1 = E2M1), 10-12 B type (1 = E2M1), 15/16 A/B
// major (0 = K), 17-22 N >> 3, 23 scale type (0 = UE4M3), 24-28 M >> 4.
template <int BN>
__device__ __forceinline__ uint32_t idesc_nvfp4() {
  return (1u << 7) | (1u << 10) | (static_cast<uint32_t>(BN >> 3) << 17) | (static_cast<uint32_t>(BM >> 4) << 24);
}
// kind::f16: bits 4-5 D type (1 = f32), 7-9 A type (1 = bf16), 10-12 B type (1 = bf16).
template <int BN>
__device__ __forceinline__ uint32_t idesc_bf16() {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(BN >> 3) << 17) |
         (static_cast<uint32_t>(BM >> 4) << 24);
}

template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
nvfp4_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                  const __grid_constant__ CUtensorMap tmU, const __grid_constant__ CUtensorMap tmL2,
                  const Params p) {
  using C = Cfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);

  const uint32_t bars = base + C::OFF_BAR;
  auto full = [&](int s) { return bars + 8u * s; };
  auto empty = [&](int s) { return bars + 8u * (kStages + s); };
  const uint32_t lr_loaded = bars + 8u * (2 * kStages);
  const uint32_t lr_ready = lr_loaded + 8u;
  const uint32_t acc_full = lr_loaded + 16u;
  const uint32_t drain = lr_loaded + 24u;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + C::OFF_MISC + 4);
  volatile int* consumed_out = reinterpret_cast<volatile int*>(gbase + C::OFF_MISC + 8);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int n0 = blockIdx.x * BN;
  const int mblk = blockIdx.y;
  const int m0 = mblk * BM;
  const int natoms = p.K / 64;                       // 64-K scale atoms per row block
  const int nkb = (p.K + BK - 1) / BK;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < kStages; ++s) { mbar_init(full(s), 1); mbar_init(empty(s), 1); }
    mbar_init(lr_loaded, 1);
    mbar_init(lr_ready, 1);                         // unused
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    *consumed_out = 0;
    fence_mbar_init();
    prefetch_tmap(&tmA); prefetch_tmap(&tmB); prefetch_tmap(&tmU); prefetch_tmap(&tmL2);
  }
  if (warp == 1) tmem_alloc<C::TMEM_COLS>(smem_addr(tmem_slot));
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  int issued = 0;
  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------------- producer
      mbar_arrive_expect_tx(lr_loaded, C::UCAT_BYTES + C::L2_BYTES);
      tma_load_2d(base + C::OFF_UCAT, &tmU, 0, m0, lr_loaded);
      tma_load_2d(base + C::OFF_L2, &tmL2, 0, n0, lr_loaded);
      for (int kb = 0; kb < nkb; ++kb) {
        const int s = kb % kStages, it = kb / kStages;
        if (!mbar_wait_bounded(empty(s), (it & 1) ^ 1, abort_flag, 1)) break;
        const int na = min(BK / 64, natoms - kb * (BK / 64));
        const uint32_t bytes = C::A_BYTES + C::B_BYTES + na * 512u * (1u + BN / 128);
        mbar_arrive_expect_tx(full(s), bytes);
        tma_load_2d(base + C::OFF_A + s * C::A_BYTES, &tmA, kb * (BK / 2), m0, full(s));
        tma_load_2d(base + C::OFF_B + s * C::B_BYTES, &tmB, kb * (BK / 2), n0, full(s));
        bulk_load(base + C::OFF_SFA + s * C::SFA_BYTES,
                  p.sfa + (static_cast<size_t>(mblk) * natoms + kb * (BK / 64)) * 512, na * 512u, full(s));
#pragma unroll
        for (int nb = 0; nb < BN / 128; ++nb)
          bulk_load(base + C::OFF_SFB + s * C::SFB_BYTES + nb * (BK / 64) * 512,
                    p.sfb + (static_cast<size_t>(n0 / 128 + nb) * natoms + kb * (BK / 64)) * 512, na * 512u,
                    full(s));
        ++issued;
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------------------- MMA issuer
      const uint32_t id4 = idesc_nvfp4<BN>();
      int done = 0;
      for (int kb = 0; kb < nkb; ++kb) {
        const int s = kb % kStages, it = kb / kStages;
        if (!mbar_wait_bounded(full(s), it & 1, abort_flag, 2)) break;
        tc_fence_after();
        const int na = min(BK / 64, natoms - kb * (BK / 64));
        const uint32_t sfa_s = base + C::OFF_SFA + s * C::SFA_BYTES;
        const uint32_t sfb_s = base + C::OFF_SFB + s * C::SFB_BYTES;
        for (int kk = 0; kk < na; ++kk) {
          tc_copy_32x128b_x4(tmem + C::TM_SFA + 4 * kk, smem_desc(sfa_s + kk * 512, 0, 128, 0));
#pragma unroll
          for (int nb = 0; nb < BN / 128; ++nb)
            tc_copy_32x128b_x4(tmem + C::TM_SFB + (kk * (BN / 128) + nb) * 4,
                               smem_desc(sfb_s + (nb * (BK / 64) + kk) * 512, 0, 128, 0));
        }
        const uint32_t a_s = base + C::OFF_A + s * C::A_BYTES;
        const uint32_t b_s = base + C::OFF_B + s * C::B_BYTES;
        for (int kk = 0; kk < na; ++kk) {
          // K-major, 128-byte swizzle: rows of 128 B, 8-row groups 1024 B apart; K step = 32 B
          const uint64_t ad = smem_desc(a_s + kk * 32, 16, 1024, 2);
          const uint64_t bd = smem_desc(b_s + kk * 32, 16, 1024, 2);
          umma_nvfp4(tmem, ad, bd, id4, tmem + C::TM_SFA + 4 * kk, tmem + C::TM_SFB + kk * (BN / 128) * 4,
                     (kb | kk) != 0 ? 1u : 0u);
        }
        tc_commit(empty(s));
        ++done;
      }
      *consumed_out = done;
      if (done == nkb && mbar_wait_bounded(lr_loaded, 0, abort_flag, 3)) {
        tc_fence_after();
        const uint32_t idb = idesc_bf16<BN>();
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          // A: [U'_hi | U'_lo], K-major, 128-byte swizzle (rows of 64 bf16); B: L2^T, K-major,
          // 64-byte swizzle (rows of 32 bf16), K steps 0, 16, 0, 16.  K step = 16 bf16 = 32 B.
          const uint64_t ud = smem_desc(base + C::OFF_UCAT + j * 32, 16, 1024, 2);
          const uint64_t ld = smem_desc(base + C::OFF_L2 + (j & 1) * 32, 16, 512, 4);
          umma_bf16(tmem, ud, ld, idb, 1u);
        }
        tc_commit(acc_full);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ epilogue

    const int quarter = warp & 3;                    // tensor-memory lanes 32*quarter .. +31
    const int row = quarter * 32 + lane;
    const int m = m0 + row;
    if (mbar_wait_bounded(acc_full, 0, abort_flag, 5)) {
      tc_fence_after();
      const uint32_t trow = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
      for (int c0 = 0; c0 < BN; c0 += 32) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(trow + c0, r);
        tmem_wait_ld();
        if (m < p.M) {
          const uint4* bp = reinterpret_cast<const uint4*>(p.bias + n0 + c0);
          uint4 out[4];
          uint32_t* o = reinterpret_cast<uint32_t*>(out);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint4 bv = __ldg(bp + i);
            const uint32_t* b = reinterpret_cast<const uint32_t*>(&bv);
#pragma unroll
            for (int t = 0; t < 4; ++t) {
              const int j = i * 8 + t * 2;
              const float lo = fmaf(p.alpha, __uint_as_float(r[j]), bf16lo_to_f32(b[t]));
              const float hi = fmaf(p.alpha, __uint_as_float(r[j + 1]), bf16hi_to_f32(b[t]));
              o[i * 4 + t] = pack_bf16x2(lo, hi);
            }
          }
          uint4* dst = reinterpret_cast<uint4*>(p.Y + static_cast<size_t>(m) * p.N + n0 + c0);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = out[i];
        }
      }
    }
    tc_fence_before();
  }

  __syncthreads();
  if (*abort_flag) {
    // a wait ran out: let the MMAs and copies already issued finish before the memory goes away
    if (warp == 1) {
      if (lane == 0) { tc_commit(drain); mbar_wait_bounded(drain, 0, nullptr, 6); }
      __syncwarp();
    } else if (warp == 0) {
      if (lane == 0) {
        for (int i = *consumed_out; i < issued; ++i)
          mbar_wait_bounded(full(i % kStages), (i / kStages) & 1, nullptr, 7);
      }
      __syncwarp();
    }
    __syncthreads();
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc<C::TMEM_COLS>(tmem);
  }
}

}  // namespace k2
}  // namespace svdq
