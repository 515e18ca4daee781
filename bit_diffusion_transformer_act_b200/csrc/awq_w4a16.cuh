// Kernel 3: AWQ-style W4A16 linear, int4 weights with a bf16 scale and an
// integer zero point per (output row, group of 64 along K):
//
//   y[m, n] = sum_g s[n, g] * sum_{k in g} (q[n, k] - z[n, g]) x[m, k]  (+ b[n])
//
// Method: "Nunchaku Lite" docs, "Supported quantization types" (awq_w4a16 /
// int4 / group 64, an AWQ-style INT4 weight-only kernel); the Nunchaku Lite
// article: used for the adaptive-normalisation layers, activations stay 16-bit.
//
// Design (sm_100a, memory-bound at small M).  A CTA owns 64 output rows (four
// warps of 16) and all M <= 64 tokens, and streams its 64 x K/2 bytes of
// packed weights exactly once through a 4-stage cp.async ring (256 K per
// stage, 16-byte pieces XOR-swizzled against bank conflicts); the token
// activations ride along in the same stages (they are shared by all CTAs and
// come from L2).  The weights are the A operand of mma.sync m16n8k16 (swap-AB:
// 16 weight rows x 8 tokens), dequantized in registers: a nibble q becomes the
// bf16 128+q by bit placement, and one packed subtraction of 128+z gives q - z
// exactly, so every product (q - z) x is exact and each group's fp32 partial
// sum is scaled by s once.  Inside every 32-K step the K order is permuted
// (the same permutation for A and B): lane quad position p takes real K
// elements 8p..8p+7, i.e. one 32-bit word of nibbles per weight row and one
// 16-byte load of activations per token tile.
#pragma once

#include "ptx.cuh"

namespace svdq {
namespace k3 {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kRows = 64;                  // output rows (weight rows) per CTA
constexpr int kChunk = 256;                // K per stage
constexpr int kStages = 4;
constexpr int kGroup = 64;

template <int NT>
struct __align__(128) Smem {
  uint8_t w[kStages][kRows * 128];                 // 64 rows x 128 B (256 nibbles)
  __nv_bfloat16 x[kStages][NT * 8 * kChunk];       // NT*8 token rows x 512 B
  __nv_bfloat16 sc[kStages][kRows * 4];            // 4 groups per stage
  __nv_bfloat16 zr[kStages][kRows * 4];
};

struct Params {
  const __nv_bfloat16* X;          // [M, K]
  const uint8_t* qw;               // [N, K/2]
  const __nv_bfloat16* scales;     // [N, K/64]
  const __nv_bfloat16* zeros;      // [N, K/64]
  const __nv_bfloat16* bias;       // [N] or null
  __nv_bfloat16* Y;                // [M, N]
  int M, N, K;
};

__device__ __forceinline__ void cp_async_8(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(dst), "l"(reinterpret_cast<uint64_t>(src)) : "memory");
}

template <int NT>
__device__ __forceinline__ void load_stage(Smem<NT>& s, int st, const Params& p, int n0, int kb) {
  const int tid = threadIdx.x;
  const int kc = kb * kChunk;
  const uint32_t wb = smem_addr(s.w[st]);
  for (int i = tid; i < kRows * 8; i += kThreads) {
    const int r = i >> 3, pc = i & 7;
    cp_async_16(wb + r * 128 + ((pc ^ (r & 7)) << 4),
                p.qw + static_cast<size_t>(n0 + r) * (p.K / 2) + kc / 2 + pc * 16, 16u);
  }
  const uint32_t xb = smem_addr(s.x[st]);
  for (int i = tid; i < NT * 8 * 32; i += kThreads) {
    const int r = i >> 5, pc = i & 31;
    const bool ok = r < p.M;
    const __nv_bfloat16* src = p.X + (ok ? static_cast<size_t>(r) * p.K + kc + pc * 8 : 0);
    cp_async_16(xb + r * 512 + ((pc ^ (r & 7)) << 4), src, ok ? 16u : 0u);
  }
  const int gpr = p.K / kGroup;                    // groups per weight row
  if (tid < kRows) {
    cp_async_8(smem_addr(&s.sc[st][tid * 4]), p.scales + static_cast<size_t>(n0 + tid) * gpr + kb * 4);
  } else {
    const int r = tid - kRows;
    cp_async_8(smem_addr(&s.zr[st][r * 4]), p.zeros + static_cast<size_t>(n0 + r) * gpr + kb * 4);
  }
  cp_async_commit();
}

// bf16x2 {128 + nibble of byte b of lo-word, 128 + nibble of byte b of hi-word}
__device__ __forceinline__ uint32_t nib_pair(uint32_t lo_nibs, uint32_t hi_nibs, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(lo_nibs), "r"(hi_nibs), "r"(sel));
  return (r & 0x00FF00FFu) | 0x43004300u;
}

__device__ __forceinline__ uint32_t bf16x2_sub(uint32_t a, uint32_t b) {
  __nv_bfloat162 r = __hsub2(*reinterpret_cast<__nv_bfloat162*>(&a), *reinterpret_cast<__nv_bfloat162*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}

template <int NT>
__global__ void __launch_bounds__(kThreads)
awq_gemm_kernel(const Params p) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  Smem<NT>& s = *reinterpret_cast<Smem<NT>*>(smem_raw);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int g = lane >> 2, q = lane & 3;
  const int n0 = blockIdx.x * kRows;
  const int nkb = p.K / kChunk;
  const int rg = warp * 16 + g;                    // this lane's weight rows: rg and rg + 8

  float tot[NT][4];
#pragma unroll
  for (int j = 0; j < NT; ++j)
#pragma unroll
    for (int t = 0; t < 4; ++t) tot[j][t] = 0.f;

#pragma unroll
  for (int i = 0; i < kStages - 1; ++i) {
    if (i < nkb) load_stage<NT>(s, i, p, n0, i);
    else cp_async_commit();
  }

  for (int kb = 0; kb < nkb; ++kb) {
    cp_async_wait<kStages - 2>();
    __syncthreads();
    {
      const int nx = kb + kStages - 1;
      if (nx < nkb) load_stage<NT>(s, nx % kStages, p, n0, nx);
      else cp_async_commit();
    }
    const int st = kb % kStages;
    const uint8_t* wrow_g = s.w[st] + rg * 128;
    const uint8_t* wrow_h = s.w[st] + (rg + 8) * 128;
    const uint8_t* xs = reinterpret_cast<const uint8_t*>(s.x[st]);

#pragma unroll
    for (int grp = 0; grp < 4; ++grp) {
      const float sg = __bfloat162float(s.sc[st][rg * 4 + grp]);
      const float sh = __bfloat162float(s.sc[st][(rg + 8) * 4 + grp]);
      const float zg = __bfloat162float(s.zr[st][rg * 4 + grp]) + 128.f;
      const float zh = __bfloat162float(s.zr[st][(rg + 8) * 4 + grp]) + 128.f;
      const uint32_t zzg = pack_bf16x2(zg, zg), zzh = pack_bf16x2(zh, zh);

      float ga[NT][4];
#pragma unroll
      for (int j = 0; j < NT; ++j)
#pragma unroll
        for (int t = 0; t < 4; ++t) ga[j][t] = 0.f;

#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int t32 = grp * 2 + half;            // 32-K step within the stage (16-B piece index)
        const uint32_t wg = *reinterpret_cast<const uint32_t*>(wrow_g + ((t32 ^ (rg & 7)) << 4) + 4 * q);
        const uint32_t wh = *reinterpret_cast<const uint32_t*>(wrow_h + ((t32 ^ ((rg + 8) & 7)) << 4) + 4 * q);
        const uint32_t lg = wg & 0x0F0F0F0Fu, hg = (wg >> 4) & 0x0F0F0F0Fu;
        const uint32_t lh = wh & 0x0F0F0F0Fu, hh = (wh >> 4) & 0x0F0F0F0Fu;
        // pair b (real K elements 8q + 2b, 8q + 2b + 1) = byte b: selector puts lo byte b at 0, hi byte b at 2
        uint32_t A[2][4];
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
          // result byte 0 <- byte 2ks of lo (a), result byte 2 <- byte 2ks of hi (b = source bytes 4..7)
          const uint32_t sel0 = static_cast<uint32_t>(2 * ks) | (static_cast<uint32_t>(4 + 2 * ks) << 8);
          const uint32_t sel1 = static_cast<uint32_t>(2 * ks + 1) | (static_cast<uint32_t>(5 + 2 * ks) << 8);
          A[ks][0] = bf16x2_sub(nib_pair(lg, hg, sel0), zzg);   // row g,   logical k 2q, 2q+1
          A[ks][1] = bf16x2_sub(nib_pair(lh, hh, sel0), zzh);   // row g+8
          A[ks][2] = bf16x2_sub(nib_pair(lg, hg, sel1), zzg);   // row g,   logical k 2q+8, 2q+9
          A[ks][3] = bf16x2_sub(nib_pair(lh, hh, sel1), zzh);
        }
#pragma unroll
        for (int j = 0; j < NT; ++j) {
          const int tr = 8 * j + g;                  // token row
          const uint4 xv = *reinterpret_cast<const uint4*>(xs + tr * 512 + (((4 * t32 + q) ^ (tr & 7)) << 4));
          mma_bf16_16816(ga[j], A[0][0], A[0][1], A[0][2], A[0][3], xv.x, xv.y);
          mma_bf16_16816(ga[j], A[1][0], A[1][1], A[1][2], A[1][3], xv.z, xv.w);
        }
      }
#pragma unroll
      for (int j = 0; j < NT; ++j) {
        tot[j][0] = fmaf(sg, ga[j][0], tot[j][0]);
        tot[j][1] = fmaf(sg, ga[j][1], tot[j][1]);
        tot[j][2] = fmaf(sh, ga[j][2], tot[j][2]);
        tot[j][3] = fmaf(sh, ga[j][3], tot[j][3]);
      }
    }
  }
  cp_async_wait<0>();

  // D fragment: c0 (row g, token 2q), c1 (row g, token 2q+1), c2/c3 the same for row g+8
  const int na = n0 + rg, nb = na + 8;
  const float ba = p.bias ? __bfloat162float(p.bias[na]) : 0.f;
  const float bb = p.bias ? __bfloat162float(p.bias[nb]) : 0.f;
#pragma unroll
  for (int j = 0; j < NT; ++j) {
    const int t0 = 8 * j + 2 * q, t1 = t0 + 1;
    if (t0 < p.M) {
      p.Y[static_cast<size_t>(t0) * p.N + na] = __float2bfloat16_rn(tot[j][0] + ba);
      p.Y[static_cast<size_t>(t0) * p.N + nb] = __float2bfloat16_rn(tot[j][2] + bb);
    }
    if (t1 < p.M) {
      p.Y[static_cast<size_t>(t1) * p.N + na] = __float2bfloat16_rn(tot[j][1] + ba);
      p.Y[static_cast<size_t>(t1) * p.N + nb] = __float2bfloat16_rn(tot[j][3] + bb);
    }
  }
}

}  // namespace k3
}  // namespace svdq
