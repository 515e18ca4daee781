// Kernel 1: activation smoothing, NVFP4 quantization and the rank-32
// down-projection, in one pass over X.
//
// Method ("Nunchaku Lite" docs, "Supported quantization types": svdq_w4a4 /
// nvfp4 / group 16; the Nunchaku Lite article: outliers go to a 16-bit
// low-rank branch): X_hat = X * smooth_inv; per 16 K elements one E4M3 scale
// S = RNE(amax / (6 g_a)) and E2M1 codes RNE(clamp(X_hat / (S g_a))); and
// U = X_hat L1 (rank 32, fp32) from the same smoothed values.
//
// Design (sm_100a).  A CTA owns 64 rows and one K slice; the K slices of a row
// block form a thread-block cluster (1..8 CTAs) so the grid fills the 148 SMs
// even for a few thousand rows, and the partial U of the slices is summed over
// distributed shared memory -- no global scratch, no atomics.  X and L1 chunks
// of 128 columns are double-buffered in shared memory with cp.async (rows past
// M are zero-filled), the four warps each read their 16 x 16 tiles with
// ldmatrix straight into the mma.sync A-fragment layout, and all the per-element
// work happens on those registers: smoothing in fp32 (the product of two bf16
// values is exact), the group amax with two xor-shuffles inside each lane
// quad, the scale, the codes and the bf16 A operand of the low-rank mma.
//
// Rounding: the scale uses a correctly rounded quotient amax/6 (x 1/g_a, a
// power of two), converted with cvt.rn.satfinite.e4m3x2.  Codes use
// q = x_hat / (S g_a) correctly rounded by one Markstein correction step
// (q0 = x r, e = fma(-q0, D, x), q = fma(e, r, q0) with r = RN(1/D)), then
// cvt.rn.satfinite.e2m1x2.  A quotient that is not exactly a rounding
// midpoint sits 2^-16 (relative) or more away from one, far above fp32
// rounding, and an exact midpoint comes out exact, so the codes equal those of
// exact arithmetic.  The sign of q is copied from x_hat (negative zero stays
// negative).
#pragma once

#include "ptx.cuh"

namespace svdq {
namespace k1 {

constexpr int kRows = 64;                 // rows per CTA
constexpr int kWarps = 4;                 // 16 rows each
constexpr int kThreads = kWarps * 32;
constexpr int kChunk = 128;               // K columns per pipeline chunk
constexpr int kRank = 32;
constexpr int kCodeStride = 80;          // bytes per staged code row (64 used; 80 spreads banks)

struct __align__(128) Smem {
  __nv_bfloat16 x[2][kRows * kChunk];     // rows of 256 B, 16-B pieces XOR-swizzled by (row & 7)
  __nv_bfloat16 l1[2][kRank * kChunk];    // L1^T chunk, same swizzle
  __nv_bfloat16 smooth[2][kChunk];
  uint8_t codes[kWarps][16 * kCodeStride];
  float upart[kRows * kRank];             // this CTA's partial U (fp32)
};

// Byte offset of element (row, col) in a swizzled [rows][128] bf16 chunk.
__device__ __forceinline__ uint32_t swz(int row, int col) {
  return static_cast<uint32_t>(row * 256 + ((((col >> 3) ^ (row & 7)) << 4)) + ((col & 7) << 1));
}

struct Params {
  const __nv_bfloat16* X;          // [M, K]
  const __nv_bfloat16* smooth;     // [K]
  const __nv_bfloat16* l1t;        // [32, K]
  uint8_t* codes;                  // [M, K/2]
  uint8_t* scales;                 // swizzled
  float* U;                        // [M, 32]
  int M, K;
  int kslices;                     // cluster size along K
  float g;                         // per-tensor scale (power of two)
  float inv_g;
};

__device__ __forceinline__ void load_chunk(Smem& s, int buf, const Params& p, int m0, int kc, int ncols) {
  const int tid = threadIdx.x;
  const int pieces = ncols / 8;                       // 16-B pieces per row
  const uint32_t xbase = smem_addr(s.x[buf]);
  for (int i = tid; i < kRows * pieces; i += kThreads) {
    const int r = i / pieces, c = (i % pieces) * 8;
    const int m = m0 + r;
    const bool ok = m < p.M;
    const __nv_bfloat16* src = p.X + (ok ? (static_cast<size_t>(m) * p.K + kc + c) : 0);
    cp_async_16(xbase + swz(r, c), src, ok ? 16u : 0u);
  }
  const uint32_t lbase = smem_addr(s.l1[buf]);
  for (int i = tid; i < kRank * pieces; i += kThreads) {
    const int r = i / pieces, c = (i % pieces) * 8;
    cp_async_16(lbase + swz(r, c), p.l1t + static_cast<size_t>(r) * p.K + kc + c, 16u);
  }
  if (tid < pieces) cp_async_16(smem_addr(&s.smooth[buf][tid * 8]), p.smooth + kc + tid * 8, 16u);
  cp_async_commit();
}

// Scale code for one group given its amax (fp32).
__device__ __forceinline__ float group_scale_arg(float amax, float inv_g) {
  return __fdiv_rn(amax, 6.0f) * inv_g;
}

// a = hi + lo exactly for each of the two values (hi = RN_bf16(a), lo = RN_bf16(a - hi), and
// a - hi fits in bf16 whenever a has at most 16 significant bits).
__device__ __forceinline__ void split_bf16x2(float a0, float a1, uint32_t& hi, uint32_t& lo) {
  hi = pack_bf16x2(a0, a1);
  lo = pack_bf16x2(a0 - bf16lo_to_f32(hi), a1 - bf16hi_to_f32(hi));
}

__device__ __forceinline__ float quotient(float x, float D, float r) {
  const float q0 = x * r;
  const float e = fmaf(-q0, D, x);
  const float q = fmaf(e, r, q0);
  return __uint_as_float((__float_as_uint(q) & 0x7FFFFFFFu) | (__float_as_uint(x) & 0x80000000u));
}

__global__ void __launch_bounds__(kThreads)
quant_act_lowrank_kernel(const Params p) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  Smem& s = *reinterpret_cast<Smem*>(smem_raw);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int g = lane / 4, q = lane % 4;
  const int m0 = blockIdx.x * kRows;
  const int slice = blockIdx.y;
  const int klen = p.K / p.kslices;
  const int kbeg = slice * klen;
  const int nchunks = (klen + kChunk - 1) / kChunk;

  float acc[4][4];
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int t = 0; t < 4; ++t) acc[j][t] = 0.f;

  load_chunk(s, 0, p, m0, kbeg, min(kChunk, klen));

  for (int ci = 0; ci < nchunks; ++ci) {
    const int buf = ci & 1;
    const int kc = kbeg + ci * kChunk;
    const int ncols = min(kChunk, kbeg + klen - kc);
    if (ci + 1 < nchunks) {
      const int kn = kc + kChunk;
      load_chunk(s, buf ^ 1, p, m0, kn, min(kChunk, kbeg + klen - kn));
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();

    const uint32_t xbase = smem_addr(s.x[buf]);
    const uint32_t lbase = smem_addr(s.l1[buf]);
    const uint32_t* sm32 = reinterpret_cast<const uint32_t*>(s.smooth[buf]);
    uint8_t* cst = s.codes[warp];
    uint32_t sc_g = 0, sc_h = 0;                     // scale bytes of rows g and g+8 for the current 64-K atom

    const int steps = ncols / 16;
    for (int st = 0; st < steps; ++st) {
      // A fragment: rows 16w + {g, g+8}, columns 16 st + {2q, 2q+1, 2q+8, 2q+9}
      uint32_t a0, a1, a2, a3;
      {
        const int mi = lane >> 3;
        const int row = warp * 16 + (lane & 7) + ((mi & 1) << 3);
        const int col = st * 16 + ((mi >> 1) << 3);
        ldmatrix_x4(xbase + swz(row, col), a0, a1, a2, a3);
      }
      const uint32_t sp0 = sm32[(st * 16 + 2 * q) >> 1];
      const uint32_t sp1 = sm32[(st * 16 + 8 + 2 * q) >> 1];
      const float s0 = bf16lo_to_f32(sp0), s1 = bf16hi_to_f32(sp0);
      const float s8 = bf16lo_to_f32(sp1), s9 = bf16hi_to_f32(sp1);
      // row g: a0 (k 2q, 2q+1), a2 (k 2q+8, 2q+9); row g+8: a1, a3
      const float x0 = bf16lo_to_f32(a0) * s0, x1 = bf16hi_to_f32(a0) * s1;
      const float x2 = bf16lo_to_f32(a2) * s8, x3 = bf16hi_to_f32(a2) * s9;
      const float y0 = bf16lo_to_f32(a1) * s0, y1 = bf16hi_to_f32(a1) * s1;
      const float y2 = bf16lo_to_f32(a3) * s8, y3 = bf16hi_to_f32(a3) * s9;

      float mx = fmaxf(fmaxf(fabsf(x0), fabsf(x1)), fmaxf(fabsf(x2), fabsf(x3)));
      float my = fmaxf(fmaxf(fabsf(y0), fabsf(y1)), fmaxf(fabsf(y2), fabsf(y3)));
      mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 1));
      my = fmaxf(my, __shfl_xor_sync(0xFFFFFFFFu, my, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 2));
      my = fmaxf(my, __shfl_xor_sync(0xFFFFFFFFu, my, 2));

      const uint32_t sc2 = cvt_e4m3x2(group_scale_arg(mx, p.inv_g), group_scale_arg(my, p.inv_g));
      float Sx, Sy;
      e4m3x2_to_f32(sc2, Sx, Sy);
      const float Dx = Sx * p.g, Dy = Sy * p.g;
      const float rx = Dx > 0.f ? __frcp_rn(Dx) : 0.f;
      const float ry = Dy > 0.f ? __frcp_rn(Dy) : 0.f;

      uint32_t cw = cvt_e2m1x8(quotient(x0, Dx, rx), quotient(x1, Dx, rx), quotient(x2, Dx, rx),
                               quotient(x3, Dx, rx), quotient(y0, Dy, ry), quotient(y1, Dy, ry),
                               quotient(y2, Dy, ry), quotient(y3, Dy, ry));
      if (Dx == 0.f) cw &= 0xFFFF0000u;
      if (Dy == 0.f) cw &= 0x0000FFFFu;
      // byte 0: row g, elements 2q..2q+1 -> code byte 8 st + q; byte 1: elements 2q+8.. -> 8 st + 4 + q
      cst[g * kCodeStride + st * 8 + q] = static_cast<uint8_t>(cw);
      cst[g * kCodeStride + st * 8 + 4 + q] = static_cast<uint8_t>(cw >> 8);
      cst[(g + 8) * kCodeStride + st * 8 + q] = static_cast<uint8_t>(cw >> 16);
      cst[(g + 8) * kCodeStride + st * 8 + 4 + q] = static_cast<uint8_t>(cw >> 24);

      const int sh = 8 * (st & 3);
      sc_g |= (sc2 & 0xFFu) << sh;
      sc_h |= ((sc2 >> 8) & 0xFFu) << sh;
      if ((st & 3) == 3) {
        const int atom = (kc + st * 16) / 64;        // 64-K atom index
        if (q < 2) {
          const int r = warp * 16 + g + 8 * q;       // lane q=0 stores row g, q=1 row g+8
          const int m = m0 + r;
          const size_t off = (static_cast<size_t>(m / 128) * (p.K / 64) + atom) * 512 +
                             (m % 32) * 16 + ((m % 128) / 32) * 4;
          *reinterpret_cast<uint32_t*>(p.scales + off) = q == 0 ? sc_g : sc_h;
        }
        sc_g = 0; sc_h = 0;
      }

      // low-rank down projection on the smoothed values.  X_hat (at most 16 significant
      // bits) is split exactly into bf16 hi + lo, so two bf16 MMAs with fp32
      // accumulation give X_hat L1 without rounding the operand.
      uint32_t H0, H1, H2, H3, L0, L1, L2, L3;
      split_bf16x2(x0, x1, H0, L0);
      split_bf16x2(y0, y1, H1, L1);
      split_bf16x2(x2, x3, H2, L2);
      split_bf16x2(y2, y3, H3, L3);
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t b00, b01, b10, b11;
        const int mi = lane >> 3;
        const int n = half * 16 + ((mi >> 1) << 3) + (lane & 7);
        const int col = st * 16 + ((mi & 1) << 3);
        ldmatrix_x4(lbase + swz(n, col), b00, b01, b10, b11);
        mma_bf16_16816(acc[half * 2 + 0], H0, H1, H2, H3, b00, b01);
        mma_bf16_16816(acc[half * 2 + 1], H0, H1, H2, H3, b10, b11);
        mma_bf16_16816(acc[half * 2 + 0], L0, L1, L2, L3, b00, b01);
        mma_bf16_16816(acc[half * 2 + 1], L0, L1, L2, L3, b10, b11);
      }
    }

    // codes of this warp's 16 rows for the chunk -> global, 16 bytes per store
    __syncwarp();
    {
      const int rowbytes = ncols / 2;
      const int per_row = rowbytes / 16;
      for (int i = lane; i < 16 * per_row; i += 32) {
        const int r = i / per_row, seg = i % per_row;
        const int m = m0 + warp * 16 + r;
        if (m < p.M) {
          const uint4 v = *reinterpret_cast<const uint4*>(cst + r * kCodeStride + seg * 16);
          *reinterpret_cast<uint4*>(p.codes + static_cast<size_t>(m) * (p.K / 2) + kc / 2 + seg * 16) = v;
        }
      }
    }
    __syncthreads();          // buffer `buf` and the code staging are free again
  }

  // partial U of this slice -> shared memory
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int col = 8 * j + 2 * q;
    const int r0 = warp * 16 + g;
    s.upart[r0 * kRank + col] = acc[j][0];
    s.upart[r0 * kRank + col + 1] = acc[j][1];
    s.upart[(r0 + 8) * kRank + col] = acc[j][2];
    s.upart[(r0 + 8) * kRank + col + 1] = acc[j][3];
  }

  // sum the slices' partials across the cluster; CTA `rank` finishes rows [rank*rpc, (rank+1)*rpc)
  const int ks = p.kslices;
  if (ks > 1) cluster_sync_all(); else __syncthreads();
  const uint32_t rank = ks > 1 ? cluster_ctarank() : 0u;
  const int rpc = kRows / ks;
  for (int i = threadIdx.x; i < rpc * kRank; i += kThreads) {
    const int r = static_cast<int>(rank) * rpc + i / kRank;
    const int c = i % kRank;
    float sum = 0.f;
    if (ks > 1) {
      for (int src = 0; src < ks; ++src) sum += ld_dsmem_f32(&s.upart[r * kRank + c], static_cast<uint32_t>(src));
    } else {
      sum = s.upart[r * kRank + c];
    }
    const int m = m0 + r;
    if (m < p.M) p.U[static_cast<size_t>(m) * kRank + c] = sum;
  }
  if (ks > 1) cluster_sync_all();   // keep this CTA's shared memory alive until the others have read it
}

}  // namespace k1
}  // namespace svdq
