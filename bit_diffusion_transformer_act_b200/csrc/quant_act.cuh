// Kernel 1: activation smoothing, NVFP4 quantization and the rank-32
// down-projection, in one pass over X.
//
// Method ("Nunchaku Lite" docs, "Supported quantization types": svdq_w4a4 /
// nvfp4 / group 16; the Nunchaku Lite article: outliers go to a 16-bit
// low-rank branch): X_hat = X * smooth_inv; per 16 K elements one E4M3 scale
// S = RNE(amax / (6 g_a)) and E2M1 codes RNE(clamp(X_hat / (S g_a))); and
// U = X_hat L1 (rank 32) from the same smoothed activations.
//
// Design (sm_100a).  A CTA (8 warps) owns 128 rows and one K slice; the K
// slices of a row block form a thread-block cluster (1..8 CTAs) so the grid
// fills the 148 SMs, and the partial U of the slices is summed over
// distributed shared memory -- no global scratch, no atomics.  X and the L1
// operand arrive in 128-column chunks, double-buffered in shared memory with
// cp.async (rows past M zero-filled) and XOR-swizzled against bank conflicts.
//   * Quantization: each thread owns one row and 64 consecutive columns (four
//     16-element groups, i.e. one 32-bit word of the scale layout and 32
//     contiguous code bytes, stored directly).
//   * Low-rank: X_hat L1 = X (diag(smooth_inv) L1); the packed weights hold
//     diag(smooth_inv) L1 split exactly into bf16 hi + lo, so ldmatrix feeds
//     the raw bf16 X tile to mma.sync twice (hi, lo) with fp32 accumulation:
//     every product is exact.  The result U / g_a is written split into bf16
//     hi + lo, the operand layout of the GEMM's low-rank MMA.
//
// Rounding.  amax/6 is formed by a Markstein-corrected multiplication by the
// rounded reciprocal of 6 (P. Markstein's correction: with y = RN(1/b) and
// q0 = RN(a y), q0 + RN(a - b q0) y rounds to RN(a/b)), then scaled by 1/g_a
// (a power of two) and converted with cvt.rn.satfinite.e4m3x2.  A code
// quotient x_hat / (S g_a) is q0 = x_hat * r with r = rcp.approx(S g_a)
// followed by the same correction step; because x_hat has at most 16
// significant bits and the E2M1 midpoints times S g_a at most 7, a quotient is
// either exactly a midpoint -- and then the corrected value is that midpoint
// exactly -- or at least 2^-16 (relative) away from one, far beyond the
// few-ulp error of q.  cvt.rn.satfinite.e2m1x2 then rounds to nearest even.
// The sign of q is copied from x_hat so that negative zero keeps its sign.
#pragma once

#include "ptx.cuh"

namespace svdq {
namespace k1 {

constexpr int kRows = 128;                // rows per CTA
constexpr int kWarps = 8;                 // 16 rows each for the low-rank MMA
constexpr int kThreads = kWarps * 32;
constexpr int kChunk = 128;               // K columns per pipeline chunk
constexpr int kRank = 32;
constexpr int kMaxSlice = 2048;           // longest K slice (columns) held as fp32 smoothing factors

struct __align__(128) Smem {
  __nv_bfloat16 x[2][kRows * kChunk];     // rows of 256 B, 16-B pieces XOR-swizzled by (row & 7)
  __nv_bfloat16 lh[2][kRank * kChunk];    // (diag(s) L1)^T high part, same swizzle
  __nv_bfloat16 ll[2][kRank * kChunk];    // low part
  float smooth[kMaxSlice];                // this CTA's slice of smooth_inv, as floats
};
// The partial U of the CTA (128 x 32 fp32) reuses the X buffers once the K loop is done.
static_assert(sizeof(__nv_bfloat16) * 2 * kRows * kChunk >= sizeof(float) * kRows * kRank, "upart alias");

// Byte offset of element (row, col) in a swizzled [rows][128] bf16 chunk.
__device__ __forceinline__ uint32_t swz(int row, int col) {
  return static_cast<uint32_t>(row * 256 + ((((col >> 3) ^ (row & 7)) << 4)) + ((col & 7) << 1));
}

struct Params {
  const __nv_bfloat16* X;          // [M, K]
  const __nv_bfloat16* smooth;     // [K]
  const __nv_bfloat16* l1s;        // [2][32][K]: (diag(smooth) L1)^T hi, then lo
  uint8_t* codes;                  // [M, K/2]
  uint8_t* scales;                 // swizzled, rows padded to 128
  __nv_bfloat16* ucat;             // [M, 64]: U / g_a as bf16 hi (0..31) and lo (32..63)
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
  const uint32_t hbase = smem_addr(s.lh[buf]), lbase = smem_addr(s.ll[buf]);
  const __nv_bfloat16* lo_src = p.l1s + static_cast<size_t>(kRank) * p.K;
  for (int i = tid; i < kRank * pieces; i += kThreads) {
    const int r = i / pieces, c = (i % pieces) * 8;
    cp_async_16(hbase + swz(r, c), p.l1s + static_cast<size_t>(r) * p.K + kc + c, 16u);
    cp_async_16(lbase + swz(r, c), lo_src + static_cast<size_t>(r) * p.K + kc + c, 16u);
  }
  cp_async_commit();
}

__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// Quotient x / D for the E2M1 decision (see the rounding note above); r ~ 1/D.
__device__ __forceinline__ float quotient(float x, float D, float r) {
  const float q0 = x * r;
  const float e = fmaf(-q0, D, x);
  const float q = fmaf(e, r, q0);
  return __uint_as_float((__float_as_uint(q) & 0x7FFFFFFFu) | (__float_as_uint(x) & 0x80000000u));
}

// RN(a / 6) for a >= 0 (Markstein correction of a * RN(1/6)).
__device__ __forceinline__ float div6(float a) {
  const float y = 0.16666667163372039794921875f;      // RN(1/6) in binary32
  const float q0 = a * y;
  const float e = fmaf(-q0, 6.0f, a);
  return fmaf(e, y, q0);
}

// Quantizes 16 smoothed values (one group): returns the E4M3 scale code, writes 8 code bytes.
__device__ __forceinline__ uint32_t quantize_group(const float (&v)[16], const Params& p, uint2& out) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const uint32_t sc = cvt_e4m3x2(div6(amax) * p.inv_g, 0.f) & 0xFFu;
  float S, unused;
  e4m3x2_to_f32(sc, S, unused);
  const float D = S * p.g;
  if (D == 0.f) {
    out = make_uint2(0u, 0u);
    return 0u;
  }
  const float r = rcp_approx(D);
  out.x = cvt_e2m1x8(quotient(v[0], D, r), quotient(v[1], D, r), quotient(v[2], D, r), quotient(v[3], D, r),
                     quotient(v[4], D, r), quotient(v[5], D, r), quotient(v[6], D, r), quotient(v[7], D, r));
  out.y = cvt_e2m1x8(quotient(v[8], D, r), quotient(v[9], D, r), quotient(v[10], D, r), quotient(v[11], D, r),
                     quotient(v[12], D, r), quotient(v[13], D, r), quotient(v[14], D, r), quotient(v[15], D, r));
  return sc;
}

__global__ void __launch_bounds__(kThreads, 2)
quant_act_lowrank_kernel(const Params p) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  Smem& s = *reinterpret_cast<Smem*>(smem_raw);

  const int tid = threadIdx.x;
  const int warp = tid / 32;
  const int lane = tid % 32;
  const int m0 = blockIdx.x * kRows;
  const int slice = blockIdx.y;
  const int klen = p.K / p.kslices;
  const int kbeg = slice * klen;
  const int nchunks = (klen + kChunk - 1) / kChunk;

  grid_dependency_wait();                          // X and the outputs may belong to the previous kernel
  grid_launch_dependents();
  load_chunk(s, 0, p, m0, kbeg, min(kChunk, klen));
  for (int i = tid; i < klen; i += kThreads) s.smooth[i] = __bfloat162float(p.smooth[kbeg + i]);

  float acc[4][4];
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int t = 0; t < 4; ++t) acc[j][t] = 0.f;

  // quantization role of this thread: row qr, columns [64 qh, 64 qh + 64) of each chunk
  const int qr = tid >> 1, qh = tid & 1;
  const int qm = m0 + qr;

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

    const uint8_t* xs = reinterpret_cast<const uint8_t*>(s.x[buf]);

    // ---------------------------------------------------------------- quantization
    if (qh * 64 < ncols) {
      const float* sm = s.smooth + (kc - kbeg) + qh * 64;
      uint32_t scw = 0;
      uint2 cb[4];
#pragma unroll
      for (int gq = 0; gq < 4; ++gq) {
        float v[16];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int col = qh * 64 + gq * 16 + h * 8;
          const uint4 xv = *reinterpret_cast<const uint4*>(xs + swz(qr, col));
          const float4 s0 = *reinterpret_cast<const float4*>(sm + gq * 16 + h * 8);
          const float4 s1 = *reinterpret_cast<const float4*>(sm + gq * 16 + h * 8 + 4);
          v[h * 8 + 0] = bf16lo_to_f32(xv.x) * s0.x;
          v[h * 8 + 1] = bf16hi_to_f32(xv.x) * s0.y;
          v[h * 8 + 2] = bf16lo_to_f32(xv.y) * s0.z;
          v[h * 8 + 3] = bf16hi_to_f32(xv.y) * s0.w;
          v[h * 8 + 4] = bf16lo_to_f32(xv.z) * s1.x;
          v[h * 8 + 5] = bf16hi_to_f32(xv.z) * s1.y;
          v[h * 8 + 6] = bf16lo_to_f32(xv.w) * s1.z;
          v[h * 8 + 7] = bf16hi_to_f32(xv.w) * s1.w;
        }
        scw |= quantize_group(v, p, cb[gq]) << (8 * gq);
      }
      const int atom = (kc + qh * 64) / 64;
      const size_t soff = (static_cast<size_t>(qm / 128) * (p.K / 64) + atom) * 512 + (qm % 32) * 16 +
                          ((qm % 128) / 32) * 4;
      *reinterpret_cast<uint32_t*>(p.scales + soff) = scw;      // rows past M get zero scales
      if (qm < p.M) {
        uint4* dst = reinterpret_cast<uint4*>(p.codes + static_cast<size_t>(qm) * (p.K / 2) + (kc + qh * 64) / 2);
        dst[0] = make_uint4(cb[0].x, cb[0].y, cb[1].x, cb[1].y);
        dst[1] = make_uint4(cb[2].x, cb[2].y, cb[3].x, cb[3].y);
      }
    }

    // ---------------------------------------------------------------- low-rank down projection
    {
      const uint32_t xbase = smem_addr(s.x[buf]);
      const uint32_t hbase = smem_addr(s.lh[buf]), lbase = smem_addr(s.ll[buf]);
      const int mi = lane >> 3;
      const int steps = ncols / 16;
      for (int st = 0; st < steps; ++st) {
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4(xbase + swz(warp * 16 + (lane & 7) + ((mi & 1) << 3), st * 16 + ((mi >> 1) << 3)),
                    a0, a1, a2, a3);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const int n = half * 16 + ((mi >> 1) << 3) + (lane & 7);
          const int col = st * 16 + ((mi & 1) << 3);
          uint32_t h00, h01, h10, h11, l00, l01, l10, l11;
          ldmatrix_x4(hbase + swz(n, col), h00, h01, h10, h11);
          ldmatrix_x4(lbase + swz(n, col), l00, l01, l10, l11);
          mma_bf16_16816(acc[half * 2 + 0], a0, a1, a2, a3, h00, h01);
          mma_bf16_16816(acc[half * 2 + 1], a0, a1, a2, a3, h10, h11);
          mma_bf16_16816(acc[half * 2 + 0], a0, a1, a2, a3, l00, l01);
          mma_bf16_16816(acc[half * 2 + 1], a0, a1, a2, a3, l10, l11);
        }
      }
    }
    __syncthreads();          // buffer `buf` is free again
  }

  // partial U of this slice -> shared memory (reusing the X buffers)
  float* upart = reinterpret_cast<float*>(s.x[0]);
  {
    const int g = lane >> 2, q = lane & 3;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int col = 8 * j + 2 * q;
      const int r0 = warp * 16 + g;
      upart[r0 * kRank + col] = acc[j][0];
      upart[r0 * kRank + col + 1] = acc[j][1];
      upart[(r0 + 8) * kRank + col] = acc[j][2];
      upart[(r0 + 8) * kRank + col + 1] = acc[j][3];
    }
  }

  // sum the slices' partials across the cluster; CTA `rank` finishes rows [rank*rpc, (rank+1)*rpc)
  const int ks = p.kslices;
  if (ks > 1) cluster_sync_all(); else __syncthreads();
  const uint32_t rank = ks > 1 ? cluster_ctarank() : 0u;
  const int rpc = kRows / ks;
  for (int i = tid; i < rpc * kRank; i += kThreads) {
    const int r = static_cast<int>(rank) * rpc + i / kRank;
    const int c = i % kRank;
    float sum = 0.f;
    if (ks > 1) {
      for (int src = 0; src < ks; ++src) sum += ld_dsmem_f32(&upart[r * kRank + c], static_cast<uint32_t>(src));
    } else {
      sum = upart[r * kRank + c];
    }
    const int m = m0 + r;
    if (m < p.M) {
      const float u = sum * p.inv_g;                   // exact: a power of two
      const __nv_bfloat16 hi = __float2bfloat16_rn(u);
      const __nv_bfloat16 lo = __float2bfloat16_rn(u - __bfloat162float(hi));
      p.ucat[static_cast<size_t>(m) * (2 * kRank) + c] = hi;
      p.ucat[static_cast<size_t>(m) * (2 * kRank) + kRank + c] = lo;
    }
  }
  if (ks > 1) cluster_sync_all();   // keep this CTA's shared memory alive until the others have read it
}

}  // namespace k1
}  // namespace svdq
