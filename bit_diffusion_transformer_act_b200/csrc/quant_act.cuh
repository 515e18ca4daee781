// Kernel 1: activation smoothing, NVFP4 quantization and the rank-32
// down-projection, in one pass over X.
//
// Method ("Nunchaku Lite" docs, "Supported quantization types": svdq_w4a4 /
// nvfp4 / group 16; the Nunchaku Lite article: outliers go to a 16-bit
// low-rank branch): X_hat = X * smooth_inv; per 16 K elements one E4M3 scale
// S = RNE(amax / (6 g_a)) and E2M1 codes RNE(clamp(X_hat / (S g_a))); and
// U = X_hat L1 (rank 32) from the same smoothed activations.
//
// Design (sm_100a).  A CTA owns 128 rows and one K slice; the K slices of a row
// block form a thread-block cluster (1..16 CTAs; 16, a non-portable size, only where the
// grid then still fits one wave, i.e. for a few row blocks) so that the grid fills the SMs
// (two CTAs per SM), and the slices' partial U are summed over distributed
// shared memory -- no global scratch, no atomics.  Warp roles:
//   warp 0     TMA producer: per 64-column chunk the X tile (128 rows, 128-byte
//              swizzle; rows past M read as zeros) and the matching 64 x 64 tile
//              of the packed low-rank operand, into a ring of stages.
//   warp 1     tensor memory and the low-rank MMA: X_hat L1 = X (diag(smooth_inv)
//              L1), and the packed weights hold diag(smooth_inv) L1 split exactly
//              into bf16 hi + lo, so one tcgen05 MMA (M = 128, N = 64 = 32 hi + 32
//              lo columns, K = 16) per 16 columns multiplies the raw X tile with
//              every product exact, accumulating in fp32 in tensor memory.
//   warps 2-9  quantizers: a thread owns 32 columns (two groups) of one row of the
//              chunk, reads X from the swizzled tile, smooths, finds the group
//              maxima, the E4M3 scales and E2M1 codes, and stores 16 code bytes and
//              2 scale bytes straight to global memory.
// A stage is free again when the eight quantizer warps have read it and the MMAs
// that read it have completed (tcgen05.commit).  At the end, warps 0, 1, 10 and 11
// (one per tensor-memory lane quarter; none of them stores to global memory) read
// U = hi + lo into a ring slot that is already free as soon as the last MMA is done, the
// cluster sums the slices, and U / g_a is written split into bf16 hi + lo, the operand
// layout of the GEMM's low-rank MMA.  Only those four warps gate the first cluster
// barrier (with release semantics): the quantizers arrive at it before their loop, so the
// sum over the slices overlaps their last chunks; the barrier that keeps shared memory
// alive until the peers have read it is relaxed.  Every mbarrier wait is bounded; a wait
// that runs out records SVDQ_ERR_TIMEOUT in the device status word and the CTA winds
// down.
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
// The quantizers hold -x_hat (the smoothing factors are stored negated) and
// form the residual as e' = q0 D - x_hat and the quotient as q0 - e' r; the
// values are those of the textbook form, and a zero x_hat keeps its sign in q
// (for x_hat = -0: q0 = -0, e' = +0, q = -0 + -0 = -0).  Pairs of values go
// through the packed fp32x2 multiply and fma of sm_100, each half rounded to
// nearest as its scalar counterpart.
#pragma once

#include "act_amax.cuh"
#include "nvfp4_quant.cuh"
#include "ptx.cuh"

namespace svdq {
namespace k1 {

constexpr int kRows = 128;                // rows per CTA (one 128-row scale block)
constexpr int kChunk = 64;                // K columns per pipeline stage
constexpr int kRank = 32;
constexpr int kQuantWarps = 8;
constexpr int kReadWarp0 = 2 + kQuantWarps;   // warps 10, 11: tensor-memory lane quarters 2, 3 of the U read-out
constexpr int kThreads = (4 + kQuantWarps) * 32;
constexpr int kStages = 4;
constexpr int kMaxSlice = 2048;           // longest K slice (columns) held as fp32 smoothing factors
constexpr int kXBytes = kRows * kChunk * 2;          // 16 KB
constexpr int kLBytes = 2 * kRank * kChunk * 2;      // 8 KB: 64 operand rows (hi, lo) x 64 columns
constexpr int kStageBytes = kXBytes + kLBytes;
constexpr int kTmemCols = 64;

struct Params {
  uint8_t* codes;                  // [M, K/2]
  uint8_t* scales;                 // swizzled, rows padded to 128
  __nv_bfloat16* ucat;             // [M, 64]: U / g_a as bf16 hi (0..31) and lo (32..63)
  const __nv_bfloat16* smooth;     // [K]
  int M, K;
  int kslices;                     // cluster size along K
  float g;                         // per-tensor scale (power of two)
  float inv_g;
  const unsigned int* amax;        // or, if not null, g from this amax word (kernel 5) at run time
};

// Shared memory (1024-byte aligned base): stages | smooth slice (fp32) | barriers.
constexpr int kOffSmooth = kStages * kStageBytes;
constexpr int kOffBar = kOffSmooth + kMaxSlice * 4;
constexpr int kNumBars = 2 * kStages + 2;           // full, empty, acc_full, drain
constexpr int kOffMisc = kOffBar + 8 * kNumBars;
constexpr int kSmemBytes = kOffMisc + 16 + 1024;
static_assert(kSmemBytes <= 113 * 1024, "two CTAs per SM");
static_assert(kRows * kRank * 4 <= kStages * kStageBytes, "partial U reuses the stages");
static_assert(kStageBytes % 1024 == 0 && kXBytes % 1024 == 0, "1 KB alignment of swizzled tiles");

// kind::f16 instruction descriptor: D f32, A and B bf16, K-major, N = 64, M = 128.
__device__ __forceinline__ uint32_t idesc_lowrank() {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(64 >> 3) << 17) |
         (static_cast<uint32_t>(128 >> 4) << 24);
}

// The int4 / group-64 row's quantizer of one 64-column group held by two neighbouring lanes (32
// columns each, as 16 pairs of -x_hat): both lanes form the group's amax (one exchange), the
// bf16 scale s = RNE_bf16(amax / 7) rounded once from the exact quotient, and this lane's 32
// codes RNE(x_hat / s) as E4M3 bytes (the integers -7..7 are exact in E4M3; with s rounded to
// nearest, |x_hat / s| <= 7 (1 + 2^-8) < 7.5, so no code needs clamping).  Returns s's bits.
// amax / 7 is the correctly rounded fp32 quotient; when that lands exactly on a bf16 midpoint
// the exact quotient decides the side (7 times the midpoint, 12 significant bits, is exact).
// x_hat / s: the corrected quotient as in the nvfp4 quantizer (x_hat has at most 16 significant
// bits and s 8, so an exact half-integer quotient is computed exactly and any other is at least
// 2^-16 away from one).  Scales below 2^-126 (amax < 7 * 2^-126) are not supported.
__device__ __forceinline__ uint16_t quantize_int4_group(const uint64_t (&nx)[16], uint4 (&out)[2]) {
  float a[32];
#pragma unroll
  for (int i = 0; i < 16; ++i) f32x2_unpack(nx[i], a[2 * i], a[2 * i + 1]);
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 32; i += 2) amax = fmax3(amax, fabsf(a[i]), fabsf(a[i + 1]));
  amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
  const float q = __fdiv_rn(amax, 7.0f);
  const uint32_t qb = __float_as_uint(q);
  uint32_t sb;
  if ((qb & 0xFFFFu) == 0x8000u) {
    const float t = 7.0f * q;                      // exact
    sb = amax > t ? (qb >> 16) + 1u : (amax < t ? (qb >> 16) : (pack_bf16x2(q, 0.f) & 0xFFFFu));
  } else {
    sb = pack_bf16x2(q, 0.f) & 0xFFFFu;            // round to nearest even
  }
  const float s = __uint_as_float(sb << 16);
  if (s == 0.f) {
    out[0] = out[1] = make_uint4(0u, 0u, 0u, 0u);
    return 0;
  }
  const float rn = -rcp_approx(s);                 // -1/s: the pairs hold -x_hat
  const uint64_t rn2 = f32x2_pack(rn, rn), s2 = f32x2_pack(s, s);
  uint32_t w[8];
#pragma unroll
  for (int i = 0; i < 16; i += 2) {
    float v[4];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const uint64_t q0 = f32x2_mul(nx[i + j], rn2);          // x_hat / s, first guess
      const uint64_t e = f32x2_fma(q0, s2, nx[i + j]);        // q0 s - x_hat, exact
      f32x2_unpack(f32x2_fma(e, rn2, q0), v[2 * j], v[2 * j + 1]);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) v[j] = rintf(v[j]);          // to nearest integer, ties to even
    w[i / 2] = cvt_e4m3x2(v[0], v[1]) | (cvt_e4m3x2(v[2], v[3]) << 16);
  }
  out[0] = make_uint4(w[0], w[1], w[2], w[3]);
  out[1] = make_uint4(w[4], w[5], w[6], w[7]);
  return static_cast<uint16_t>(sb);
}

template <bool kInt4 = false>
__global__ void __launch_bounds__(kThreads, 2)
quant_act_lowrank_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmL,
                         const Params p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t bars = base + kOffBar;
  auto full = [&](int s) { return bars + 8u * s; };
  auto empty = [&](int s) { return bars + 8u * (kStages + s); };
  const uint32_t acc_full = bars + 8u * (2 * kStages);
  const uint32_t drain = bars + 8u * (2 * kStages + 1);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + kOffMisc + 4);
  float* smooth = reinterpret_cast<float*>(gbase + kOffSmooth);   // -smooth_inv of this K slice

  const int tid = threadIdx.x;
  const int warp = tid / 32;
  const int lane = tid % 32;
  const int m0 = blockIdx.x * kRows;
  const int klen = p.K / p.kslices;
  const int kbeg = blockIdx.y * klen;
  const int nck = klen / kChunk;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < kStages; ++s) { mbar_init(full(s), 1); mbar_init(empty(s), kQuantWarps + 1); }
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmX);
    prefetch_tmap(&tmL);
  }
  if (warp == 1) tmem_alloc<kTmemCols>(smem_addr(tmem_slot));
  grid_dependency_wait();                          // X and the outputs may belong to the previous kernel
  float g = p.g, inv_g = p.inv_g;                  // the per-tensor scale: given, or from the batch's amax
  if (p.amax) {
    g = act_scale_from_amax(__uint_as_float(*p.amax));
    inv_g = 1.0f / g;                              // exact: a power of two
  }
  grid_launch_dependents();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (warp >= 2 && warp < kReadWarp0) {
    // the quantizers fetch the smoothing factors while the first tiles are in flight
    for (int i = tid - 64; i < klen; i += kQuantWarps * 32) smooth[i] = -__bfloat162float(p.smooth[kbeg + i]);
    asm volatile("bar.sync 1, %0;" ::"n"(kQuantWarps * 32) : "memory");   // quantizer warps only
  }

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer (one elected lane issues)
    for (int c = 0; c < nck; ++c) {
      const int s = c % kStages;
      const uint32_t ph = (c / kStages) & 1u;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(empty(s), ph ^ 1u, abort_flag, 11))) break;
      if (elect_one()) {
        const uint32_t sb = base + s * kStageBytes;
        mbar_arrive_expect_tx(full(s), kStageBytes);
        tma_load_2d(sb, &tmX, kbeg + c * kChunk, m0, full(s));
        tma_load_2d(sb + kXBytes, &tmL, kbeg + c * kChunk, 0, full(s));
      }
      __syncwarp();
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- low-rank MMA (one elected lane issues)
    constexpr uint32_t kHiSw128 = smem_desc_hi(1024, 2);      // K-major, 128-byte swizzle
    constexpr uint32_t kLbo = 1u << 16;
    const uint32_t idesc = idesc_lowrank();
    for (int c = 0; c < nck; ++c) {
      const int s = c % kStages;
      const uint32_t ph = (c / kStages) & 1u;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(full(s), ph, abort_flag, 12))) break;
      tc_fence_after();
      if (elect_one()) {
        const uint32_t sb = base + s * kStageBytes;
        const uint32_t a_lo = (sb >> 4) | kLbo;
        const uint32_t b_lo = ((sb + kXBytes) >> 4) | kLbo;
#pragma unroll
        for (int kk = 0; kk < kChunk / 16; ++kk)
          umma_bf16(tmem, make_desc(a_lo + kk * 2, kHiSw128), make_desc(b_lo + kk * 2, kHiSw128), idesc,
                    (c | kk) != 0 ? 1u : 0u);
        tc_commit(empty(s));
        if (c == nck - 1) tc_commit(acc_full);
      }
      __syncwarp();
    }
  } else if (warp < kReadWarp0) {
    // ---------------------------------------------------------------- quantizers
    // The first cluster barrier gates the sum of U over the slices; the quantizers publish
    // nothing it reads, so they arrive now and the sum overlaps their last chunks.
    cluster_arrive_relaxed();
    const int qt = tid - 64;                      // 0..255
    const int r = qt >> 1;                        // row of the chunk
    const int h = qt & 1;                         // columns [32 h, 32 h + 32) of the chunk
    const int m = m0 + r;
    const uint32_t sw = static_cast<uint32_t>(r & 7);
    uint8_t* code_row = p.codes + static_cast<size_t>(m) * (p.K / 2) + kbeg / 2 + h * 16;
    // scale bytes 2h, 2h + 1 of this row's word in the chunk's 512-byte atom
    uint8_t* scale_base = p.scales + static_cast<size_t>(m0 / 128) * (p.K / 64) * 512 + (r % 32) * 16 +
                          (r / 32) * 4 + 2 * h;
    const int mpad = (p.M + kRows - 1) / kRows * kRows;
    for (int c = 0; kInt4 && c < nck; ++c) {
      // int4 / group 64: the chunk is one group, shared by this lane and its neighbour
      const int s = c % kStages;
      const uint32_t ph = (c / kStages) & 1u;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(full(s), ph, abort_flag, 13))) break;
      const uint32_t row = base + s * kStageBytes + r * 128;
      const float* sm = smooth + c * kChunk + h * 32;
      uint64_t nx[16];
#pragma unroll
      for (int uu = 0; uu < 4; ++uu) {
        const uint32_t u = static_cast<uint32_t>(h * 4 + uu);
        uint32_t xw[4];
        asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(xw[0]), "=r"(xw[1]), "=r"(xw[2]), "=r"(xw[3]) : "r"(row + ((u ^ sw) << 4)));
        const ulonglong2 s01 = *reinterpret_cast<const ulonglong2*>(sm + uu * 8);
        const ulonglong2 s23 = *reinterpret_cast<const ulonglong2*>(sm + uu * 8 + 4);
        const uint64_t sp[4] = {s01.x, s01.y, s23.x, s23.y};
#pragma unroll
        for (int w = 0; w < 4; ++w)
          nx[uu * 4 + w] = f32x2_mul(f32x2_pack(bf16lo_to_f32(xw[w]), bf16hi_to_f32(xw[w])), sp[w]);
      }
      uint4 cw[2];
      const uint16_t sb = quantize_int4_group(nx, cw);
      __syncwarp();
      if (lane == 0) mbar_arrive_relaxed(empty(s));
      if (m < p.M) {
        uint4* dst = reinterpret_cast<uint4*>(p.codes + static_cast<size_t>(m) * p.K + kbeg + c * kChunk + h * 32);
        dst[0] = cw[0];
        dst[1] = cw[1];
      }
      if (h == 0)                                  // group-major [K/64][rows padded to 128]; rows past M
        reinterpret_cast<uint16_t*>(p.scales)[static_cast<size_t>((kbeg / 64) + c) * mpad + m] = sb;   // read zeros
    }
    for (int c = 0; !kInt4 && c < nck; ++c) {
      const int s = c % kStages;
      const uint32_t ph = (c / kStages) & 1u;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(full(s), ph, abort_flag, 13))) break;
      const uint32_t row = base + s * kStageBytes + r * 128;
      const float* sm = smooth + c * kChunk + h * 32;
      uint32_t sc2 = 0;
      uint2 cb[2];
#pragma unroll
      for (int gq = 0; gq < 2; ++gq) {
        uint64_t nx[8];                            // -x_hat, in pairs
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const uint32_t u = static_cast<uint32_t>(h * 4 + gq * 2 + hh);     // 16-byte unit of the row
          uint32_t xw[4];
          asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(xw[0]), "=r"(xw[1]), "=r"(xw[2]), "=r"(xw[3]) : "r"(row + ((u ^ sw) << 4)));
          const ulonglong2 s01 = *reinterpret_cast<const ulonglong2*>(sm + gq * 16 + hh * 8);
          const ulonglong2 s23 = *reinterpret_cast<const ulonglong2*>(sm + gq * 16 + hh * 8 + 4);
          const uint64_t sp[4] = {s01.x, s01.y, s23.x, s23.y};
#pragma unroll
          for (int w = 0; w < 4; ++w)
            nx[hh * 4 + w] = f32x2_mul(f32x2_pack(bf16lo_to_f32(xw[w]), bf16hi_to_f32(xw[w])), sp[w]);
        }
        sc2 |= quantize_group(nx, g, inv_g, cb[gq]) << (8 * gq);
      }
      // the tile has been read: release it to the producer (with the MMA's commit)
      __syncwarp();
      if (lane == 0) mbar_arrive_relaxed(empty(s));
      *reinterpret_cast<uint16_t*>(scale_base + static_cast<size_t>((kbeg / 64) + c) * 512) =
          static_cast<uint16_t>(sc2);            // rows past M get zero scales
      if (m < p.M)
        *reinterpret_cast<uint4*>(code_row + c * 32) = make_uint4(cb[0].x, cb[0].y, cb[1].x, cb[1].y);
    }
  }

  // ---------------------------------------------------------------- U = hi + lo, summed over the cluster
  // Read out by warps 0, 1, 10 and 11 (lane quarters 0-3) once the last MMA is done, while the
  // quantizers may still be on their last chunks.  The partial goes to the ring slot after the
  // last chunk's: free once its last chunk (nck - kStages) has been consumed, never used when
  // nck < kStages.  Only these warps arrive at the first cluster barrier now (with release:
  // their partials; none of them stores to global memory, so the arrival waits for nothing
  // else); the quantizers arrived before their loop and wait on it after.
  const int ks = p.kslices;
  const int su = nck % kStages;
  float* upart = reinterpret_cast<float*>(gbase + su * kStageBytes);   // [128][32] fp32, 16-byte pieces rotated by the row
  const bool reader = warp < 2 || warp >= kReadWarp0;
  if (reader) {
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    float u[32];
    bool ok = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(acc_full, 0, abort_flag, 14));
    if (ok && nck >= kStages)
      ok = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(empty(su), ((nck - kStages) / kStages) & 1u, abort_flag, 17));
    if (ok) {
      tc_fence_after();
      uint32_t hi[32], lo[32];
      tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(quarter * 32) << 16), hi);
      tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(quarter * 32) << 16) + 32u, lo);
      tmem_wait_ld_regs(hi);
      tmem_wait_ld_regs(lo);
#pragma unroll
      for (int j = 0; j < 32; ++j) u[j] = __uint_as_float(hi[j]) + __uint_as_float(lo[j]);
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) u[j] = 0.f;
    }
#pragma unroll
    for (int j = 0; j < 8; ++j)
      *reinterpret_cast<float4*>(upart + row * 32 + ((j + row) & 7) * 4) =
          make_float4(u[j * 4], u[j * 4 + 1], u[j * 4 + 2], u[j * 4 + 3]);
    tc_fence_before();
    cluster_arrive_release();                      // this CTA's partial is in shared memory
    cluster_wait_acquire();                        // ... and every other slice's
    const uint32_t crank = cluster_ctarank();
    const int rpc = kRows / ks;                    // rows finished by this CTA
    const int rt = (warp < 2 ? warp : warp - kReadWarp0 + 2) * 32 + lane;   // 0..127
    for (int i = rt; i < rpc * 8; i += 128) {      // one 4-column piece of one row per thread
      const int rr = static_cast<int>(crank) * rpc + i / 8;
      const int piece = i % 8;
      const float* src_addr = upart + rr * 32 + ((piece + rr) & 7) * 4;
      float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 1
      for (int s0 = 0; s0 < ks; s0 += 8) {         // up to 16 slices, eight loads in flight at a time
        float4 v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (s0 + j < ks) v[j] = ld_dsmem_f32x4(src_addr, static_cast<uint32_t>(s0 + j));
#pragma unroll
        for (int j = 0; j < 8; ++j)                // in slice order: deterministic
          if (s0 + j < ks) {
            if (s0 + j == 0) sum = v[0];
            else { sum.x += v[j].x; sum.y += v[j].y; sum.z += v[j].z; sum.w += v[j].w; }
          }
      }
      const int mm = m0 + rr;
      if (mm < p.M) {
        const float uu[4] = {sum.x * inv_g, sum.y * inv_g, sum.z * inv_g, sum.w * inv_g};  // exact
        uint32_t hw[2], lw[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const float h0 = __bfloat162float(__float2bfloat16_rn(uu[2 * j]));
          const float h1 = __bfloat162float(__float2bfloat16_rn(uu[2 * j + 1]));
          hw[j] = pack_bf16x2(h0, h1);
          lw[j] = pack_bf16x2(uu[2 * j] - h0, uu[2 * j + 1] - h1);
        }
        __nv_bfloat16* dst = p.ucat + static_cast<size_t>(mm) * (2 * kRank) + piece * 4;
        *reinterpret_cast<uint2*>(dst) = make_uint2(hw[0], hw[1]);
        *reinterpret_cast<uint2*>(dst + kRank) = make_uint2(lw[0], lw[1]);
      }
    }
  } else {
    cluster_wait_acquire();                        // the quantizers' arrival came before their loop
  }
  if (*abort_flag) {
    // a wait ran out: let the MMAs and copies already issued finish before the memory goes away
    if (warp == 1) {
      if (elect_one()) tc_commit(drain);
      __syncwarp();
      mbar_wait_bounded(drain, 0, nullptr, 15);
    }
    if (warp == 0 && lane == 0) {
      const uint64_t t0 = global_timer_ns();
      while (global_timer_ns() - t0 < 2000000ull) { }
    }
  }
  // the other CTAs are done reading this CTA's partials (their loads have returned: nothing
  // to order, so a relaxed arrival)
  __syncwarp();
  cluster_arrive_relaxed();
  cluster_wait_acquire();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc<kTmemCols>(tmem);
  }
}

}  // namespace k1
}  // namespace svdq
