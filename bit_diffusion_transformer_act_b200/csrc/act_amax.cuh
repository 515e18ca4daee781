// Kernel 5: the dynamic per-tensor activation scale -- amax = max |X[m, k] smooth_inv[k]|
// over the whole tensor, for the variant of the W4A4 layer whose activation scale g_a is
// taken from the batch itself instead of from calibration.
//
// Method: "Nunchaku Lite" docs, "Supported quantization types" (svdq_w4a4 / nvfp4 /
// group 16, with a per-tensor scale); g_a is the power of two of the per-tensor scale
// rule, g = the smallest power of two with g * 6 * 448 >= amax (1 when amax = 0).
//
// Design (sm_100a, HBM-bound: one read of X).  A grid-stride loop of 16-byte loads of X (8
// bf16), four in flight per thread, each thread on one column unit whose 8 smoothing factors
// it loads once; the products are exact in fp32 (bf16 x bf16), so the
// maximum is exact and independent of the order; a warp-shuffle and a shared-memory max per
// block, then one atomicMax per block on the bits of the non-negative float (non-negative
// floats order like their bit patterns) into a partial word.  The last block to finish (a
// counter) moves the partial into the result word and resets the partial and the counter,
// so the three words need clearing only once, at allocation (no clearing pass per call, and
// a replayed CUDA graph finds them clean).  Kernels 1 and 2 read the result word after
// their grid-dependency wait and form g there (act_scale_from_amax).
#pragma once

#include "ptx.cuh"

namespace svdq {

// Smallest power of two g with g * 2688 >= amax (2688 = 6 * 448), 1 for amax = 0.  Every
// product g * 2688 is exact (2688 = 21 * 2^7; an overflow to +inf compares correctly), so
// the comparisons decide exactly.  The first guess from the rounded quotient is off by at
// most one power of two, so two bounded correction steps each way suffice, and the function
// ends for every input: NaN gives 1, +inf (an infinite activation) the largest power of two,
// and amax below 2688 * 2^-126 (not supported) a wrong but finite scale.
__device__ __forceinline__ float act_scale_from_amax(float amax) {
  if (!(amax > 0.f)) return 1.f;
  if (isinf(amax)) return 0x1p127f;
  int e;
  (void)frexpf(amax / 2688.f, &e);                 // amax / 2688 in [2^(e-1), 2^e), up to rounding
  float g = ldexpf(1.f, e);
#pragma unroll
  for (int i = 0; i < 2; ++i)
    if (g * 2688.f < amax) g *= 2.f;
#pragma unroll
  for (int i = 0; i < 2; ++i)
    if (g * (0.5f * 2688.f) >= amax) g *= 0.5f;
  return g;
}

namespace k5 {

constexpr int kThreads = 256;

// max |x_j s_j| over the 8 bf16 pairs of one 16-byte unit of X and its smoothing factors
__device__ __forceinline__ float absmax8(const uint4& x, const float (&s)[8], float m) {
  const uint32_t xw[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
  for (int j = 0; j < 4; ++j)
    m = fmax3(m, fabsf(bf16lo_to_f32(xw[j]) * s[2 * j]), fabsf(bf16hi_to_f32(xw[j]) * s[2 * j + 1]));
  return m;
}

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// The grid's thread count is a multiple of the row length in 16-byte units (the host picks
// the grid so), so a thread's column -- and its eight smoothing factors -- stay fixed over
// the grid-stride loop; four units are in flight per thread.
__global__ void __launch_bounds__(kThreads)
act_amax_kernel(const __nv_bfloat16* __restrict__ X, const __nv_bfloat16* __restrict__ smooth, int M, int K,
                unsigned int* words) {              // [0] amax (result), [1] partial max, [2] blocks done
  grid_dependency_wait();                          // X and the cleared word may come from the stream
  grid_launch_dependents();
  const size_t kv = static_cast<size_t>(K / 8);    // 16-byte units per row
  const size_t nvec = static_cast<size_t>(M) * kv;
  const size_t T = static_cast<size_t>(gridDim.x) * kThreads;
  const size_t base = static_cast<size_t>(blockIdx.x) * kThreads + threadIdx.x;
  const uint4* X4 = reinterpret_cast<const uint4*>(X);
  float m = 0.f;
  if (base < nvec) {
    const uint4 sv = __ldg(reinterpret_cast<const uint4*>(smooth) + base % kv);
    const float s[8] = {bf16lo_to_f32(sv.x), bf16hi_to_f32(sv.x), bf16lo_to_f32(sv.y), bf16hi_to_f32(sv.y),
                        bf16lo_to_f32(sv.z), bf16hi_to_f32(sv.z), bf16lo_to_f32(sv.w), bf16hi_to_f32(sv.w)};
    size_t i = base;
    for (; i + 3 * T < nvec; i += 4 * T) {
      const uint4 x0 = ld_stream(X4 + i), x1 = ld_stream(X4 + i + T);
      const uint4 x2 = ld_stream(X4 + i + 2 * T), x3 = ld_stream(X4 + i + 3 * T);
      m = absmax8(x3, s, absmax8(x2, s, absmax8(x1, s, absmax8(x0, s, m))));
    }
    for (; i < nvec; i += T) m = absmax8(ld_stream(X4 + i), s, m);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  __shared__ float wmax[kThreads / 32];
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float b = wmax[0];
#pragma unroll
    for (int w = 1; w < kThreads / 32; ++w) b = fmaxf(b, wmax[w]);
    atomicMax(words + 1, __float_as_uint(b));
    __threadfence();                               // the max is in before this block is counted
    if (atomicAdd(words + 2, 1u) == gridDim.x - 1) {
      __threadfence();
      words[0] = atomicExch(words + 1, 0u);        // every block's max is in: publish, reset
      atomicExch(words + 2, 0u);
    }
  }
}

}  // namespace k5
}  // namespace svdq
