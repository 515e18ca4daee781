// Kernel 5: the dynamic per-tensor activation scale -- amax = max |X[m, k] smooth_inv[k]|
// over the whole tensor, for the variant of the W4A4 layer whose activation scale g_a is
// taken from the batch itself instead of from calibration.
//
// Method: "Nunchaku Lite" docs, "Supported quantization types" (svdq_w4a4 / nvfp4 /
// group 16, with a per-tensor scale); g_a is the power of two of the per-tensor scale
// rule, g = the smallest power of two with g * 6 * 448 >= amax (1 when amax = 0).
//
// Design (sm_100a, HBM-bound: one read of X).  A grid-stride loop of 16-byte loads (8 bf16
// of X and of the smoothing factors); the products are exact in fp32 (bf16 x bf16), so the
// maximum is exact and independent of the order; a warp-shuffle and a shared-memory max per
// block, then one atomicMax per block on the bits of the non-negative float (non-negative
// floats order like their bit patterns).  The caller's amax word is cleared on the stream
// first.  Kernels 1 and 2 read the word after their grid-dependency wait and form g there
// (act_scale_from_amax).
#pragma once

#include "ptx.cuh"

namespace svdq {

// Smallest power of two g with g * 2688 >= amax (2688 = 6 * 448), 1 for amax = 0.  Every
// product g * 2688 is exact (2688 = 21 * 2^7), so the comparisons decide exactly.
__device__ __forceinline__ float act_scale_from_amax(float amax) {
  if (!(amax > 0.f)) return 1.f;
  int e;
  (void)frexpf(amax / 2688.f, &e);                 // a first guess within a factor of two
  float g = ldexpf(1.f, e);
  while (g * 2688.f < amax) g *= 2.f;
  while (g * (0.5f * 2688.f) >= amax) g *= 0.5f;
  return g;
}

namespace k5 {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads)
act_amax_kernel(const __nv_bfloat16* __restrict__ X, const __nv_bfloat16* __restrict__ smooth, int M, int K,
                unsigned int* amax) {
  grid_dependency_wait();                          // X and the cleared word may come from the stream
  grid_launch_dependents();
  const int kv = K / 8;                            // 16-byte vectors per row
  const size_t nvec = static_cast<size_t>(M) * kv;
  float m = 0.f;
  for (size_t i = static_cast<size_t>(blockIdx.x) * kThreads + threadIdx.x; i < nvec;
       i += static_cast<size_t>(gridDim.x) * kThreads) {
    uint4 x, s;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(x.x), "=r"(x.y), "=r"(x.z), "=r"(x.w)
                 : "l"(reinterpret_cast<const uint4*>(X) + i));
    s = __ldg(reinterpret_cast<const uint4*>(smooth) + (i % kv));
    const uint32_t xw[4] = {x.x, x.y, x.z, x.w}, sw[4] = {s.x, s.y, s.z, s.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      m = fmax3(m, fabsf(bf16lo_to_f32(xw[j]) * bf16lo_to_f32(sw[j])), fabsf(bf16hi_to_f32(xw[j]) * bf16hi_to_f32(sw[j])));
    }
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
    atomicMax(amax, __float_as_uint(b));
  }
}

}  // namespace k5
}  // namespace svdq
