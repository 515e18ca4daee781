// GPU entry points of libsvdq (declared in include/svdq.h): argument checks,
// device checks, TMA descriptor encoding and kernel launches.  One translation
// unit so that the device status word is shared by all kernels.

#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <numeric>
#include <cmath>
#include <mutex>
#include <unordered_map>

#include "../../include/svdq.h"
#include "layout.h"
#include "ptx.cuh"
#include "act_amax.cuh"
#include "quant_act.cuh"
#include "gemm_nvfp4.cuh"
#include "awq_w4a16.cuh"
#include "awq_umma.cuh"
#include "gemm_gelu_quant.cuh"
#include "gemm_int4.cuh"

// Scratch of svdq_act_amax_noalloc: kernel 5's result word, partial maximum and block
// counter, for callers that cannot allocate device memory.  Every GPU that loads this
// library holds these 256 bytes until the process exits; all calls on a device share them.
static __device__ __align__(256) unsigned int g_amax_noalloc_scratch[64];

namespace {

constexpr int kMaxDevices = 64;
constexpr size_t kAmaxScratchWords = 3;       // words of g_amax_noalloc_scratch kernel 5 uses
static_assert(kAmaxScratchWords * sizeof(unsigned int) <= sizeof(g_amax_noalloc_scratch),
              "kernel 5 needs three words whatever M and K are");

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool is_pow2_scale(float g) {
  if (!(g > 0.f) || !std::isfinite(g)) return false;
  int e;
  return std::frexp(static_cast<double>(g), &e) == 0.5;
}

// Current device, checked to be compute capability 10.0 (cached per device; the caches of
// this file are atomics, so calls from several host threads are safe).
int current_device_ok(int* dev_out) {
  static std::atomic<int> cc[kMaxDevices];         // 0: not yet known, else 100 major + minor + 1
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SVDQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return SVDQ_ERR_CUDA;
  int v = cc[dev].load(std::memory_order_acquire);
  if (v == 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return SVDQ_ERR_CUDA;
    v = 100 * major + minor + 1;
    cc[dev].store(v, std::memory_order_release);
  }
  if (v != 100 * 10 + 0 + 1) return SVDQ_ERR_ARCH;
  *dev_out = dev;
  return SVDQ_OK;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// Encoded tensor maps by everything that goes into the encoding (a map describes an address
// range and its layout, not its contents, so a hit is always the map the encoder would give).
// An eager call of the GEMM needs seven maps; encoding them is most of the call's host cost.
struct TmapKey {
  uintptr_t ptr;
  uint64_t rows, cols;
  uint32_t box_cols, box_rows;
  int dt, elem, sw;
  bool operator==(const TmapKey& o) const {
    return ptr == o.ptr && rows == o.rows && cols == o.cols && box_cols == o.box_cols && box_rows == o.box_rows &&
           dt == o.dt && elem == o.elem && sw == o.sw;
  }
};
struct TmapKeyHash {
  size_t operator()(const TmapKey& k) const {
    uint64_t h = k.ptr * 0x9E3779B97F4A7C15ull;
    for (uint64_t v : {k.rows, k.cols, static_cast<uint64_t>(k.box_cols) << 32 | k.box_rows,
                       static_cast<uint64_t>(k.dt) << 16 | static_cast<uint64_t>(k.elem) << 8 |
                           static_cast<uint64_t>(k.sw)})
      h = (h ^ v) * 0x100000001B3ull;
    return static_cast<size_t>(h);
  }
};
constexpr size_t kTmapCacheMax = 4096;            // cleared when full

// 2-D row-major tensor [rows, cols] of `elem` bytes per element; box {box_cols, box_rows}.
bool make_tmap(CUtensorMap* m, const void* ptr, CUtensorMapDataType dt, int elem, uint64_t rows, uint64_t cols,
               uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle sw) {
  static std::mutex mu;
  static std::unordered_map<TmapKey, CUtensorMap, TmapKeyHash> cache;
  const TmapKey key{reinterpret_cast<uintptr_t>(ptr), rows, cols, box_cols, box_rows, static_cast<int>(dt), elem,
                    static_cast<int>(sw)};
  {
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(key);
    if (it != cache.end()) {
      *m = it->second;
      return true;
    }
  }
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * static_cast<uint64_t>(elem)};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  if (fn(m, dt, 2, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  std::lock_guard<std::mutex> lock(mu);
  if (cache.size() >= kTmapCacheMax) cache.clear();
  cache.emplace(key, *m);
  return true;
}

// Raises the dynamic shared-memory limit of one kernel, once per device.
template <auto Kernel>
bool set_smem_once(int bytes, int dev) {
  static std::atomic<bool> done[kMaxDevices];
  if (done[dev].load(std::memory_order_acquire)) return true;
  // two threads may both get here: the attribute call is idempotent
  if (cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) return false;
  done[dev].store(true, std::memory_order_release);
  return true;
}

// Allows cluster sizes above 8 for one kernel, once per device.
template <auto Kernel>
bool allow_nonportable_cluster_once(int dev) {
  static std::atomic<bool> done[kMaxDevices];
  if (done[dev].load(std::memory_order_acquire)) return true;
  if (cudaFuncSetAttribute(Kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) return false;
  done[dev].store(true, std::memory_order_release);
  return true;
}

// Number of SMs of a device (cached).
int sm_count(int dev) {
  static std::atomic<int> count[kMaxDevices];
  int c = count[dev].load(std::memory_order_relaxed);
  if (c == 0) {
    if (cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || c <= 0) c = 148;
    count[dev].store(c, std::memory_order_relaxed);
  }
  return c;
}

// Device address of g_amax_noalloc_scratch on device `dev` (which must be current).  In host
// code the array's name only stands for it: the address comes from cudaGetSymbolAddress, asked
// once per device (by the first call on that device) and cached.
int amax_noalloc_scratch(int dev, unsigned int** out) {
  static std::atomic<uintptr_t> addr[kMaxDevices];
  uintptr_t a = addr[dev].load(std::memory_order_acquire);
  if (a == 0) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_amax_noalloc_scratch) != cudaSuccess || p == nullptr) {
      (void)cudaGetLastError();
      return SVDQ_ERR_CUDA;
    }
    a = reinterpret_cast<uintptr_t>(p);
    addr[dev].store(a, std::memory_order_release);   // two threads may both get here: same value
  }
  *out = reinterpret_cast<unsigned int*>(a);
  return SVDQ_OK;
}

int launch_status() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SVDQ_OK : SVDQ_ERR_CUDA;
}

// The failure path of every kernel's bounded waits, on its own: one warp waits (through the
// same mbar_wait_bounded) for a phase of a shared-memory mbarrier at which nothing ever
// arrives, so the wait runs out after its limit, records SVDQ_ERR_TIMEOUT (site 99) in the
// device status word and the kernel returns.  No copy or tensor-core operation is in flight.
__global__ void selftest_wait_kernel() {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  const uint32_t b = svdq::smem_addr(&bar);
  if (threadIdx.x == 0) {
    svdq::mbar_init(b, 1);
    abort_flag = 0;
    svdq::fence_mbar_init();
  }
  __syncwarp();
  (void)__all_sync(0xFFFFFFFFu, svdq::mbar_wait_bounded(b, 0, &abort_flag, 99));
}

}  // namespace

extern "C" {

// Kernel 1 with the activation scale given (act_amax null) or formed on the device from the
// amax word of kernel 5.
static int quantize_impl(const void* X, const void* smooth_inv, const void* packed_w, int M, int K, int rank,
                         float act_global_scale, const void* act_amax, void* act_codes, void* act_scales,
                         void* lowrank_act, void* stream, bool int4 = false) {
  if (M < 0 || K <= 0 || rank <= 0) return SVDQ_ERR_INVALID_ARG;
  if (!act_amax && !is_pow2_scale(act_global_scale)) return SVDQ_ERR_INVALID_ARG;
  if (act_amax && (reinterpret_cast<uintptr_t>(act_amax) & 3u)) return SVDQ_ERR_INVALID_ARG;
  if (rank != svdq::kRank || K % 64 != 0) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return SVDQ_OK;                       // empty batch: nothing to read or write
  if (!X || !smooth_inv || !packed_w || !act_codes || !act_scales || !lowrank_act) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(smooth_inv) || !aligned16(packed_w) || !aligned16(act_codes) ||
      !aligned16(act_scales) || !aligned16(lowrank_act))
    return SVDQ_ERR_INVALID_ARG;
  int dev;
  if (int st = current_device_ok(&dev)) return st;

  namespace k1 = svdq::k1;
  const svdq::BlobLayout L = svdq::blob_layout(0, K, rank);   // the L1 section does not depend on N
  k1::Params p;
  p.smooth = static_cast<const __nv_bfloat16*>(smooth_inv);
  p.codes = static_cast<uint8_t*>(act_codes);
  p.scales = static_cast<uint8_t*>(act_scales);
  p.ucat = static_cast<__nv_bfloat16*>(lowrank_act);
  p.M = M;
  p.K = K;
  p.g = act_amax ? 1.0f : act_global_scale;
  p.inv_g = 1.0f / p.g;                // exact: a power of two
  p.amax = static_cast<const unsigned int*>(act_amax);

  const int rowblocks = (M + 127) / 128;               // 128-row CTAs covering the scale padding
  const int kgroups = K / 64;
  // K slices per row block (one cluster): the fewest of 1, 2, 4, 8 that keep every slice
  // whole (a multiple of 64) and within the kernel's smoothing buffer, then more while
  // the grid has fewer CTAs than two per SM
  int ks = 0;
  for (int c : {1, 2, 4, 8}) {
    if (kgroups % c == 0 && K / c <= k1::kMaxSlice) { ks = c; break; }
  }
  if (ks == 0) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  while (ks < 8 && kgroups % (2 * ks) == 0 && rowblocks * ks < 2 * sm_count(dev)) ks *= 2;
  // few row blocks (small M): 16 slices (a non-portable cluster size) while the grid still fits
  // one wave at two CTAs per SM -- shorter slices, each streamed in one round trip
  if (ks == 8 && kgroups % 16 == 0 && rowblocks * 16 <= 2 * sm_count(dev)) ks = 16;
  p.kslices = ks;

  CUtensorMap tX, tL;
  if (!make_tmap(&tX, X, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, M, K, k1::kChunk, k1::kRows,
                 CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap(&tL, static_cast<const uint8_t*>(packed_w) + L.l1s, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                 2 * k1::kRank, K, k1::kChunk, 2 * k1::kRank, CU_TENSOR_MAP_SWIZZLE_128B))
    return SVDQ_ERR_CUDA;
  const int smem = k1::kSmemBytes;
  if (!set_smem_once<k1::quant_act_lowrank_kernel<false>>(smem, dev) ||
      !set_smem_once<k1::quant_act_lowrank_kernel<true>>(smem, dev))
    return SVDQ_ERR_CUDA;
  if (ks > 8 && (!allow_nonportable_cluster_once<k1::quant_act_lowrank_kernel<false>>(dev) ||
                 !allow_nonportable_cluster_once<k1::quant_act_lowrank_kernel<true>>(dev)))
    return SVDQ_ERR_CUDA;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(rowblocks, ks, 1);
  cfg.blockDim = dim3(k1::kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = ks;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // see grid_dependency_wait
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  if ((int4 ? cudaLaunchKernelEx(&cfg, k1::quant_act_lowrank_kernel<true>, tX, tL, p)
            : cudaLaunchKernelEx(&cfg, k1::quant_act_lowrank_kernel<false>, tX, tL, p)) != cudaSuccess) {
    (void)cudaGetLastError();
    return SVDQ_ERR_CUDA;
  }
  return launch_status();
}

int svdq_quantize_act_lowrank_down(const void* X, const void* smooth_inv, const void* packed_w, int M, int K,
                                   int rank, float act_global_scale, void* act_codes, void* act_scales,
                                   void* lowrank_act, void* stream) {
  return quantize_impl(X, smooth_inv, packed_w, M, K, rank, act_global_scale, nullptr, act_codes, act_scales,
                       lowrank_act, stream);
}

int svdq_quantize_act_lowrank_down_dyn(const void* X, const void* smooth_inv, const void* packed_w, int M, int K,
                                       int rank, const void* act_amax, void* act_codes, void* act_scales,
                                       void* lowrank_act, void* stream) {
  if (!act_amax) return SVDQ_ERR_INVALID_ARG;
  return quantize_impl(X, smooth_inv, packed_w, M, K, rank, 1.0f, act_amax, act_codes, act_scales, lowrank_act,
                       stream);
}

// The QKV epilogue's extra arguments (svdq_w4a4_nvfp4_linear_qkv).
struct QkvArgs {
  int heads;
  const void* norm_wq;
  const void* norm_wk;
  float eps;
  const void* rope_cos;
  const void* rope_sin;
};

// Kernel 2 with the activation scale given (act_amax null) or formed on the device from the
// amax word of kernel 5; with qkv non-null, the instantiation whose epilogue normalises and
// rotates q and k.
static int linear_impl(const void* act_codes, const void* act_scales, const void* lowrank_act,
                       float act_global_scale, const void* act_amax, const void* packed_w, float w_global_scale,
                       int M, int N, int K, int rank, void* Y, void* stream, const QkvArgs* qkv = nullptr) {
  if (M < 0 || N <= 0 || K <= 0 || rank <= 0) return SVDQ_ERR_INVALID_ARG;
  if (!is_pow2_scale(w_global_scale)) return SVDQ_ERR_INVALID_ARG;
  if (!act_amax && !is_pow2_scale(act_global_scale)) return SVDQ_ERR_INVALID_ARG;
  if (act_amax && (reinterpret_cast<uintptr_t>(act_amax) & 3u)) return SVDQ_ERR_INVALID_ARG;
  if (act_amax) act_global_scale = 1.0f;
  if (rank != svdq::kRank || K % 64 != 0 || N % 64 != 0) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return SVDQ_OK;
  if (!act_codes || !act_scales || !lowrank_act || !packed_w || !Y) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(act_codes) || !aligned16(act_scales) || !aligned16(lowrank_act) || !aligned16(packed_w) ||
      !aligned16(Y))
    return SVDQ_ERR_INVALID_ARG;
  const double alpha = static_cast<double>(act_global_scale) * w_global_scale;
  if (!(alpha >= 0x1p-126 && alpha <= 0x1p126)) return SVDQ_ERR_INVALID_ARG;
  int dev;
  if (int st = current_device_ok(&dev)) return st;

  namespace k2 = svdq::k2;
  const uint8_t* blob = static_cast<const uint8_t*>(packed_w);
  const svdq::BlobLayout L = svdq::blob_layout(N, K, rank);
  // Output tile width: the widest that divides N (128 with a ragged last tile when N % 128 == 64:
  // its B rows, scales and L2 rows past N read as zeros, its bias from the blob's zero padding,
  // and its store is clipped at N), unless at this M its tiles would leave CTA pairs idle (few
  // rows: the kernel is bound by streaming the weights, and every pair should stream its share)
  // -- then the width giving the most tiles up to one per pair.
  const int mtiles = (M + 255) / 256;
  const int npairs = sm_count(dev) / 2;
  int BN = (N % 256 == 0) ? 256 : (N % 192 == 0 ? 192 : 128);
  if (qkv) BN = ((N / 3) % 256 == 0) ? 256 : 128;      // whole heads per tile, q/k/v thirds never straddled
  if (mtiles * (N / BN) < npairs) {
    for (int bn : {192, 128}) {
      if (qkv && bn == 192) continue;
      if (bn < BN && N % bn == 0 && mtiles * (N / bn) <= npairs && mtiles * (N / bn) > mtiles * (N / BN)) BN = bn;
    }
  }
  k2::Params p;
  p.bias = reinterpret_cast<const __nv_bfloat16*>(blob + L.bias);
  p.Y = static_cast<__nv_bfloat16*>(Y);
  p.M = M;
  p.N = N;
  p.K = K;
  p.tiles_n = (N + BN - 1) / BN;
  p.tiles = ((M + 255) / 256) * p.tiles_n;
  p.alpha = static_cast<float>(alpha);
  p.amax = static_cast<const unsigned int*>(act_amax);
  p.w_scale = w_global_scale;
  p.norm_wq = p.norm_wk = nullptr;
  p.rope_cos = p.rope_sin = nullptr;
  p.eps = 0.f;
  p.third = N;
  if (qkv) {
    p.norm_wq = static_cast<const __nv_bfloat16*>(qkv->norm_wq);
    p.norm_wk = static_cast<const __nv_bfloat16*>(qkv->norm_wk);
    p.rope_cos = static_cast<const float*>(qkv->rope_cos);
    p.rope_sin = static_cast<const float*>(qkv->rope_sin);
    p.eps = qkv->eps;
    p.third = N / 3;
  }

  const int natoms = K / 64;
  const uint64_t sfa_rows = static_cast<uint64_t>((M + 127) / 128) * natoms;
  const uint64_t sfb_rows = static_cast<uint64_t>((N + 127) / 128) * natoms;   // scale rows padded to 128
  CUtensorMap tA, tB, tSFA, tSFB, tU, tL2, tY;
  if (!make_tmap(&tA, act_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, M, K / 2, 128, k2::BM,
                 CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap(&tB, blob + L.codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, N, K / 2, 128, BN / 2,
                 CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap(&tSFA, act_scales, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, sfa_rows, 128, 128, k2::BK / 64,
                 CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_tmap(&tSFB, blob + L.scales, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, sfb_rows, 128, 128, k2::BK / 64,
                 CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_tmap(&tU, lowrank_act, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, M, 2 * rank, 2 * rank, k2::BM,
                 CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap(&tL2, blob + L.l2t, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, N, rank, rank, BN / 2,
                 CU_TENSOR_MAP_SWIZZLE_64B) ||
      !make_tmap(&tY, Y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, M, N, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B))
    return SVDQ_ERR_CUDA;

  const int pairs = std::min(p.tiles, sm_count(dev) / 2);
  const dim3 grid(2 * pairs, 1, 1);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
#define SVDQ_GEMM_LAUNCH(BN_, QKV_)                                                                 \
  do {                                                                                              \
    const int smem = k2::Cfg<BN_, QKV_>::SMEM_BYTES;                                                \
    if (!set_smem_once<k2::nvfp4_gemm_kernel<BN_, QKV_>>(smem, dev)) return SVDQ_ERR_CUDA;          \
    cudaLaunchConfig_t cfg = {};                                                                    \
    cfg.gridDim = grid;                                                                             \
    cfg.blockDim = dim3(k2::kThreads, 1, 1);                                                        \
    cfg.dynamicSmemBytes = smem;                                                                    \
    cfg.stream = s;                                                                                 \
    cudaLaunchAttribute attr[1];                                                                    \
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;                                \
    attr[0].val.programmaticStreamSerializationAllowed = 1;                                         \
    cfg.attrs = attr;                                                                               \
    cfg.numAttrs = 1;                                                                               \
    if (cudaLaunchKernelEx(&cfg, k2::nvfp4_gemm_kernel<BN_, QKV_>, tA, tB, tSFA, tSFB, tU, tL2, tY, p) != \
        cudaSuccess) {                                                                              \
      (void)cudaGetLastError();                                                                     \
      return SVDQ_ERR_CUDA;                                                                         \
    }                                                                                               \
  } while (0)
  if (qkv) {
    if (BN == 256) SVDQ_GEMM_LAUNCH(256, true);
    else SVDQ_GEMM_LAUNCH(128, true);
  } else if (BN == 192) {
    SVDQ_GEMM_LAUNCH(192, false);
  } else if (BN == 256) {
    SVDQ_GEMM_LAUNCH(256, false);
  } else {
    SVDQ_GEMM_LAUNCH(128, false);
  }
#undef SVDQ_GEMM_LAUNCH
  return launch_status();
}

int svdq_w4a4_nvfp4_linear(const void* act_codes, const void* act_scales, const void* lowrank_act,
                           float act_global_scale, const void* packed_w, float w_global_scale, int M, int N, int K,
                           int rank, void* Y, void* stream) {
  return linear_impl(act_codes, act_scales, lowrank_act, act_global_scale, nullptr, packed_w, w_global_scale, M, N,
                     K, rank, Y, stream);
}

int svdq_w4a4_nvfp4_linear_dyn(const void* act_codes, const void* act_scales, const void* lowrank_act,
                               const void* act_amax, const void* packed_w, float w_global_scale, int M, int N, int K,
                               int rank, void* Y, void* stream) {
  if (!act_amax) return SVDQ_ERR_INVALID_ARG;
  return linear_impl(act_codes, act_scales, lowrank_act, 1.0f, act_amax, packed_w, w_global_scale, M, N, K, rank, Y,
                     stream);
}

int svdq_w4a4_nvfp4_linear_qkv(const void* act_codes, const void* act_scales, const void* lowrank_act,
                               float act_global_scale, const void* packed_w, float w_global_scale, int M, int N,
                               int K, int rank, int heads, int head_dim, const void* norm_wq, const void* norm_wk,
                               float eps, const void* rope_cos, const void* rope_sin, void* Y, void* stream) {
  if (heads <= 0 || head_dim <= 0 || !(eps >= 0.f) || !std::isfinite(eps)) return SVDQ_ERR_INVALID_ARG;
  if (head_dim != 128 || N != 3 * heads * head_dim) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  if (M > 0) {
    if (!norm_wq || !norm_wk || !rope_cos || !rope_sin) return SVDQ_ERR_INVALID_ARG;
    if (!aligned16(norm_wq) || !aligned16(norm_wk) || !aligned16(rope_cos) || !aligned16(rope_sin))
      return SVDQ_ERR_INVALID_ARG;
  }
  const QkvArgs q{heads, norm_wq, norm_wk, eps, rope_cos, rope_sin};
  return linear_impl(act_codes, act_scales, lowrank_act, act_global_scale, nullptr, packed_w, w_global_scale, M, N,
                     K, rank, Y, stream, &q);
}

// Tile partition of kernel 6: pairs, and the partial slots per pair (row blocks a pair's
// contiguous range of the row-major tile order can touch).
static void gelu_quant_partition(int M, int N, int dev, int* npairs, int* slots) {
  const int tiles_n = N / svdq::k6::BN;
  const int tiles = ((M + 255) / 256) * tiles_n;
  const int P = std::max(1, std::min(tiles, sm_count(dev) / 2));
  int sl = 1;
  for (int p = 0; p < P; ++p) {
    const int a = svdq::k6::range_start(p, tiles, P), b = svdq::k6::range_start(p + 1, tiles, P);
    if (b > a) sl = std::max(sl, (b - 1) / tiles_n - a / tiles_n + 1);
  }
  *npairs = P;
  *slots = sl;
}

size_t svdq_gelu_table_bytes(void) { return 65536 * sizeof(uint16_t); }

int svdq_gelu_table_fill(void* table, void* stream) {
  if (!table || !aligned16(table)) return SVDQ_ERR_INVALID_ARG;
  int dev;
  if (int st = current_device_ok(&dev)) return st;
  svdq::k6::gelu_table_kernel<<<256, 256, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<uint16_t*>(table));
  return launch_status();
}

size_t svdq_gelu_quant_workspace_bytes(int M, int N) {
  if (M <= 0 || N <= 0 || N % 128 != 0) return 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    (void)cudaGetLastError();
    return 0;
  }
  int P, slots;
  gelu_quant_partition(M, N, dev, &P, &slots);
  return static_cast<size_t>(P) * slots * 256 * 32 * sizeof(float);
}

int svdq_w4a4_nvfp4_linear_gelu_quant(const void* act_codes, const void* act_scales, const void* lowrank_act,
                                      float act_global_scale, const void* packed_w, float w_global_scale, int M,
                                      int N, int K, int rank, const void* down_smooth_inv, const void* down_packed_w,
                                      float down_act_global_scale, void* out_codes, void* out_scales,
                                      void* out_lowrank_act, void* workspace, size_t workspace_bytes,
                                      const void* gelu_table, void* h_out, void* stream) {
  if (M < 0 || N <= 0 || K <= 0 || rank <= 0) return SVDQ_ERR_INVALID_ARG;
  if (!is_pow2_scale(act_global_scale) || !is_pow2_scale(w_global_scale) || !is_pow2_scale(down_act_global_scale))
    return SVDQ_ERR_INVALID_ARG;
  if (rank != svdq::kRank || K % 64 != 0 || N % 128 != 0) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  const double alpha = static_cast<double>(act_global_scale) * w_global_scale;
  if (!(alpha >= 0x1p-126 && alpha <= 0x1p126)) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  if (!act_codes || !act_scales || !lowrank_act || !packed_w || !down_smooth_inv || !down_packed_w || !out_codes ||
      !out_scales || !out_lowrank_act || !workspace || !gelu_table)
    return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(act_codes) || !aligned16(act_scales) || !aligned16(lowrank_act) || !aligned16(packed_w) ||
      !aligned16(down_smooth_inv) || !aligned16(down_packed_w) || !aligned16(out_codes) || !aligned16(out_scales) ||
      !aligned16(out_lowrank_act) || !aligned16(workspace) || !aligned16(gelu_table) || (h_out && !aligned16(h_out)))
    return SVDQ_ERR_INVALID_ARG;
  int dev;
  if (int st = current_device_ok(&dev)) return st;
  namespace k6 = svdq::k6;
  int P, slots;
  gelu_quant_partition(M, N, dev, &P, &slots);
  if (workspace_bytes < static_cast<size_t>(P) * slots * 256 * 32 * sizeof(float)) return SVDQ_ERR_INVALID_ARG;

  const uint8_t* blob = static_cast<const uint8_t*>(packed_w);
  const svdq::BlobLayout L = svdq::blob_layout(N, K, rank);
  const svdq::BlobLayout LD = svdq::blob_layout(0, N, rank);   // the down blob's L1 section (its K is N)
  k6::Params p;
  p.bias = reinterpret_cast<const __nv_bfloat16*>(blob + L.bias);
  p.smooth = static_cast<const __nv_bfloat16*>(down_smooth_inv);
  p.codes = static_cast<uint8_t*>(out_codes);
  p.scales = static_cast<uint8_t*>(out_scales);
  p.ws = static_cast<float*>(workspace);
  p.h_out = static_cast<__nv_bfloat16*>(h_out);
  p.gelu = static_cast<const uint16_t*>(gelu_table);
  p.M = M;
  p.N = N;
  p.K = K;
  p.tiles_n = N / k6::BN;
  p.tiles = ((M + 255) / 256) * p.tiles_n;
  p.slots = slots;
  p.alpha = static_cast<float>(alpha);
  p.g = down_act_global_scale;
  p.inv_g = 1.0f / down_act_global_scale;         // exact: a power of two

  const int natoms = K / 64;
  const uint64_t sfa_rows = static_cast<uint64_t>((M + 127) / 128) * natoms;
  const uint64_t sfb_rows = static_cast<uint64_t>(N / 128) * natoms;
  CUtensorMap tA, tB, tSFA, tSFB, tU, tL2, tL1;
  if (!make_tmap(&tA, act_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, M, K / 2, 128, k6::BM,
                 CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap(&tB, blob + L.codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, N, K / 2, 128, k6::BN_HALF,
                 CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap(&tSFA, act_scales, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, sfa_rows, 128, 128, k6::BK / 64,
                 CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_tmap(&tSFB, blob + L.scales, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, sfb_rows, 128, 128, k6::BK / 64,
                 CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_tmap(&tU, lowrank_act, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, M, 2 * rank, 2 * rank, k6::BM,
                 CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap(&tL2, blob + L.l2t, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, N, rank, rank, k6::BN_HALF,
                 CU_TENSOR_MAP_SWIZZLE_64B) ||
      !make_tmap(&tL1, static_cast<const uint8_t*>(down_packed_w) + LD.l1s, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                 2 * rank, N, 64, 16, CU_TENSOR_MAP_SWIZZLE_128B))
    return SVDQ_ERR_CUDA;
  if (!set_smem_once<k6::gemm_gelu_quant_kernel>(k6::SMEM_BYTES, dev)) return SVDQ_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * P, 1, 1);
  cfg.blockDim = dim3(k6::kThreads, 1, 1);
  cfg.dynamicSmemBytes = k6::SMEM_BYTES;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, k6::gemm_gelu_quant_kernel, tA, tB, tSFA, tSFB, tU, tL2, tL1, p) != cudaSuccess) {
    (void)cudaGetLastError();
    return SVDQ_ERR_CUDA;
  }
  cudaLaunchConfig_t cfg2 = {};
  cfg2.gridDim = dim3((M * 8 + 255) / 256, 1, 1);
  cfg2.blockDim = dim3(256, 1, 1);
  cfg2.stream = s;
  cfg2.attrs = attr;
  cfg2.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg2, k6::u_reduce_kernel, static_cast<const float*>(workspace), M, p.tiles_n, p.tiles, P,
                         slots, p.inv_g, static_cast<__nv_bfloat16*>(out_lowrank_act)) != cudaSuccess) {
    (void)cudaGetLastError();
    return SVDQ_ERR_CUDA;
  }
  return launch_status();
}

int svdq_int4_quantize_act_lowrank_down(const void* X, const void* smooth_inv, const void* packed_w, int M, int K,
                                        int rank, void* act_codes, void* act_scales, void* lowrank_act, void* stream) {
  return quantize_impl(X, smooth_inv, packed_w, M, K, rank, 1.0f, nullptr, act_codes, act_scales, lowrank_act, stream,
                       true);
}

int svdq_w4a4_int4_linear(const void* act_codes, const void* act_scales, const void* lowrank_act, const void* packed_w,
                          int M, int N, int K, int rank, void* Y, void* stream) {
  if (M < 0 || N <= 0 || K <= 0 || rank <= 0) return SVDQ_ERR_INVALID_ARG;
  if (rank != svdq::kRank || K % 64 != 0 || N % 128 != 0) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return SVDQ_OK;
  if (!act_codes || !act_scales || !lowrank_act || !packed_w || !Y) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(act_codes) || !aligned16(act_scales) || !aligned16(lowrank_act) || !aligned16(packed_w) ||
      !aligned16(Y))
    return SVDQ_ERR_INVALID_ARG;
  int dev;
  if (int st = current_device_ok(&dev)) return st;
  namespace k8 = svdq::k8;
  const uint8_t* blob = static_cast<const uint8_t*>(packed_w);
  const svdq::BlobLayout L = svdq::blob_layout_int4(N, K, rank);
  k8::Params p;
  const float* w_scales = reinterpret_cast<const float*>(blob + L.scales);
  p.bias = reinterpret_cast<const __nv_bfloat16*>(blob + L.bias);
  p.M = M;
  p.N = N;
  p.K = K;
  p.tiles_n = N / k8::BN;
  p.tiles = ((M + k8::BM - 1) / k8::BM) * p.tiles_n;
  CUtensorMap tA, tB, tU, tL2, tY, tWS, tAS;
  const int mpad = (M + 127) / 128 * 128;
  if (!make_tmap(&tA, act_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, M, K, 128, k8::BM, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap(&tB, blob + L.codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, N, K, 128, k8::BN,
                 CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap(&tU, lowrank_act, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, M, 2 * rank, 2 * rank, k8::BM,
                 CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap(&tL2, blob + L.l2t, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, N, rank, rank, k8::BN,
                 CU_TENSOR_MAP_SWIZZLE_64B) ||
      !make_tmap(&tY, Y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, M, N, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B) ||
      !make_tmap(&tWS, w_scales, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, K / 64, N, k8::BN, 1,
                 CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_tmap(&tAS, act_scales, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, K / 64, mpad, k8::BM, 1,
                 CU_TENSOR_MAP_SWIZZLE_NONE))
    return SVDQ_ERR_CUDA;
  if (!set_smem_once<k8::int4_gemm_kernel>(k8::SMEM_BYTES, dev)) return SVDQ_ERR_CUDA;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(std::min(p.tiles, sm_count(dev)), 1, 1);
  cfg.blockDim = dim3(k8::kThreads, 1, 1);
  cfg.dynamicSmemBytes = k8::SMEM_BYTES;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, k8::int4_gemm_kernel, tA, tB, tU, tL2, tY, tWS, tAS, p) != cudaSuccess) {
    (void)cudaGetLastError();
    return SVDQ_ERR_CUDA;
  }
  return launch_status();
}

int svdq_act_amax(const void* X, const void* smooth_inv, int M, int K, void* act_amax, void* stream) {
  if (M < 0 || K <= 0 || K % 64 != 0) return SVDQ_ERR_INVALID_ARG;
  if (!act_amax || !aligned16(act_amax)) return SVDQ_ERR_INVALID_ARG;
  if (M > 0 && (!X || !smooth_inv || !aligned16(X) || !aligned16(smooth_inv))) return SVDQ_ERR_INVALID_ARG;
  int dev;
  if (int st = current_device_ok(&dev)) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (M == 0) {                                     // amax of an empty batch: 0 (g = 1)
    if (cudaMemsetAsync(act_amax, 0, sizeof(unsigned int), s) != cudaSuccess) {
      (void)cudaGetLastError();
      return SVDQ_ERR_CUDA;
    }
    return SVDQ_OK;
  }
  namespace k5 = svdq::k5;
  // a multiple of q blocks, so that the grid's thread count is a multiple of the row's K / 8
  // units (the kernel keeps one column per thread); up to 8 blocks per SM
  const int kv = K / 8;
  const int q = kv / std::gcd(kv, k5::kThreads);
  const size_t nvec = static_cast<size_t>(M) * kv;
  const size_t want = (nvec + k5::kThreads - 1) / k5::kThreads;
  const size_t cap = static_cast<size_t>(sm_count(dev)) * 8;
  const int blocks = static_cast<int>(std::max<size_t>(q, std::min(want, cap) / q * q));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(blocks, 1, 1);
  cfg.blockDim = dim3(k5::kThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, k5::act_amax_kernel, static_cast<const __nv_bfloat16*>(X),
                         static_cast<const __nv_bfloat16*>(smooth_inv), M, K,
                         static_cast<unsigned int*>(act_amax)) != cudaSuccess) {
    (void)cudaGetLastError();
    return SVDQ_ERR_CUDA;
  }
  return launch_status();
}

// Kernel 5 with its scratch words in g_amax_noalloc_scratch instead of a caller buffer: the
// scratch is cleared, the kernel runs on it, and its result word is copied to `amax`.  Nothing
// is allocated.  Calls that overlap on the GPU share the scratch and race.
int svdq_act_amax_noalloc(const void* X, const void* smooth_inv, int M, int K, void* amax, void* stream) {
  if (M < 0 || K <= 0 || K % 64 != 0) return SVDQ_ERR_INVALID_ARG;
  if (!amax || (reinterpret_cast<uintptr_t>(amax) & 3u)) return SVDQ_ERR_INVALID_ARG;
  if (M > 0 && (!X || !smooth_inv || !aligned16(X) || !aligned16(smooth_inv))) return SVDQ_ERR_INVALID_ARG;
  int dev;
  if (int st = current_device_ok(&dev)) return st;
  unsigned int* scratch = nullptr;
  if (int st = amax_noalloc_scratch(dev, &scratch)) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the kernel expects its partial maximum and block counter at zero; it leaves them so, but a
  // call is not to depend on what an earlier one left behind
  if (cudaMemsetAsync(scratch, 0, kAmaxScratchWords * sizeof(unsigned int), s) != cudaSuccess) {
    (void)cudaGetLastError();
    return SVDQ_ERR_CUDA;
  }
  if (M > 0) {
    namespace k5 = svdq::k5;
    const int kv = K / 8;
    const int q = kv / std::gcd(kv, k5::kThreads);
    const size_t nvec = static_cast<size_t>(M) * kv;
    const size_t want = (nvec + k5::kThreads - 1) / k5::kThreads;
    const size_t cap = static_cast<size_t>(sm_count(dev)) * 8;
    const int blocks = static_cast<int>(std::max<size_t>(q, std::min(want, cap) / q * q));
    k5::act_amax_kernel<<<blocks, k5::kThreads, 0, s>>>(static_cast<const __nv_bfloat16*>(X),
                                                         static_cast<const __nv_bfloat16*>(smooth_inv), M, K,
                                                         scratch);
    if (cudaGetLastError() != cudaSuccess) return SVDQ_ERR_CUDA;
  }
  // word 0: the result (0 for an empty batch, from the clearing above)
  if (cudaMemcpyAsync(amax, scratch, sizeof(unsigned int), cudaMemcpyDeviceToDevice, s) != cudaSuccess) {
    (void)cudaGetLastError();
    return SVDQ_ERR_CUDA;
  }
  return SVDQ_OK;
}

int awq_w4a16_linear(const void* X, const void* qweight, const void* scales, const void* zeros, const void* bias,
                     int M, int N, int K, void* Y, void* stream) {
  if (M < 0 || N <= 0 || K <= 0) return SVDQ_ERR_INVALID_ARG;
  if (N % 64 != 0 || K % 64 != 0) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return SVDQ_OK;
  if (!X || !qweight || !scales || !zeros || !Y) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(qweight) || !aligned16(Y) || (reinterpret_cast<uintptr_t>(scales) & 1u) ||
      (reinterpret_cast<uintptr_t>(zeros) & 1u) || (bias && (reinterpret_cast<uintptr_t>(bias) & 1u)))
    return SVDQ_ERR_INVALID_ARG;
  int dev;
  if (int st = current_device_ok(&dev)) return st;

  namespace k3 = svdq::k3;
  k3::Params p;
  p.scales = static_cast<const __nv_bfloat16*>(scales);
  p.zeros = static_cast<const __nv_bfloat16*>(zeros);
  p.bias = static_cast<const __nv_bfloat16*>(bias);
  p.Y = static_cast<__nv_bfloat16*>(Y);
  p.M = M;
  p.N = N;
  p.K = K;
  const bool vec = K % 256 == 0 && !(reinterpret_cast<uintptr_t>(scales) & 7u) &&
                   !(reinterpret_cast<uintptr_t>(zeros) & 7u);   // 8-byte loads of four groups
  // M <= 8: mma.sync kernel (one 8-token tile); M > 8: tcgen05 kernel with T = 16, 32 or 64 token
  // columns, M > 64 in 64-token tiles (a grid row per tile; each re-reads the weights, from L2)
  const int tx = M <= 8 ? 8 : (M <= 16 ? 16 : (M <= 32 ? 32 : 64));
  CUtensorMap tW, tX;
  if (!make_tmap(&tW, qweight, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, N, K / 2, 128, k3::kRows,
                 CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap(&tX, X, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, M, K, 64, tx, CU_TENSOR_MAP_SWIZZLE_128B))
    return SVDQ_ERR_CUDA;
  const dim3 grid((N + k3::kRows - 1) / k3::kRows, (M + tx - 1) / tx, 1);
  cudaStream_t s = static_cast<cudaStream_t>(stream);

#define SVDQ_AWQ_LAUNCH(KERNEL, SMEM_, THREADS_, ...)                                           \
  do {                                                                                          \
    const int smem = SMEM_;                                                                     \
    if (!set_smem_once<KERNEL>(smem, dev)) return SVDQ_ERR_CUDA;                                \
    cudaLaunchConfig_t cfg = {};                                                                \
    cfg.gridDim = grid;                                                                         \
    cfg.blockDim = dim3(THREADS_, 1, 1);                                                        \
    cfg.dynamicSmemBytes = smem;                                                                \
    cfg.stream = s;                                                                             \
    cudaLaunchAttribute attr[1];                                                                \
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;                            \
    attr[0].val.programmaticStreamSerializationAllowed = 1;                                     \
    cfg.attrs = attr;                                                                           \
    cfg.numAttrs = 1;                                                                           \
    if (cudaLaunchKernelEx(&cfg, KERNEL, __VA_ARGS__) != cudaSuccess) {                         \
      (void)cudaGetLastError();                                                                 \
      return SVDQ_ERR_CUDA;                                                                     \
    }                                                                                           \
  } while (0)

  // the CTA's scale and zero rows staged in shared memory by two copies (K / 64 groups of 128 rows
  // each; the copies want 16-byte rows and a 16-byte aligned base)
  const int gpr = K / 64;
  CUtensorMap tS = tW, tZ = tW;
  static_assert(k3::kMaxSzGroups == svdq::k4::kMaxSzGroups && k3::kRows == svdq::k4::kRows, "one staging rule");
  const bool sz = K % 512 == 0 && gpr <= k3::kMaxSzGroups && aligned16(scales) && aligned16(zeros) &&
                  make_tmap(&tS, scales, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, N, gpr, gpr, k3::kRows,
                            CU_TENSOR_MAP_SWIZZLE_NONE) &&
                  make_tmap(&tZ, zeros, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, N, gpr, gpr, k3::kRows,
                            CU_TENSOR_MAP_SWIZZLE_NONE);
  if (tx == 8) {
    if (sz) SVDQ_AWQ_LAUNCH((k3::awq_gemm_kernel<true, true>), k3::kSmem, k3::kThreads, tW, tX, tS, tZ, p);
    else if (vec) SVDQ_AWQ_LAUNCH((k3::awq_gemm_kernel<true, false>), k3::kSmem, k3::kThreads, tW, tX, tS, tZ, p);
    else SVDQ_AWQ_LAUNCH((k3::awq_gemm_kernel<false, false>), k3::kSmem, k3::kThreads, tW, tX, tS, tZ, p);
  } else {
    namespace k4 = svdq::k4;
    k4::Params q;
    q.scales = p.scales;
    q.zeros = p.zeros;
    q.bias = p.bias;
    q.Y = p.Y;
    q.M = M;
    q.N = N;
    q.K = K;
    if (tx == 16) {
      if (sz) SVDQ_AWQ_LAUNCH((k4::awq_umma_kernel<16, true, true>), k4::Cfg<16>::SMEM, k4::kThreads, tW, tX, tS, tZ, q);
      else if (vec) SVDQ_AWQ_LAUNCH((k4::awq_umma_kernel<16, true, false>), k4::Cfg<16>::SMEM, k4::kThreads, tW, tX, tS, tZ, q);
      else SVDQ_AWQ_LAUNCH((k4::awq_umma_kernel<16, false, false>), k4::Cfg<16>::SMEM, k4::kThreads, tW, tX, tS, tZ, q);
    } else if (tx == 32) {
      if (sz) SVDQ_AWQ_LAUNCH((k4::awq_umma_kernel<32, true, true>), k4::Cfg<32>::SMEM, k4::kThreads, tW, tX, tS, tZ, q);
      else if (vec) SVDQ_AWQ_LAUNCH((k4::awq_umma_kernel<32, true, false>), k4::Cfg<32>::SMEM, k4::kThreads, tW, tX, tS, tZ, q);
      else SVDQ_AWQ_LAUNCH((k4::awq_umma_kernel<32, false, false>), k4::Cfg<32>::SMEM, k4::kThreads, tW, tX, tS, tZ, q);
    } else {
      if (sz) SVDQ_AWQ_LAUNCH((k4::awq_umma_kernel<64, true, true>), k4::Cfg<64>::SMEM, k4::kThreads, tW, tX, tS, tZ, q);
      else if (vec) SVDQ_AWQ_LAUNCH((k4::awq_umma_kernel<64, true, false>), k4::Cfg<64>::SMEM, k4::kThreads, tW, tX, tS, tZ, q);
      else SVDQ_AWQ_LAUNCH((k4::awq_umma_kernel<64, false, false>), k4::Cfg<64>::SMEM, k4::kThreads, tW, tX, tS, tZ, q);
    }
  }
#undef SVDQ_AWQ_LAUNCH
  return launch_status();
}

int svdq_selftest_wait_timeout(void* stream) {
  int dev;
  if (int st = current_device_ok(&dev)) return st;
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>();
  return launch_status();
}

int svdq_device_status(int clear) {
  unsigned int v = 0;
  if (cudaDeviceSynchronize() != cudaSuccess) return SVDQ_ERR_CUDA;
  if (cudaMemcpyFromSymbol(&v, svdq::g_device_status, sizeof(v)) != cudaSuccess) return SVDQ_ERR_CUDA;
  if (clear) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(svdq::g_device_status, &zero, sizeof(zero)) != cudaSuccess) return SVDQ_ERR_CUDA;
  }
  if (v & 1u) return SVDQ_ERR_TIMEOUT;
  return (v & 2u) ? SVDQ_ERR_SCALE_RANGE : SVDQ_OK;
}

}  // extern "C"
