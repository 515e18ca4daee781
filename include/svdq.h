/*
 * svdq.h -- C ABI of libsvdq: the SVDQuant W4A4 (NVFP4) linear layer and the
 * AWQ-style W4A16 (int4, group 64) linear layer on NVIDIA B200 (sm_100a).
 *
 * What is computed.  "Nunchaku Lite" (Hugging Face Diffusers docs), section
 * "Supported quantization types": svdq_w4a4 with nvfp4 precision and group
 * size 16 runs an NVFP4 runtime kernel with an SVDQ low-rank correction;
 * awq_w4a16 with int4 precision and group size 64 runs an AWQ-style INT4
 * weight-only kernel.  Section "NunchakuLiteQuantizationConfig": rank 32.  The
 * Indonesian article on Nunchaku Lite (section on what happens when a
 * diffusion model is quantized) describes the split: activation outliers go to
 * a 16-bit low-rank branch, the rest runs with 4-bit weights and 4-bit
 * activations.  The layer is
 *
 *     X_hat = X * smooth_inv                (smooth_inv[k] = 1/lambda_k)
 *     y     = g_a g_w (Q(X_hat) Q(R)^T) + (X_hat L1) L2 + b
 *
 * with Q the NVFP4 quantizer: one E4M3 scale per 16 contiguous K elements,
 * E2M1 codes, and a power-of-two per-tensor scale g (g_a for activations,
 * supplied by the caller from calibration; g_w for the weight residual R,
 * computed by svdq_pack_weights).  Block scale S = RNE_E4M3(amax/(6 g)),
 * saturating at 448; code = RNE_E2M1(clamp(x/(S g), -6, 6)) with the IEEE sign
 * kept; a block whose scale rounds to 0 gets all-zero codes.
 *
 * Conventions shared by every call.
 *   - Matrices are row-major.  W, R are stored [N, K] (nn.Linear layout, K
 *     contiguous); X, Y are [M, K] and [M, N].  bf16 tensors are passed as
 *     uint16 bit patterns (host) or raw device pointers.
 *   - Packed 4-bit codes: two per byte, element 2i in the low nibble.
 *   - Scale-factor tensors ("swizzled scales") hold E4M3 codes in 512-byte
 *     atoms of 128 rows x 4 scales (64 K elements): row blocks of 128 rows are
 *     outermost, the K/64 atoms of a row block follow each other, and inside an
 *     atom the scale of row i (0..127), group j (0..3) is at byte
 *     (i % 32) * 16 + (i / 32) * 4 + j.  Row counts are padded up to 128.
 *   - Ownership: the caller allocates and frees every buffer (host and
 *     device).  The GPU entry points allocate nothing, never synchronize, and
 *     enqueue their kernels on `stream` (a cudaStream_t; NULL is the legacy
 *     default stream) of the current device.
 *   - Errors: every call checks its arguments first and returns a status
 *     without launching anything when one is wrong.  Launch failures return
 *     SVDQ_ERR_CUDA.  The kernels bound every wait on an mbarrier; a wait that
 *     runs out (about one second) records SVDQ_ERR_TIMEOUT in a device-side
 *     status word that svdq_device_status() reads, and the kernel releases its
 *     tensor memory and returns instead of hanging.
 *   - M == 0 is a valid empty call: once the sizes and scales pass their
 *     checks it returns SVDQ_OK without touching the device (the M-sized
 *     buffers may then be NULL).
 */
#ifndef SVDQ_H_
#define SVDQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SVDQ_OK = 0,
  SVDQ_ERR_INVALID_ARG = 1,        /* null pointer, bad count, misaligned pointer, non power-of-two scale */
  SVDQ_ERR_UNSUPPORTED_SHAPE = 2,  /* a dimension outside the supported tiling */
  SVDQ_ERR_ARCH = 3,               /* current device is not compute capability 10.0 (B200) */
  SVDQ_ERR_CUDA = 4,               /* a CUDA runtime/driver call or a launch failed */
  SVDQ_ERR_TIMEOUT = 5,            /* a kernel gave up on a bounded wait (see svdq_device_status) */
  SVDQ_ERR_SCALE_RANGE = 6         /* a device-side g_a g_w left [2^-126, 2^126] (see svdq_device_status) */
} svdq_status;

/* Fixed parameters of the method table ("Supported quantization types"). */
#define SVDQ_RANK 32
#define SVDQ_NVFP4_GROUP 16
#define SVDQ_AWQ_GROUP 64

/* Human-readable name of a status code.  Never returns NULL. */
const char* svdq_status_string(int status);

/* ABI version of this header (bumped on any incompatible change). */
int svdq_abi_version(void);

/* ------------------------------------------------------------------ weights */

/* Bytes of the packed weight blob for an [N, K] residual with rank `rank`.
 * Returns 0 for unsupported arguments (see svdq_pack_weights). */
size_t svdq_packed_weight_bytes(int N, int K, int rank);

/* Host-side weight preparation (no GPU work).
 *   R     float32 [N, K]   residual weight W diag(lambda) - (L1 L2)^T.
 *   L1    bf16   [K, rank] low-rank down factor (math orientation).
 *   L2    bf16   [rank, N] low-rank up factor.
 *   bias  bf16   [N] or NULL (then the bias is zero).
 *   smooth_inv bf16 [K]    the layer's 1/lambda; the same vector must be passed
 *                          to svdq_quantize_act_lowrank_down.
 *   N % 64 == 0, K % 64 == 0, N, K > 0, rank == 32 (the fused QKV and MLP calls and the int4 row
 *   need N % 128 == 0).
 *   out   host buffer of out_bytes >= svdq_packed_weight_bytes(N, K, rank).
 *   w_global_scale  receives g_w = 2^ceil(log2(amax(R) / 2688)) (1 if R == 0).
 * The blob is device-private: copy it to the GPU as it is and pass that copy
 * as `packed_w`.  It holds: a 1 KB header ("SVDQNVF4", N, K, rank, g_w);
 * (diag(smooth_inv) L1)^T [rank, K] split exactly into a high and a low bf16
 * part (each product of two bf16 values has at most 16 significant bits); the
 * NVFP4 codes of R [N, K/2] and their swizzled E4M3 scales; (L2 / g_w)
 * transposed to [N, rank] (exact: g_w is a power of two); the bias [N] (bf16).
 * Sections are aligned to 1024 bytes.  Codes and scales are bit-exact to the
 * definition above (RNE on exact quotients).
 * Returns SVDQ_ERR_INVALID_ARG for null pointers or a short buffer, and
 * SVDQ_ERR_UNSUPPORTED_SHAPE for dimensions outside the rules above, or when R
 * holds a NaN or infinity. */
int svdq_pack_weights(const float* R, const uint16_t* L1, const uint16_t* L2,
                      const uint16_t* bias, const uint16_t* smooth_inv, int N, int K, int rank,
                      void* out, size_t out_bytes, float* w_global_scale);

/* ------------------------------------------------------------- activations */

/* Bytes of a swizzled activation-scale buffer for M rows and K columns:
 * ceil(M/128)*128 * K/16.  Rows M..ceil(M/128)*128-1 are written as zero. */
size_t svdq_act_scale_bytes(int M, int K);

/* Kernel 1: smoothing, NVFP4 quantization and the rank-32 down-projection, in
 * one pass over X (the low-rank branch, kept in 16-bit precision, is fed from
 * the same smoothed values that are quantized).
 *   X           device bf16 [M, K] (16-byte aligned rows: K % 64 == 0)
 *   smooth_inv  device bf16 [K], the per-channel 1/lambda
 *   packed_w    device copy of the blob from svdq_pack_weights (its L1 is used;
 *               N is not needed here)
 *   act_global_scale  g_a > 0, a power of two (static calibration)
 *   act_codes   device u8 [M, K/2] out: E2M1 codes of X_hat
 *   act_scales  device u8 [svdq_act_scale_bytes(M, K)] out: swizzled E4M3 scales
 *   lowrank_act device bf16 [M, 2*rank] out: U / g_a with U = X_hat L1,
 *               stored as a high part (columns 0..rank-1) and a low part
 *               (columns rank..2*rank-1), U = g_a (hi + lo) to 2^-16 relative.
 *               The product is formed exactly (X times the packed exact split
 *               of diag(smooth_inv) L1) and accumulated in fp32.
 * K % 64 == 0, rank == 32, M >= 0.  Asynchronous on `stream`. */
int svdq_quantize_act_lowrank_down(const void* X, const void* smooth_inv,
                                   const void* packed_w, int M, int K, int rank,
                                   float act_global_scale, void* act_codes,
                                   void* act_scales, void* lowrank_act, void* stream);

/* Kernel 2: the NVFP4 block-scaled GEMM on tcgen05 with the low-rank up
 * projection, the bias and the bf16 cast fused in the epilogue:
 *   Y = bf16( g_a g_w (Q(X_hat) Q(R)^T) + lowrank_act L2 + b ).
 * The low-rank term is (hi + lo)(L2 / g_w) accumulated with the FP4 products
 * in one fp32 accumulator and scaled by g_a g_w once, in the epilogue.
 *   act_codes, act_scales, lowrank_act  outputs of kernel 1 for the same M, K
 *   act_global_scale  the g_a given to kernel 1 (power of two)
 *   packed_w          device copy of the blob; w_global_scale its g_w
 *   Y                 device bf16 [M, N] out
 * N % 64 == 0 (when N % 128 == 64 the last output tile is 128 columns wide and ragged), K % 64 ==
 * 0, rank == 32, M >= 0; all pointers 16-byte aligned.  Asynchronous on `stream`. */
int svdq_w4a4_nvfp4_linear(const void* act_codes, const void* act_scales,
                           const void* lowrank_act, float act_global_scale,
                           const void* packed_w, float w_global_scale,
                           int M, int N, int K, int rank, void* Y, void* stream);

/* Kernel 2 for a fused Q/K/V projection, with the per-head RMSNorm of q and k and their
 * rotary position embedding (RoPE) done in the GEMM's epilogue -- "Nunchaku Lite" docs,
 * section on fused kernels: the original engine fuses the Q, K, V projections with RMSNorm and
 * RoPE (its benchmark table gives the RMSNorm + RoPE epilogue 1.236x and the whole fusion
 * 1.27x).  The pages name the operations only; the readings used:
 *   - Y [M, N] holds q, k, v side by side, N = 3 * heads * head_dim, each third head-major
 *     (head h at columns h * head_dim .. + head_dim - 1 of its third);
 *   - y = g_a g_w (Q(X_hat) Q(R)^T) + lowrank_act L2 + b as in svdq_w4a4_nvfp4_linear, kept in
 *     fp32 (not rounded to bf16 before the normalisation);
 *   - q and k heads: x / sqrt(mean(x^2) + eps) * w, with w = norm_wq (q) or norm_wk (k), bf16
 *     [head_dim] shared by the heads; then pair i = (x[2i], x[2i+1]) of every head of token m
 *     rotated: (x0 c - x1 s, x0 s + x1 c) with c = rope_cos[m, i], s = rope_sin[m, i];
 *   - v is stored as the plain layer stores it; everything is rounded to bf16 once, at the end.
 * The cos / sin tables are inputs, fp32 and pair-major: [head_dim / 2, M], the value for pair
 * i of token m at [i * M + m] (so that 32 consecutive tokens' values of one pair are one
 * 128-byte line); a model's position scheme (one axis, or several as in image transformers)
 * only changes the tables.
 * head_dim == 128; N == 3 * heads * 128; other arguments and errors as svdq_w4a4_nvfp4_linear;
 * norm_wq, norm_wk, rope_cos, rope_sin device pointers, 16-byte aligned; eps >= 0 finite.
 * Asynchronous on `stream`. */
int svdq_w4a4_nvfp4_linear_qkv(const void* act_codes, const void* act_scales, const void* lowrank_act,
                               float act_global_scale, const void* packed_w, float w_global_scale, int M, int N,
                               int K, int rank, int heads, int head_dim, const void* norm_wq, const void* norm_wk,
                               float eps, const void* rope_cos, const void* rope_sin, void* Y, void* stream);

/* Kernels 6 and 7: the MLP up projection with GELU and the down projection's activation pass in
 * its epilogue -- "Nunchaku Lite" docs, section on fused kernels: the original engine runs the
 * MLP with a fused GELU kernel (its benchmark table gives the GELU-MLP fusion 1.06x).  The
 * pages name the fusion only; the reading used is that it computes what the unfused pipeline
 * computes, without the hidden state ever reaching memory:
 *   y = bf16(g_a g_w (Q(X_hat) Q(R)^T) + lowrank_act L2 + b)        (svdq_w4a4_nvfp4_linear)
 *   h = bf16(GELU(y)),  GELU(x) = x Phi(x) (erf form)
 *   out_codes, out_scales, out_lowrank_act = svdq_quantize_act_lowrank_down(h, down_smooth_inv,
 *       down_packed_w, down_act_global_scale)   (the down projection's activation pass on h)
 * The low-rank product U = h_hat L1 of the down projection needs every column of a row; the GEMM
 * keeps it in tensor memory over each CTA pair's consecutive output tiles of a row block and
 * writes one fp32 partial per (pair, row block) to `workspace`; kernel 7 sums them in a fixed
 * order (repeat calls are bit-identical).  Against the unfused pipeline the result can differ
 * only through the fp32 rounding of y before GELU (and of an fp32 GELU, if the unfused pipeline
 * used one); codes and scales are exact for the h this call forms.
 *   act_codes, act_scales, lowrank_act, packed_w, g's: as svdq_w4a4_nvfp4_linear (N = the MLP
 *     width, the down projection's K)
 *   down_smooth_inv   device bf16 [N]; down_packed_w the down projection's packed blob (only its
 *     header and low-rank section, the first 1024 + 4 rank N bytes, are read)
 *   down_act_global_scale  the down projection's static g_a (a power of two)
 *   out_codes   u8 [M, N/2]; out_scales u8 [svdq_act_scale_bytes(M, N)]; out_lowrank_act bf16 [M, 2 rank]
 *   workspace   device scratch of at least svdq_gelu_quant_workspace_bytes(M, N) bytes
 *     (the caller allocates it; contents need no initialisation and are overwritten)
 *   gelu_table  device buffer of svdq_gelu_table_bytes() bytes filled by svdq_gelu_table_fill
 *     (once; read only here): GELU of a bf16 y rounded to bf16 is one lookup, and h is then the
 *     double-precision GELU rounded once -- the unfused pipeline's value except where its fp32
 *     GELU would round the other way at a bf16 midpoint
 *   h_out       device bf16 [M, N] or NULL: if given, also receives h (for inspection)
 * N % 128 == 0, K % 64 == 0, rank == 32; 16-byte aligned pointers.  Asynchronous on `stream`. */
size_t svdq_gelu_quant_workspace_bytes(int M, int N);   /* for the current device; 0 if invalid */
size_t svdq_gelu_table_bytes(void);                      /* 131072: 65536 bf16 entries */
/* Fills `table` (device, 16-byte aligned, svdq_gelu_table_bytes()) with bf16(x Phi(x)) for every
 * bf16 bit pattern x, Phi(x) = erfc(-x / sqrt 2) / 2 in double precision, rounded once to
 * nearest even.  Asynchronous on `stream`. */
int svdq_gelu_table_fill(void* table, void* stream);
int svdq_w4a4_nvfp4_linear_gelu_quant(const void* act_codes, const void* act_scales, const void* lowrank_act,
                                      float act_global_scale, const void* packed_w, float w_global_scale, int M,
                                      int N, int K, int rank, const void* down_smooth_inv, const void* down_packed_w,
                                      float down_act_global_scale, void* out_codes, void* out_scales,
                                      void* out_lowrank_act, void* workspace, size_t workspace_bytes,
                                      const void* gelu_table, void* h_out, void* stream);

/* ------------------------------------------------- SVDQ W4A4, int4 / group 64 */

/* The svdq_w4a4 row with int4 precision and group size 64 ("Nunchaku Lite" docs, "Supported
 * quantization types"; the docs add that nvfp4 is the faster of the two on Blackwell).  The
 * pages give no formula; the reading: symmetric signed 4-bit codes, one bf16 scale per 64 K
 * elements of every row of both operands, s = RNE_bf16(amax / 7) rounded once from the exact
 * quotient, codes RNE(x / s) (within -7..7, the 8-bit scale rounding to nearest), the same
 * smoothing and rank-32 low-rank branch as the nvfp4 row, no per-tensor scale:
 *     y = sum_g s_a[m, g] s_w[n, g] sum_{k in g} c_a[m, k] c_w[n, k] + (X_hat L1) L2 + b.
 * The tensor cores have no 4-bit integer MMA: a code travels as its E4M3 byte (every integer
 * -8..8 is exact in E4M3) and the fp8 MMA (fp32 accumulation) multiplies the integers
 * exactly; each group's sum gets its own accumulator and the epilogue applies s_a s_w.
 *
 * svdq_int4_pack_weights: R, L1, L2, bias, smooth_inv as svdq_pack_weights (N % 128 == 0,
 *   K % 64 == 0, rank 32); blob of svdq_int4_packed_weight_bytes: 1 KB header ("SVDQINT4"),
 *   the low-rank factor section as svdq_pack_weights, codes u8 [N, K] (E4M3 bytes), the scales
 *   widened to fp32 and group-major [K/64, N], L2^T bf16 [N, rank], bias bf16 [N].
 * svdq_int4_quantize_act_lowrank_down: kernel 1's pass with this quantizer -- act_codes u8
 *   [M, K] (E4M3 bytes), act_scales bf16 [K/64, Mp] (group-major, Mp = M rounded up to a
 *   multiple of 128; the rows past M get zero scales), lowrank_act bf16 [M, 2 rank] (U as hi then
 *   lo).  X, smooth_inv, packed_w (its low-rank section) as the nvfp4 call.
 *   Activation scales below 2^-126 (a group amax below 7 * 2^-126) are not supported.
 * svdq_w4a4_int4_linear: Y bf16 [M, N] from those and the packed weights.
 * Errors and asynchrony as the nvfp4 calls. */
size_t svdq_int4_packed_weight_bytes(int N, int K, int rank);
int svdq_int4_pack_weights(const float* R, const uint16_t* L1, const uint16_t* L2, const uint16_t* bias,
                           const uint16_t* smooth_inv, int N, int K, int rank, void* out, size_t out_bytes);
int svdq_int4_quantize_act_lowrank_down(const void* X, const void* smooth_inv, const void* packed_w, int M, int K,
                                        int rank, void* act_codes, void* act_scales, void* lowrank_act, void* stream);
int svdq_w4a4_int4_linear(const void* act_codes, const void* act_scales, const void* lowrank_act, const void* packed_w,
                          int M, int N, int K, int rank, void* Y, void* stream);

/* -------------------------------------------- dynamic per-tensor activation scale */

/* Kernel 5: the variant of the W4A4 layer whose activation scale g_a comes from the batch
 * (max |X smooth_inv| over the whole tensor) instead of from calibration.
 * "Nunchaku Lite" docs, "Supported quantization types" (svdq_w4a4 / nvfp4 / group 16); the
 * per-tensor scale rule: g_a = the smallest power of two with g_a * 6 * 448 >= amax, 1 for
 * amax = 0.
 *
 * svdq_act_amax writes amax = max |X[m,k] smooth_inv[k]| into word 0 of act_amax as the bits
 * of a non-negative float (the products are exact in fp32, so the word is exact).  act_amax is
 * a 16-byte device buffer that the caller zero-fills once, at allocation; each call leaves
 * words 1-3 zero again (there is no clearing pass per call, and graph replays find it clean).
 * X device bf16 [M, K], smooth_inv device bf16 [K]; M >= 0 (M = 0 writes 0), K % 64 == 0;
 * X, smooth_inv and act_amax 16-byte aligned.  Calls sharing one act_amax must be stream-ordered.
 *
 * svdq_quantize_act_lowrank_down_dyn and svdq_w4a4_nvfp4_linear_dyn are the calls of kernels 1
 * and 2 with g_a read from word 0 of act_amax on the device (after the previous kernel of the stream has
 * finished) instead of passed in: the same outputs as the static calls given that g_a, and
 * lowrank_act holds U / g_a of that g_a.  Other arguments and errors as the static calls, with one
 * exception: the static call refuses a product g_a g_w outside [2^-126, 2^126] on the host, and the
 * dynamic call, which forms it on the device, clamps it to that range instead and records
 * SVDQ_ERR_SCALE_RANGE in the device status word (svdq_device_status), so the outputs are finite
 * but wrong for such a batch.  (An infinite amax gives g_a = 2^127.) */
int svdq_act_amax(const void* X, const void* smooth_inv, int M, int K, void* act_amax, void* stream);
int svdq_quantize_act_lowrank_down_dyn(const void* X, const void* smooth_inv, const void* packed_w, int M, int K,
                                       int rank, const void* act_amax, void* act_codes, void* act_scales,
                                       void* lowrank_act, void* stream);
int svdq_w4a4_nvfp4_linear_dyn(const void* act_codes, const void* act_scales, const void* lowrank_act,
                               const void* act_amax, const void* packed_w, float w_global_scale, int M, int N, int K,
                               int rank, void* Y, void* stream);

/* The amax of svdq_act_amax for callers that cannot allocate device memory -- code that runs
 * where cudaMalloc is not allowed or not wanted: inside an inference engine or plugin whose
 * memory is planned up front by the host application, in a real-time path that must not call
 * into the allocator, or under a caching allocator that does not own this library's buffers.
 * The pages describe no such call; it is a convenience of this library with no counterpart
 * there.
 *
 * Writes max |X[m,k] smooth_inv[k]| (the bits of a non-negative float, exact, as svdq_act_amax
 * writes into its word 0) to the 4-byte device word `amax`, which the caller passes like any
 * other output; M = 0 writes 0.  The kernel's scratch (its result, partial maximum and block
 * counter: three 32-bit words, whatever M and K are) lives in a 256-byte array that the
 * library holds on every GPU that loads it, until the process exits; since no M or K needs
 * more than those three words, no size is refused for want of scratch.  The call clears the
 * scratch before its kernel, then copies the result out; it calls no cudaMalloc, cudaFree or
 * other allocating routine.
 *   - The first call on a device looks up the array's device address there (with that device
 *     current) and caches it; make that first call before any stream capture.
 *   - Every call on a device shares the one array: calls whose work overlaps on the GPU (other
 *     streams, or other host threads, without ordering between them) race and give wrong
 *     results.  Order them on one stream.
 * X device bf16 [M, K], smooth_inv device bf16 [K]; M >= 0, K % 64 == 0; X and smooth_inv
 * 16-byte aligned, amax 4-byte aligned.  Errors as svdq_act_amax.  Asynchronous on `stream`. */
int svdq_act_amax_noalloc(const void* X, const void* smooth_inv, int M, int K, void* amax, void* stream);

/* ---------------------------------------------------------------- AWQ W4A16 */

/* y = X ((q - z) s)^T (+ b), weight-only int4 with group 64 along K.  M <= 8 runs the
 * mma.sync kernel (kernel 3), M >= 9 the tcgen05 kernel (kernel 4, 16, 32 or 64 token
 * columns; past 64 tokens one row of CTAs per 64-token tile, each re-reading the weights from
 * L2 -- correct at any M, but the layer is built for the small token counts of the adaptive
 * normalisation).  Both form every product exactly and scale each group's fp32 sum by s
 * once; kernel 4 multiplies (q - z) x, kernel 3 forms s (sum (128 + q) x - (128 + z) sum x),
 * so the two differ only in fp32 rounding.
 *   X        device bf16 [M, K]
 *   qweight  device u8 [N, K/2], element 2i of a row in the low nibble
 *   scales   device bf16 [N, K/64]
 *   zeros    device bf16 [N, K/64], integer zero points 0..15
 *   bias     device bf16 [N] or NULL
 *   Y        device bf16 [M, N] out
 * M >= 0 (M == 0 does nothing), N % 64 == 0, K % 64 == 0 (a K that is not a multiple of 256
 * ends in a partial 256-K stage); X, qweight and Y 16-byte aligned, scales, zeros and bias
 * 2-byte aligned.  With K % 512 == 0, K <= 4096 and scales and zeros 16-byte aligned, both
 * kernels copy each CTA's scale and zero rows into shared memory up front (the faster path;
 * the results are bit-identical to those of the other alignments).  Asynchronous on `stream`. */
int awq_w4a16_linear(const void* X, const void* qweight, const void* scales,
                     const void* zeros, const void* bias, int M, int N, int K,
                     void* Y, void* stream);

/* ----------------------------------------------------------------- helpers */

/* Host: convert a swizzled scale buffer (rows rounded up to 128) into plain
 * row-major [rows, K/16] E4M3 codes, and back. */
int svdq_unswizzle_scales(const void* swizzled, int rows, int K, uint8_t* out);
int svdq_swizzle_scales(const uint8_t* plain, int rows, int K, void* swizzled);

/* Diagnostic of the failure path (the pages have no counterpart): launches one warp that waits,
 * through the same bounded wait as every kernel, for an mbarrier phase at which nothing
 * arrives.  The wait gives up after its limit (about one second), records SVDQ_ERR_TIMEOUT in
 * the device status word and the kernel returns; no copy or tensor-core operation is in
 * flight, so the context stays usable.  Returns the launch status; read the outcome with
 * svdq_device_status.  Asynchronous on `stream`. */
int svdq_selftest_wait_timeout(void* stream);

/* Reads (and with clear != 0, resets) the device-side status word of the
 * current device that kernels set when a bounded wait runs out or a dynamic
 * scale product is out of range.  Returns SVDQ_OK, SVDQ_ERR_TIMEOUT (which
 * wins when both happened) or SVDQ_ERR_SCALE_RANGE; SVDQ_ERR_CUDA if the read
 * itself failed.
 * This call synchronizes the device; it is meant for tests and diagnostics. */
int svdq_device_status(int clear);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* SVDQ_H_ */
