// Kernel 2: NVFP4 block-scaled GEMM on tcgen05 with the SVDQuant epilogue.
//
//   Y = bf16( alpha * (Q(X_hat) Q(R)^T) + U L2 + b ),  alpha = g_a g_w
//
// Method: "Nunchaku Lite" docs, "Supported quantization types" (svdq_w4a4,
// nvfp4, group 16: an NVFP4 runtime kernel with an SVDQ low-rank correction);
// the Nunchaku Lite article: the low-rank branch is 16-bit.
//
// Design (sm_100a).  Persistent kernel over 256 x BN output tiles, each computed
// by a pair of CTAs (a 2-CTA cluster) with the pair-wide tensor-core MMA
// (tcgen05 cta_group::2, M = 256): CTA r holds A rows [128 r, 128 r + 128) and B
// rows [BN/2 r, BN/2 r + BN/2) of the tile, so each SM stages half of B and the
// pair reads every operand byte from L2 once.  320 threads per CTA:
//   warp 0  TMA producer (both CTAs): code tiles of A and B (128-byte swizzle,
//           256 K per stage), their E4M3 scale atoms, and, as one extra stage per
//           tile, the low-rank tiles (bf16 [U/g_a hi | lo] in the A slot, (L2/g_w)^T
//           in the B slot).  Completion of both CTAs' copies is counted on the
//           leader's full barrier of the stage's issue group (two stages, or the
//           tile's odd one).
//   warp 1  tensor memory (both CTAs, pair allocation); in the leader one thread
//           issues the scale copies (tcgen05.cp, shared -> tensor memory in both
//           CTAs), the block-scaled MMAs (kind::mxf4nvf4, block16, K = 64) into a
//           double-buffered fp32 accumulator, and the four bf16 low-rank MMAs
//           (K = 16); commits release the stage in both CTAs and publish the
//           accumulator to both epilogues.  One barrier wait covers a group of two
//           stages: a wait costs the issuing thread about as much as a quarter of a
//           stage's tensor work, and the issuing thread is the mainloop's limit.
//   warps 2-9  epilogue (both CTAs): two warps per tensor-memory lane quarter (32
//           accumulator rows), each taking every other 32-column chunk; tcgen05.ld in a
//           three-register-set rotation, y = alpha acc + b (one fma, bias staged in
//           shared memory), bf16 into a 64-byte-swizzled 32 x 32 staging tile, one TMA
//           tensor store per chunk.  The accumulator buffer is handed back as soon as the
//           columns the next tile will overwrite are in registers.
// Every mbarrier wait is bounded (about one second); a wait that runs out records
// SVDQ_ERR_TIMEOUT in the device status word, the other roles give up, the MMAs in
// flight are drained (bounded), tensor memory is freed and the kernel returns.
#pragma once

#include "act_amax.cuh"
#include "ptx.cuh"

namespace svdq {
namespace k2 {

constexpr int BM = 128;                    // A rows per CTA (256 per pair)
constexpr int BK = 256;                    // K elements per pipeline stage
constexpr int kEpiWarps = 8;                // two per tensor-memory lane quarter
constexpr int kThreads = (2 + kEpiWarps) * 32;

template <int BN, bool QKV = false>
struct Cfg {
  static_assert(BN == 128 || BN == 192 || BN == 256, "tile width");
  static_assert(!QKV || BN != 192, "the QKV epilogue's tiles hold whole 128-column heads");
  static constexpr int BN_HALF = BN / 2;                       // B rows staged by each CTA
  static constexpr int SFB_ATOMS = BN == 128 ? 1 : 2;          // 128-row scale blocks spanned by a tile
  static constexpr int A_BYTES = BM * BK / 2;
  static constexpr int B_BYTES = BN_HALF * BK / 2;
  static constexpr int SFA_BYTES = (BK / 64) * 512;
  static constexpr int SFB_BYTES = SFB_ATOMS * (BK / 64) * 512;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
  static constexpr int UCAT_BYTES = BM * 64 * 2;               // low-rank A tile (fits the A slot)
  static constexpr int L2_BYTES = BN_HALF * 32 * 2;            // low-rank B tile (fits the B slot)
  static constexpr int STAGES = BN == 128 ? 7 : (BN == 192 ? 6 : 5);
  // scale factors of one stage in tensor memory: A 4 columns per MMA, B 4 per 128 rows per MMA;
  // two such regions alternate between consecutive stages
  static constexpr int SF_COLS = 4 * (BK / 64) + 4 * SFB_ATOMS * (BK / 64);
  // Two accumulator buffers.  When two full buffers and the scale regions do not fit in
  // the 512 columns (BN = 256), the second buffer overlaps the end of the first; the
  // epilogue reads the shared columns first and releases the accumulator as soon as
  // they are in registers (one barrier stage instead of two).
  static constexpr bool OVERLAP = 2 * BN + 2 * SF_COLS > 512;
  static constexpr int ACC1 = OVERLAP ? 512 - 2 * SF_COLS - BN : BN;   // first column of buffer 1
  static constexpr int NCH = BN / 32;                                  // 32-column epilogue chunks
  static constexpr int OV_CHUNKS = OVERLAP ? (BN - ACC1 + 31) / 32 : 0;
  static constexpr int ACC_STAGES = OVERLAP ? 1 : 2;                   // accumulator barrier stages
  static constexpr uint32_t TM_SF = ACC1 + BN;
  static constexpr uint32_t SFB_OFF = 4 * (BK / 64);            // B's columns after A's within a region
  static constexpr int TMEM_COLS = 512;
  static constexpr int OFF_BAR = STAGES * STAGE_BYTES;
  // One full barrier per MMA-issue group (two stages, or one at a tile's end): the issuing
  // thread waits once per group.  The producer reuses a slot only after the MMAs of the stage
  // STAGES back have completed, and those STAGES + 1 stages span at most STAGES + 1 groups, so
  // with NBF > STAGES no barrier is posted for a group while an earlier group still owns it.
  static constexpr int NBF = 8;
  static constexpr int NUM_BARS = NBF + STAGES + 5;            // full[NBF], empty, acc_full[2], acc_empty[2], drain
  static constexpr int OFF_MISC = OFF_BAR + 8 * NUM_BARS;
  static constexpr int OFF_BIAS = (OFF_MISC + 64 + 127) / 128 * 128;  // per epilogue warp: the tile's bias (BN bf16)
  static constexpr int OFF_NW = OFF_BIAS + kEpiWarps * 512;    // QKV epilogue, per epilogue warp: q and k norm weights
  static constexpr int NW_BYTES = QKV ? kEpiWarps * 512 : 0;
  static constexpr int OFF_STAGE = (OFF_NW + NW_BYTES + 1023) / 1024 * 1024;  // per epilogue warp: 32 x 32 bf16
  static constexpr int SMEM_BYTES = OFF_STAGE + kEpiWarps * 2048 + 1024;  // + slack to align the base to 1024
  static constexpr uint32_t TX_MAIN = 2u * STAGE_BYTES;        // bytes landing per stage, both CTAs
  static constexpr uint32_t TX_LOWRANK = 2u * (UCAT_BYTES + L2_BYTES);
  static_assert(TM_SF + 2 * SF_COLS <= TMEM_COLS, "tensor memory overflow");
  static_assert(NBF > STAGES, "a full barrier is reused only after its group was consumed");
  static_assert(!OVERLAP || (ACC1 % 32 == 0 && ACC1 > 0), "overlap is a whole number of epilogue chunks");
  static_assert(STAGE_BYTES % 1024 == 0 && B_BYTES % 1024 == 0, "1 KB alignment of swizzled tiles");
  static_assert(UCAT_BYTES <= A_BYTES && L2_BYTES <= B_BYTES, "low-rank tiles fit the stage slots");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
  static_assert(OFF_BIAS % 16 == 0, "16-byte shared stores of the bias");
  static_assert(OFF_STAGE % 1024 == 0, "64-byte-swizzled store staging needs 512-byte alignment");
  static_assert(!OVERLAP || (NCH == 8 && OV_CHUNKS == 3), "chunk order of the overlapping buffers");
};

struct Params {
  const __nv_bfloat16* bias;       // [N]
  __nv_bfloat16* Y;                // [M, N]
  int M, N, K;
  int tiles_n;                     // N / BN
  int tiles;                       // ceil(M / 256) * tiles_n
  float alpha;                     // g_a g_w
  const unsigned int* amax;        // or, if not null, g_a from this amax word (kernel 5) ...
  float w_scale;                   // ... times g_w
  // QKV epilogue (the kQkv instantiation): q, k, v thirds of `third` columns each (heads x 128);
  // q and k RMS-normalised per 128-column head and rotated by RoPE
  const __nv_bfloat16* norm_wq;    // [128]
  const __nv_bfloat16* norm_wk;    // [128]
  const float* rope_cos;           // [64, M]: cos of the angle of pair i (dims 2i, 2i + 1) of token m at [i][m]
  const float* rope_sin;           // [64, M]
  float eps;
  int third;
};

// Instruction descriptors (tcgen05 "instruction descriptor" bit fields).
// Block-scaled: bits 7-9 A type (1 = E2M1), 10-12 B type (1 = E2M1), 15/16 A/B
// major (0 = K), 17-22 N >> 3, 23 scale type (0 = UE4M3), 24-28 M >> 4.
template <int BN>
__device__ __forceinline__ uint32_t idesc_nvfp4_m256() {
  return (1u << 7) | (1u << 10) | (static_cast<uint32_t>(BN >> 3) << 17) | (static_cast<uint32_t>(256 >> 4) << 24);
}
// kind::f16: bits 4-5 D type (1 = f32), 7-9 A type (1 = bf16), 10-12 B type (1 = bf16).
template <int BN>
__device__ __forceinline__ uint32_t idesc_bf16_m256() {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(BN >> 3) << 17) |
         (static_cast<uint32_t>(256 >> 4) << 24);
}

// y = bf16(alpha acc + b) for 32 consecutive columns of one row: fp32 accumulators in r,
// their bias (32 bf16) at bias (shared memory).  The 64 result bytes are this lane's row
// of a 32 x 32 staging tile in the 64-byte swizzle of the store's tensor map (16-byte
// unit u of row r at r * 64 + 16 (u ^ ((r >> 1) & 3))).
__device__ __forceinline__ void epilogue_stage32(const uint32_t (&r)[32], const uint4* bias, float alpha,
                                                 uint32_t row_smem, uint32_t sw) {
  uint32_t o[16];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 bv = bias[q];
    const uint32_t bw[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const int j = q * 8 + w * 2;
      const float lo = fmaf(alpha, __uint_as_float(r[j]), bf16lo_to_f32(bw[w]));
      const float hi = fmaf(alpha, __uint_as_float(r[j + 1]), bf16hi_to_f32(bw[w]));
      o[q * 4 + w] = pack_bf16x2(lo, hi);
    }
  }
#pragma unroll
  for (int q = 0; q < 4; ++q)
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                 ::"r"(row_smem + ((static_cast<uint32_t>(q) ^ sw) << 4)), "r"(o[q * 4]), "r"(o[q * 4 + 1]),
                   "r"(o[q * 4 + 2]), "r"(o[q * 4 + 3])
                 : "memory");
}

template <int BN, bool kQkv = false>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
nvfp4_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                  const __grid_constant__ CUtensorMap tmSFA, const __grid_constant__ CUtensorMap tmSFB,
                  const __grid_constant__ CUtensorMap tmU, const __grid_constant__ CUtensorMap tmL2,
                  const __grid_constant__ CUtensorMap tmY, const Params p) {
  using C = Cfg<BN, kQkv>;
  constexpr int S = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);

  const uint32_t bars = base + C::OFF_BAR;
  constexpr int NBF = C::NBF;
  auto full = [&](uint32_t it) { return bars + 8u * (it % NBF); };   // group `it` of the MMA issue order
  auto empty = [&](int s) { return bars + 8u * (NBF + s); };
  auto acc_full = [&](int b) { return bars + 8u * (NBF + S + b); };
  auto acc_empty = [&](int b) { return bars + 8u * (NBF + S + 2 + b); };
  const uint32_t drain = bars + 8u * (NBF + S + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + C::OFF_MISC + 4);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const uint32_t cta = cluster_ctarank();          // 0: leader of the pair, 1: follower
  const bool leader = cta == 0;
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;
  const int natoms = p.K / 64;                     // 64-K scale atoms per 128-row block
  const int nkb = (p.K + BK - 1) / BK;

  if (warp == 0 && lane == 0) {
    for (int i = 0; i < NBF; ++i) mbar_init(full(i), 2);    // the leader's two arrivals per group
    for (int s = 0; s < S; ++s) mbar_init(empty(s), 1);
    for (int b = 0; b < 2; ++b) { mbar_init(acc_full(b), 1); mbar_init(acc_empty(b), 2 * kEpiWarps); }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmA); prefetch_tmap(&tmB); prefetch_tmap(&tmSFA);
    prefetch_tmap(&tmSFB); prefetch_tmap(&tmU); prefetch_tmap(&tmL2); prefetch_tmap(&tmY);
  }
  if (warp == 1) tmem_alloc_pair<C::TMEM_COLS>(smem_addr(tmem_slot));
  tc_fence_before();
  cluster_sync_all();                              // barriers of both CTAs initialised and visible
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // The weights do not depend on the previous kernel: the first tile's first stages of B and
  // its scales are loaded before waiting for it (their stages are free at the start; the
  // full barrier of each stage's issue group gets the whole stage's byte count here, A and
  // its scales follow after the wait).  A stage's issue group is kb / 2 for the first tile.
  const int npre = pair < p.tiles ? min(S, nkb) : 0;
  if (warp == 0) {
    if (elect_one()) {
      const int nt0 = pair % p.tiles_n;
      const int bn0 = nt0 * BN + static_cast<int>(cta) * C::BN_HALF, nb0 = nt0 * BN / 128;
      for (int kb = 0; kb < npre; ++kb) {
        const uint32_t sb = base + kb * C::STAGE_BYTES;
        const uint32_t fbar = full(static_cast<uint32_t>(kb / 2));
        const uint32_t fb = map_to_cta(fbar, 0);
        if (leader) mbar_arrive_expect_tx(fbar, C::TX_MAIN);
        tma_load_2d_pair(sb + C::A_BYTES, &tmB, kb * (BK / 2), bn0, fb);
#pragma unroll
        for (int a = 0; a < C::SFB_ATOMS; ++a)
          tma_load_2d_pair(sb + C::A_BYTES + C::B_BYTES + C::SFA_BYTES + a * (BK / 64) * 512, &tmSFB, 0,
                           (nb0 + a) * natoms + kb * (BK / 64), fb);
        if (leader && kb + 1 == nkb && (nkb & 1)) mbar_arrive(fbar);   // a one-stage group's second arrival
      }
    }
    __syncwarp();
  }
  // everything above overlaps the previous kernel of the stream; its outputs (this
  // kernel's inputs) and its reads of Y are complete past this point
  grid_dependency_wait();
  grid_launch_dependents();

  if (warp == 0) {
    {
      // ------------------------------------------------------------------ producer (whole warp, one lane issues)
      uint32_t g = 0, it = 0;                      // stage and issue-group counters
      bool ok = true;
      for (int t = pair; ok && t < p.tiles; t += npairs) {
        const int mt = t / p.tiles_n, nt = t % p.tiles_n;
        const int m0 = mt * 256 + static_cast<int>(cta) * BM;      // this CTA's A rows
        const int n0 = nt * BN;
        const int bn0 = n0 + static_cast<int>(cta) * C::BN_HALF;   // this CTA's B rows
        const int rb = m0 / 128, nb = n0 / 128;
        for (int kb0 = 0; ok && kb0 <= nkb; ++it) {                 // kb == nkb: the low-rank stage
          const int cnt = kb0 + 1 < nkb ? 2 : 1;                    // the MMA warp's grouping
          const uint32_t fbar = full(it);
          const uint32_t fb = map_to_cta(fbar, 0);
          for (int c = 0; c < cnt; ++c) {
            const int kb = kb0 + c;
            const int s = g % S;
            const uint32_t ph = (g / S) & 1u;
            if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(empty(s), ph ^ 1u, abort_flag, 1))) { ok = false; break; }
            const uint32_t sb = base + s * C::STAGE_BYTES;
            const bool pre = t == pair && kb < npre;  // B, its scales and the byte count went out already
            if (elect_one()) {
              if (pre) {
                tma_load_2d_pair(sb, &tmA, kb * (BK / 2), m0, fb);
                tma_load_2d_pair(sb + C::A_BYTES + C::B_BYTES, &tmSFA, 0, rb * natoms + kb * (BK / 64), fb);
              } else if (kb < nkb) {
                if (leader) mbar_arrive_expect_tx(fbar, C::TX_MAIN);
                tma_load_2d_pair(sb, &tmA, kb * (BK / 2), m0, fb);
                tma_load_2d_pair(sb + C::A_BYTES, &tmB, kb * (BK / 2), bn0, fb);
                tma_load_2d_pair(sb + C::A_BYTES + C::B_BYTES, &tmSFA, 0, rb * natoms + kb * (BK / 64), fb);
#pragma unroll
                for (int a = 0; a < C::SFB_ATOMS; ++a)
                  tma_load_2d_pair(sb + C::A_BYTES + C::B_BYTES + C::SFA_BYTES + a * (BK / 64) * 512, &tmSFB, 0,
                                   (nb + a) * natoms + kb * (BK / 64), fb);
              } else {
                if (leader) mbar_arrive_expect_tx(fbar, C::TX_LOWRANK);
                tma_load_2d_pair(sb, &tmU, 0, m0, fb);
                tma_load_2d_pair(sb + C::A_BYTES, &tmL2, 0, bn0, fb);
              }
              if (cnt == 1 && leader && !pre) mbar_arrive(fbar);  // a one-stage group's second arrival
            }
            __syncwarp();
            ++g;
          }
          kb0 += cnt;
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (leader) {
      // ------------------------------------------------------------------ MMA issuer (pair leader; whole warp, one lane issues)
      const uint32_t id4 = idesc_nvfp4_m256<BN>();
      const uint32_t idb = idesc_bf16_m256<BN>();
      // descriptor high words (stride, version, layout) never change; the low word is the
      // start address >> 4 with the leading-byte-offset field set to 1 (16 B) for swizzled tiles
      constexpr uint32_t kHiSw128 = smem_desc_hi(1024, 2);      // K-major, 128-byte swizzle
      constexpr uint32_t kHiSw64 = smem_desc_hi(512, 4);        // K-major, 64-byte swizzle
      constexpr uint32_t kHiSf = smem_desc_hi(128, 0);          // scale atoms: 8 rows x 16 B groups
      constexpr uint32_t kLbo = 1u << 16;
      uint32_t g = 0, it = 0;                      // stage and issue-group counters
      int i = 0;
      bool ok = true;
      for (int t = pair; ok && t < p.tiles; t += npairs, ++i) {
        const int nt = t % p.tiles_n;
        const int b = i & 1;                       // accumulator buffer
        const int ab = C::ACC_STAGES == 2 ? b : 0; // its barrier stage
        const int use = C::ACC_STAGES == 2 ? (i >> 1) : i;
        if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(acc_empty(ab), (use & 1) ^ 1, abort_flag, 2))) break;
        tc_fence_after();
        const uint32_t dacc = tmem + static_cast<uint32_t>(b * C::ACC1);
        const uint32_t sfb_shift = static_cast<uint32_t>(((nt * BN) % 128) / 32);
        // two 256-K stages per group (one barrier wait, one elect), the tile's odd stage alone
        for (int kb = 0; kb <= nkb; ++it) {
          const int cnt = kb + 1 < nkb ? 2 : 1;
          if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(full(it), (it / NBF) & 1u, abort_flag, 3))) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (elect_one()) {
            for (int c = 0; c < cnt; ++c) {
              const uint32_t gg = g + c;
              const int kbb = kb + c;
              const int s = gg % S;
              const uint32_t sb = base + s * C::STAGE_BYTES;
              const uint32_t a_lo = (sb >> 4) | kLbo;
              const uint32_t b_lo = ((sb + C::A_BYTES) >> 4) | kLbo;
              if (kbb < nkb) {
                const int na = min(BK / 64, natoms - kbb * (BK / 64));
                const uint32_t sfa_lo = (sb + C::A_BYTES + C::B_BYTES) >> 4;
                const uint32_t sfb_lo = sfa_lo + C::SFA_BYTES / 16;
                const uint32_t tsf = tmem + C::TM_SF + (gg & 1u) * C::SF_COLS;
                // per 64-K atom its scale copies, then its MMA: a copy waits only for the MMAs
                // issued before it, so the next atom's copies can run while this atom's MMA does
#pragma unroll
                for (int kk = 0; kk < BK / 64; ++kk) {
                  if (kk < na) {
                    tc_copy_32x128b_x4_pair(tsf + 4 * kk, make_desc(sfa_lo + kk * 32, kHiSf));
#pragma unroll
                    for (int a = 0; a < C::SFB_ATOMS; ++a)
                      tc_copy_32x128b_x4_pair(tsf + C::SFB_OFF + (kk * C::SFB_ATOMS + a) * 4,
                                              make_desc(sfb_lo + (a * (BK / 64) + kk) * 32, kHiSf));
                    umma_nvfp4_pair(dacc, make_desc(a_lo + kk * 2, kHiSw128), make_desc(b_lo + kk * 2, kHiSw128),
                                    id4, tsf + 4 * kk, tsf + C::SFB_OFF + kk * C::SFB_ATOMS * 4 + sfb_shift,
                                    (kbb | kk) != 0 ? 1u : 0u);
                  }
                }
              } else {
                // A: [U hi | U lo] / g_a (128-byte swizzle); B: (L2 / g_w)^T (64-byte swizzle),
                // K steps 0, 16, 0, 16; one K step = 16 bf16 = 32 B
                const uint32_t l_lo = ((sb + C::A_BYTES) >> 4) | kLbo;
#pragma unroll
                for (int j = 0; j < 4; ++j)
                  umma_bf16_pair(dacc, make_desc(a_lo + j * 2, kHiSw128), make_desc(l_lo + (j & 1) * 2, kHiSw64),
                                 idb, 1u);
              }
              tc_commit_pair(empty(s), 0x3);
            }
            if (kb + cnt - 1 == nkb) tc_commit_pair(acc_full(ab), 0x3);
          }
          __syncwarp();
          g += cnt;
          kb += cnt;
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ epilogue (both CTAs)
    const int quarter = warp & 3;                  // tensor-memory lanes 32*quarter .. +31
    const int ew = warp - 2;
    float alpha = p.alpha;
    if (p.amax) {
      // the host checks g_a g_w for the static call; here it is formed on the device, so a
      // product outside [2^-126, 2^126] is clamped and reported instead of refused
      alpha = act_scale_from_amax(__uint_as_float(*p.amax)) * p.w_scale;
      if (!(alpha >= 0x1p-126f && alpha <= 0x1p126f)) {
        if (pair == 0 && threadIdx.x == 64) atomicOr(&g_device_status, 2u);
        alpha = fminf(fmaxf(alpha, 0x1p-126f), 0x1p126f);
      }
    }
    const int eh = ew >> 2;                        // this warp takes every other chunk, starting at eh
    constexpr int NCW = C::NCH / 2;                // chunks per warp per tile
    uint8_t* sbias = gbase + C::OFF_BIAS + ew * 512;
    const uint32_t stage_tile = base + C::OFF_STAGE + ew * 2048;
    const uint32_t stage_row = stage_tile + lane * 64;                      // this lane's staging row
    const uint32_t sw = (static_cast<uint32_t>(lane) >> 1) & 3u;
    int i = 0;
    if constexpr (kQkv) {
      // ---------------------------------------------------------------- QKV epilogue
      // A warp owns one 128-column head of its 32 rows (BN = 256: the tile's head eh; BN = 128:
      // the tile's one head, taken by the eh = 0 warps while their partners only hand the
      // accumulator back), so RMSNorm's sum of squares and RoPE's pairs stay in one thread.
      // Two passes over the head's four 32-column chunks of tensor memory: the sum of squares,
      // then one chunk at a time (norm weight, rotation, bf16 into the warp's staging tile, one
      // TMA store) with the next chunk's cos / sin loads in flight -- 32 accumulator registers
      // live instead of 128.  The tables are pair-major, so a warp's load of one pair covers
      // its 32 consecutive tokens in one 128-byte line.
      uint8_t* snw = gbase + C::OFF_NW + ew * 512;                          // q weights, then k weights
      {
        const __nv_bfloat16* src = lane < 16 ? p.norm_wq : p.norm_wk;
        *reinterpret_cast<uint4*>(snw + lane * 16) = __ldg(reinterpret_cast<const uint4*>(src) + (lane & 15));
        __syncwarp();
      }
      const bool active = BN == 256 || eh == 0;
      const int hcol = BN == 256 ? eh * 128 : 0;                            // the head's first tile column
      for (int t = pair; t < p.tiles; t += npairs, ++i) {
        const int mt = t / p.tiles_n, nt = t % p.tiles_n;
        const int m0 = mt * 256 + static_cast<int>(cta) * BM + quarter * 32;
        const int n0 = nt * BN;
        const int b = i & 1;
        const int ab = C::ACC_STAGES == 2 ? b : 0;
        const int use = C::ACC_STAGES == 2 ? (i >> 1) : i;
        const int part = (n0 + hcol) / p.third;    // 0 q, 1 k, 2 v (a tile never straddles two)
        const bool live = active && m0 < p.M;      // warp-uniform
        const int m = min(m0 + lane, p.M - 1);
        // Order of the head's four chunks in the second pass, and the point of release.  With
        // overlapping buffers (BN = 256) the next tile overwrites buffer 0's columns ACC1..255
        // (head 1's chunks 1-3) or buffer 1's first 256 - ACC1 columns (head 0's chunks 0-2):
        // the warp holding them reads those first and hands the accumulator back once they
        // are in registers; the other warp hands it back after the first pass.  With two
        // separate buffers (BN = 128) the accumulator is handed back after the last read.
        const bool shared = BN == 256 && ((b == 0 && eh == 1) || (b == 1 && eh == 0));
        const int first = (BN == 256 && b == 0 && eh == 1) ? 1 : 0;
        auto chunk_of = [&](int jj) { return (first + jj) & 3; };
        const int rel_after = BN == 256 ? (shared ? 2 : -1) : 3;   // pass-2 position after whose read to release
        if (lane < BN / 8)
          *reinterpret_cast<uint4*>(sbias + lane * 16) = __ldg(reinterpret_cast<const uint4*>(p.bias + n0) + lane);
        __syncwarp();
        // the rotation tables of the first chunk do not depend on the accumulator
        float tc[16], ts[16];
        const float* ccol = p.rope_cos + m;        // pair i of token m at [i * M + m]
        const float* scol = p.rope_sin + m;
        auto load_tables = [&](int j, float (&c)[16], float (&sn)[16]) {
#pragma unroll
          for (int x = 0; x < 16; ++x) {
            c[x] = __ldg(ccol + static_cast<size_t>(16 * j + x) * p.M);
            sn[x] = __ldg(scol + static_cast<size_t>(16 * j + x) * p.M);
          }
        };
        if (live && part < 2) load_tables(chunk_of(0), tc, ts);
        if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(acc_full(ab), use & 1, abort_flag, 4))) break;
        tc_fence_after();
        const uint32_t trow = tmem + (static_cast<uint32_t>(quarter * 32) << 16) +
                              static_cast<uint32_t>(b * C::ACC1 + hcol);
        auto release = [&]() {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_remote(map_to_cta(acc_empty(ab), 0));
        };
        if (!live) {
          release();
          continue;
        }
        const uint4* bh = reinterpret_cast<const uint4*>(sbias + hcol * 2);
        // y = alpha acc + b for 32 columns (chunk j of the head), in place
        auto affine = [&](uint32_t (&r)[32], int j) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint4 bv = bh[j * 4 + q];
            const uint32_t bw[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
            for (int w = 0; w < 4; ++w) {
              const int k = q * 8 + w * 2;
              r[k] = __float_as_uint(fmaf(alpha, __uint_as_float(r[k]), bf16lo_to_f32(bw[w])));
              r[k + 1] = __float_as_uint(fmaf(alpha, __uint_as_float(r[k + 1]), bf16hi_to_f32(bw[w])));
            }
          }
        };
        // first pass (q and k): the head's sum of squares, two chunks at a time
        float rinv = 1.f;
        if (part < 2) {
          float ss = 0.f;
#pragma unroll
          for (int j = 0; j < 4; j += 2) {
            uint32_t A[32], B[32];
            tmem_ld_32x32b_x32(trow + 32u * j, A);
            tmem_ld_32x32b_x32(trow + 32u * (j + 1), B);
            tmem_wait_ld_regs(A);
            tmem_wait_ld_regs(B);
            affine(A, j);
            affine(B, j + 1);
#pragma unroll
            for (int k = 0; k < 32; ++k) {
              ss = fmaf(__uint_as_float(A[k]), __uint_as_float(A[k]), ss);
              ss = fmaf(__uint_as_float(B[k]), __uint_as_float(B[k]), ss);
            }
          }
          rinv = rsqrtf(ss * (1.0f / 128.0f) + p.eps);
        }
        if (rel_after < 0) release();
        const uint32_t* wn = reinterpret_cast<const uint32_t*>(snw + (part == 1 ? 256 : 0));
        // second pass: one chunk at a time, the next chunk's tables in flight meanwhile
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const int j = chunk_of(jj);
          uint32_t r[32];
          tmem_ld_32x32b_x32(trow + 32u * j, r);
          float nc[16], ns[16];
          if (part < 2 && jj + 1 < 4) load_tables(chunk_of(jj + 1), nc, ns);
          tmem_wait_ld_regs(r);
          if (jj == rel_after) release();
          affine(r, j);
          if (part < 2) {
            // RMSNorm weight, then the rotation of pairs 16 j .. 16 j + 15
#pragma unroll
            for (int pr = 0; pr < 16; ++pr) {
              const uint32_t ww = wn[16 * j + pr];                            // weights of dims 2 pr, 2 pr + 1
              const float x0 = __uint_as_float(r[2 * pr]) * rinv * bf16lo_to_f32(ww);
              const float x1 = __uint_as_float(r[2 * pr + 1]) * rinv * bf16hi_to_f32(ww);
              r[2 * pr] = __float_as_uint(fmaf(x0, tc[pr], -x1 * ts[pr]));
              r[2 * pr + 1] = __float_as_uint(fmaf(x0, ts[pr], x1 * tc[pr]));
            }
#pragma unroll
            for (int x = 0; x < 16; ++x) {
              tc[x] = nc[x];
              ts[x] = ns[x];
            }
          }
          // bf16 into the staging tile (once the previous store from it has read it), one TMA store
          if (lane == 0) bulk_wait_group_read<0>();
          __syncwarp();
          {
            uint32_t o[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) o[k] = pack_bf16x2(__uint_as_float(r[2 * k]), __uint_as_float(r[2 * k + 1]));
#pragma unroll
            for (int q = 0; q < 4; ++q)
              asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                           ::"r"(stage_row + ((static_cast<uint32_t>(q) ^ sw) << 4)), "r"(o[q * 4]), "r"(o[q * 4 + 1]),
                             "r"(o[q * 4 + 2]), "r"(o[q * 4 + 3])
                           : "memory");
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tmY, stage_tile, n0 + hcol + 32 * j, m0);
            bulk_commit_group();
          }
        }
      }
    } else
    for (int t = pair; t < p.tiles; t += npairs, ++i) {
      const int mt = t / p.tiles_n, nt = t % p.tiles_n;
      const int m0 = mt * 256 + static_cast<int>(cta) * BM + quarter * 32;   // this warp's first row
      const int n0 = nt * BN;
      const int b = i & 1;
      const int ab = C::ACC_STAGES == 2 ? b : 0;
      const int use = C::ACC_STAGES == 2 ? (i >> 1) : i;
      // the tile's bias goes to this warp's shared-memory slot while the mainloop runs
      if (lane < BN / 8)
        *reinterpret_cast<uint4*>(sbias + lane * 16) = __ldg(reinterpret_cast<const uint4*>(p.bias + n0) + lane);
      __syncwarp();
      if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(acc_full(ab), use & 1, abort_flag, 4))) break;
      tc_fence_after();
      const uint32_t trow = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(b * C::ACC1);
      const bool live = m0 < p.M;                  // warp-uniform: rows past M are clipped by the store
      // Processing order of the tile's 32-column chunks.  With overlapping buffers the
      // columns shared with the other buffer come first (chunks 5-7 of buffer 0, 0-2 of
      // buffer 1) and each warp releases the accumulator once its share of them is in
      // registers; otherwise after its last chunk.  This warp takes positions eh, eh + 2, ...
      const bool swap = C::OVERLAP && b == 0;
      auto chunk = [&](int jj) {
        const int j = 2 * jj + eh;
        if (!swap) return j;
        return j < 2 ? 6 + j : (j < 4 ? 7 - j : j - 4);        // 6 7 5 4 0 1 2 3
      };
      constexpr int kRelease = C::OVERLAP ? C::OV_CHUNKS : C::NCH;
      const int nrel = (kRelease - eh + 1) / 2;    // this warp's chunks among the first kRelease
      const int jrel = 3 * ((nrel - 1) / 3);       // the wait that covers the last of them
      auto release = [&]() {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(map_to_cta(acc_empty(ab), 0));
      };
      // converts one chunk into the staging tile and stores it with one TMA store (the
      // previous store from the tile must have finished reading it)
      auto emit = [&](const uint32_t (&r)[32], int jj) {
        const int c = chunk(jj);
        if (lane == 0) bulk_wait_group_read<0>();
        __syncwarp();
        epilogue_stage32(r, reinterpret_cast<const uint4*>(sbias + c * 64), alpha, stage_row, sw);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&tmY, stage_tile, n0 + c * 32, m0);
          bulk_commit_group();
        }
      };
      // Three register sets in rotation: this warp's first three chunks are loaded up front;
      // every third chunk one wait covers the three loads issued while the previous three
      // were converted.
      uint32_t R[3][32];
#pragma unroll
      for (int jj = 0; jj < 3 && jj < NCW; ++jj) tmem_ld_32x32b_x32(trow + chunk(jj) * 32, R[jj]);
#pragma unroll
      for (int jj = 0; jj < NCW; ++jj) {
        if (jj % 3 == 0) {
#pragma unroll
          for (int k = 0; k < 3 && jj + k < NCW; ++k) tmem_wait_ld_regs(R[k]);
          if (jj == jrel) release();
        }
        if (live) emit(R[jj % 3], jj);
        if (jj + 3 < NCW) tmem_ld_32x32b_x32(trow + chunk(jj + 3) * 32, R[jj % 3]);
      }
    }
    if (lane == 0) bulk_wait_group<0>();           // stores complete before shared memory goes away
    __syncwarp();
  }

  __syncthreads();
  if (*abort_flag) {
    // a wait ran out: let the MMAs and copies already issued finish before the memory goes away
    if (warp == 1 && leader) {
      if (elect_one()) tc_commit_pair(drain, 0x1);
      __syncwarp();
      mbar_wait_bounded(drain, 0, nullptr, 6);
    }
    if (warp == 0 && lane == 0) {
      const uint64_t t0 = global_timer_ns();
      while (global_timer_ns() - t0 < 2000000ull) { }
    }
    __syncthreads();
  }
  tc_fence_before();
  cluster_sync_all();                              // the peer is done with this CTA's tensor memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair<C::TMEM_COLS>(tmem);
  }
}

}  // namespace k2
}  // namespace svdq
