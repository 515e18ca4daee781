// Byte layouts shared by the host packer and the CUDA launchers.
//
// Packed weight blob (device-private; produced on the host by svdq_pack_weights):
//   [0, 1024)    header: "SVDQNVF4", abi version, N, K, rank, g_w (zero padded)
//   l1s          bf16 [2][rank][K] (diag(smooth_inv) L1)^T split exactly into a
//                                 high and a low bf16 part (K contiguous) -- read
//                                 by the activation kernel, which knows K but not
//                                 N, so it comes first
//   codes        u8   [N][K/2]    E2M1 codes of R, element 2i in the low nibble
//   scales       u8   swizzled E4M3 block scales of R (128-row x 64-K atoms)
//   l2t          bf16 [N][rank]   (L2 / g_w) transposed (rank contiguous)
//   bias         bf16 [N]         zeros when the layer has no bias; zero-padded to a multiple
//                                 of 256 columns, so an output tile of N's ragged end (N % 64
//                                 == 0) reads its bias inside the blob
// Every section starts on a 1024-byte boundary.
#pragma once

#include <stddef.h>
#include <stdint.h>

namespace svdq {

constexpr int kAbiVersion = 2;
constexpr int kRank = 32;
constexpr size_t kBlobAlign = 1024;

struct BlobLayout {
  size_t l1s, codes, scales, l2t, bias, total;
};

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Bytes of the swizzled scale tensor for `rows` rows and K columns (rows padded to 128).
inline size_t swizzled_scale_bytes(size_t rows, size_t K) {
  return align_up(rows, 128) * (K / 16);
}

// Offset of the scale of (row, group) in a swizzled scale tensor with K columns.
inline size_t swizzled_scale_offset(size_t row, size_t group, size_t K) {
  const size_t rb = row / 128, r = row % 128;
  const size_t atom = group / 4, j = group % 4;
  return (rb * (K / 64) + atom) * 512 + (r % 32) * 16 + (r / 32) * 4 + j;
}

inline BlobLayout blob_layout(size_t N, size_t K, size_t rank) {
  BlobLayout L;
  size_t off = kBlobAlign;                      // header, padded
  L.l1s = off;    off = align_up(off + 2 * rank * K * 2, kBlobAlign);
  L.codes = off;  off = align_up(off + N * K / 2, kBlobAlign);
  L.scales = off; off = align_up(off + swizzled_scale_bytes(N, K), kBlobAlign);
  L.l2t = off;    off = align_up(off + N * rank * 2, kBlobAlign);
  L.bias = off;   off = align_up(off + align_up(N, 256) * 2, kBlobAlign);
  L.total = off;
  return L;
}

// Packed weight blob of the int4 / group-64 row (svdq_int4_pack_weights): the same 1 KB header
// ("SVDQINT4") and l1s section, then
//   codes        u8   [N][K]      each int4 code -7..7 as its E4M3 byte (exact: the fp8 MMA
//                                 multiplies the integers exactly)
//   scales       f32  [K/64][N]   the per-64 bf16 scales widened to fp32 (exact), group-major:
//                                 a tile's columns of one group are contiguous
//   l2t          bf16 [N][rank]   L2 transposed (no per-tensor scale in this format)
//   bias         bf16 [N]
inline BlobLayout blob_layout_int4(size_t N, size_t K, size_t rank) {
  BlobLayout L;
  size_t off = kBlobAlign;
  L.l1s = off;    off = align_up(off + 2 * rank * K * 2, kBlobAlign);
  L.codes = off;  off = align_up(off + N * K, kBlobAlign);
  L.scales = off; off = align_up(off + N * (K / 64) * 4, kBlobAlign);
  L.l2t = off;    off = align_up(off + N * rank * 2, kBlobAlign);
  L.bias = off;   off = align_up(off + N * 2, kBlobAlign);
  L.total = off;
  return L;
}

struct BlobHeader {
  char magic[8];        // "SVDQNVF4"
  int32_t abi_version;
  int32_t N, K, rank;
  float w_global_scale;
};

}  // namespace svdq
