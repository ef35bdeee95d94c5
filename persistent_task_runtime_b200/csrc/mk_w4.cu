// Host-side packing of 4-bit weight matrices (W4A16) into the layout the
// persistent kernel streams: the tensor-core-aware reordering of the Ada-MK
// summary ("Quantisierungs-bewusste Optimierung"), written for this kernel's
// mma.sync fragments.  See mk.h (MK_W4_*) for the layout.

#include <cstring>

#include "mk_internal.h"

namespace {

inline int64_t packed_bytes(int rows, int cols) {
  if (rows < 1 || cols < MK_W4_BLOCK_COLS || cols % MK_W4_BLOCK_COLS) return -1;
  return static_cast<int64_t>((rows + 15) / 16) * (cols / MK_W4_BLOCK_COLS) * MK_W4_BLOCK_BYTES;
}

}  // namespace

extern "C" {

MK_API int64_t mk_w4_packed_bytes(int rows, int cols) { return packed_bytes(rows, cols); }

MK_API int mk_w4_pack(const uint8_t *codes, const void *scales, int rows, int cols, void *packed) {
  mk::set_last_error("");
  if (codes == nullptr || scales == nullptr || packed == nullptr) {
    mk::set_last_error("mk_w4_pack: NULL pointer");
    return MK_ERR_INVALID_ARG;
  }
  if (packed_bytes(rows, cols) < 0) {
    mk::set_last_error("mk_w4_pack: rows >= 1 and cols a positive multiple of 1024 needed");
    return MK_ERR_INVALID_ARG;
  }
  const uint16_t *sc = static_cast<const uint16_t *>(scales);   // bf16 bits
  uint8_t *out = static_cast<uint8_t *>(packed);
  const int tiles = (rows + 15) / 16, blocks = cols / MK_W4_BLOCK_COLS, groups = cols / MK_W4_GROUP;
  for (size_t i = 0; i < static_cast<size_t>(rows) * cols; ++i)
    if (codes[i] > 15) {
      mk::set_last_error("mk_w4_pack: a code above 15");
      return MK_ERR_INVALID_ARG;
    }
  for (int t = 0; t < tiles; ++t)
    for (int b = 0; b < blocks; ++b) {
      uint8_t *blk = out + (static_cast<size_t>(t) * blocks + b) * MK_W4_BLOCK_BYTES;
      // scales: group-major, 16 rows per group (rows past the end: 0)
      uint16_t *bs = reinterpret_cast<uint16_t *>(blk);
      for (int j = 0; j < MK_W4_BLOCK_COLS / MK_W4_GROUP; ++j)
        for (int r = 0; r < 16; ++r) {
          const int row = 16 * t + r;
          bs[j * 16 + r] = row < rows
                               ? sc[static_cast<size_t>(row) * groups + b * (MK_W4_BLOCK_COLS / MK_W4_GROUP) + j]
                               : 0;
        }
      // codes: 32 sub-blocks of 32 columns; per mma lane (g, q) 8 bytes:
      // row g then row g + 8, columns 8 q .. 8 q + 7
      uint32_t *bw = reinterpret_cast<uint32_t *>(blk + 256);
      for (int s = 0; s < 32; ++s)
        for (int lane = 0; lane < 32; ++lane)
          for (int h = 0; h < 2; ++h) {
            const int g = lane >> 2, q = lane & 3;
            const int row = 16 * t + g + 8 * h;
            const int col0 = b * MK_W4_BLOCK_COLS + 32 * s + 8 * q;
            uint32_t w = 0;
            for (int i = 0; i < 8; ++i) {
              const uint32_t n = row < rows ? codes[static_cast<size_t>(row) * cols + col0 + i] : 8u;
              // columns 2k, 2k+1 -> bits 4k (low half) and 16 + 4k (high half)
              w |= n << ((i & 1) * 16 + (i >> 1) * 4);
            }
            bw[s * 64 + lane * 2 + h] = w;
          }
    }
  return MK_OK;
}

}  // extern "C"
