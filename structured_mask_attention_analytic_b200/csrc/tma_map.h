// Host-side TMA tensor maps of the [batch][len][heads][d] operands.
#pragma once

#include <cuda.h>
#include <stddef.h>
#include <stdint.h>

namespace sma {

// 4D map over [B][len][heads][d] (d contiguous, 16-bit elements), box =
// 64 x box_heads x (128 / box_heads) x 1, 128-byte swizzle, zero fill
// outside the tensor.  A box of several heads lands in shared memory as 128
// rows ordered (row, head): row r of the tile is head r % box_heads of
// sequence row r / box_heads.  Returns false and writes a message if the
// driver entry point is missing or the encoding is rejected.
bool encode_map(CUtensorMap* map, const void* ptr, int dtype, int d, int heads, int len, int batch,
                int64_t s_head, int64_t s_row, int64_t s_batch, char* msg, size_t msg_len,
                int box_heads = 1);

// 4D map over a float32 [B][len][heads][d] accumulator for bulk reductions:
// box = box_d x 1 x box_rows x 1, 128-byte swizzle (box_d * 4 must be 128).
bool encode_map_f32(CUtensorMap* map, const void* ptr, int d, int heads, int len, int batch,
                    int box_d, int box_rows, char* msg, size_t msg_len);

}  // namespace sma
