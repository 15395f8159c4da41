// Host helper: 2-D TMA tensor maps for row-major matrices.
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace r2l {

// Row-major matrix [rows, inner] of `elem_bytes`-byte elements (2 = bf16,
// 4 = fp32) with a row stride of `ld_bytes`, moved in boxes of box_inner ×
// box_rows.  swizzle_bytes: 0 (the box lands in shared memory row after row),
// 64 or 128 (the 16-byte chunks of each row are permuted by the row index, as
// tensor-core operands and bank-conflict-free staging want).  Out-of-range
// elements read as zero and are not written.  Returns false if the driver
// rejects the map.
bool make_tmap_2d(CUtensorMap* m, const void* base, int elem_bytes, long long inner, long long rows,
                  long long ld_bytes, int box_inner, int box_rows, int swizzle_bytes);

// The same matrix (rows even) seen as {inner, parity, rows / 2}: a box
// {box_inner, 1, box_rows} at coordinates (x, p, i0) holds rows 2·(i0 + i) + p
// for i = 0 .. box_rows − 1, i.e. every second row starting at 2·i0 + p.
bool make_tmap_rows_by_parity(CUtensorMap* m, const void* base, int elem_bytes, long long inner, long long rows,
                              long long ld_bytes, int box_inner, int box_rows, int swizzle_bytes);

}  // namespace r2l
