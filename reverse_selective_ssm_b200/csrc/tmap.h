// Host helper: 2-D TMA tensor maps for row-major matrices.
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace r2l {

// Row-major matrix [rows, inner] of `elem_bytes`-byte elements (2 = bf16,
// 4 = fp32) with a row stride of `ld_bytes`, read in boxes of box_inner ×
// box_rows.  swizzle128 selects the 128-byte swizzle (tensor-core operands);
// otherwise the box lands in shared memory row after row.  Out-of-range
// elements read as zero.  Returns false if the driver rejects the map.
bool make_tmap_2d(CUtensorMap* m, const void* base, int elem_bytes, long long inner, long long rows,
                  long long ld_bytes, int box_inner, int box_rows, bool swizzle128);

}  // namespace r2l
