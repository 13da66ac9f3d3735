// Host helper: TMA tensor maps over bf16 arrays laid out [heads][rows][d].
#pragma once

#include <cuda.h>

namespace ssa {

// 3-D map (d, rows, heads) of a contiguous [heads][rows][d] bf16 array with
// boxes of 64 d x box_rows rows x 1 head and the 128-byte swizzle (a box row
// is one 128-byte swizzle row).  Rows past `rows` read as zeros.  Returns
// false if the driver's encoder is unavailable or rejects the arguments
// (base not 16-byte aligned, d not a multiple of 64, box_rows > 256, ...).
bool make_bf16_map(CUtensorMap* m, const void* ptr, int d, int rows, int heads, int box_rows);

}  // namespace ssa
