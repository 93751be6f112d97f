// TMA tensor maps of the (batch, seq, heads, dim) arrays the tcgen05 kernels read (host side).
#pragma once

#include <cuda.h>

namespace sdpa {

// A (batch, seq, heads, dim) 16-bit array as a 4-d tensor map: box = 64 dims x 1 head x 128
// rows x 1 batch, 128-byte swizzle (the K-major / MN-major operand layout of the tcgen05 shared
// memory descriptors). Rows past `seq` read as 0. False if the driver's encoder is unavailable
// or refuses the array (base not 16-byte aligned).
bool make_map(CUtensorMap* m, const void* base, int dtype, int D, int heads, int seq, int batch);

}  // namespace sdpa
