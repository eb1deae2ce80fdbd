// Host helpers for TMA tensor maps (cuTensorMapEncodeTiled through the
// runtime's driver entry point, so the library links only cudart).
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <stdint.h>

namespace pa {

// cuTensorMapEncodeTiled, or nullptr when the driver does not provide it.
PFN_cuTensorMapEncodeTiled_v12000 encode_fn();

// 2-D view of a pool [NB, Hk, 16, d]: rows = NB * Hk * 16 tokens, d columns;
// boxes of 16 rows x 128 bytes, 128-byte swizzle.
bool encode_pool_map(CUtensorMap *m, const void *base, int elem_bytes, int d, int64_t rows);

}  // namespace pa
