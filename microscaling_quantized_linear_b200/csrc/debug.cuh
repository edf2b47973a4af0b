// debug.cuh -- device-side bounds checks of the debug build.
//
// The library compiled with NVQ_DEBUG defined (libnvq_debug.so) checks, before
// each global access whose address a kernel computes from its indices, that
// the accessed bytes lie inside the buffer the launch was given, whose extent
// follows from the call's sizes (rows, blocks per row, pitch, tile counts).
// A failed check sets kStatusBounds in the device status word and the access
// is skipped: a store writes nothing, a load reads zeros, a bulk copy into a
// pipeline stage counts its bytes on the stage's barrier without data, so no
// wait is left to run out.  Nothing traps.  In the normal build every check
// is the constant true and compiles away.
#pragma once
#include <cstdint>

namespace nvq {

constexpr unsigned int kStatusBounds = 8;

#ifdef NVQ_DEBUG
constexpr bool kDebugBuild = true;
#else
constexpr bool kDebugBuild = false;
#endif

// [off, off + bytes) inside [0, extent)?  (Any unit, the same for all three.)
__device__ __forceinline__ bool in_bounds(uint64_t off, uint64_t bytes, uint64_t extent, unsigned int* status) {
#ifdef NVQ_DEBUG
    if (off + bytes <= extent) return true;
    atomicOr(status, kStatusBounds);
    return false;
#else
    (void)off;
    (void)bytes;
    (void)extent;
    (void)status;
    return true;
#endif
}

// Bytes of a scale array in the 128x4 tile order: rows padded to 128, ctiles
// column tiles of 4 scales.
__device__ __forceinline__ uint64_t sf_extent(uint32_t rows, uint32_t ctiles) {
    return (uint64_t)((rows + 127u) & ~127u) * ctiles * 4u;
}

// Elements of a row-major [rows, cols] array with row pitch ld.
__device__ __forceinline__ uint64_t pitched_extent(uint32_t rows, uint32_t cols, uint32_t ld) {
    return rows == 0 ? 0 : (uint64_t)(rows - 1) * ld + cols;
}

}  // namespace nvq
