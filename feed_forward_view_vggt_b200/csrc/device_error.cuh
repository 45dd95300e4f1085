// device_error.cuh -- the library's 4-byte device error word and the
// optional device index checks.
//
// Bits of g_vggt_error:
//   bit 0        a bounded wait ran out (kErrTimeout); bits 8..15 = the code
//                of the first wait site that gave up;
//   bit 1        (built with -DVGGT_DEBUG only) an index check failed
//                (kErrBounds); bits 16..23 = the code of the first check
//                site that failed.
// vggt_check() reads and clears the word.
#pragma once
#include <cstdint>

namespace vggt {

enum : uint32_t { kErrTimeout = 1u, kErrBounds = 2u };

// Index-check sites (bits 16..23 of the error word).
enum : uint32_t {
    kCheckAttnRow = 1,   // attention: output / lse row and head
    kCheckSgaSeed,       // attention (SGA): the query's own K row, mult, kbar
    kCheckMeanfillRead,  // mean-fill: token row read
    kCheckMeanfillSlot,  // mean-fill: gathered slot written
    kCheckIndexToken,    // index build: kept token id
    kCheckQkvRow         // QKV projection epilogue: output row
};

__device__ unsigned int g_vggt_error;

__device__ __forceinline__ bool record_bounds_failure(uint32_t site)
{
    atomicCAS(&g_vggt_error, 0u, kErrBounds | (site << 16));
    atomicOr(&g_vggt_error, kErrBounds);
    return false;
}

} // namespace vggt

// VGGT_IN_RANGE(cond, site): true when the access guarded by `cond` may go
// ahead.  Release builds compile it away (the index arithmetic is correct by
// construction and tested); -DVGGT_DEBUG builds evaluate `cond` and, when it
// fails, record the site in the error word and make the caller skip the
// access (no trap, no assert).
#ifdef VGGT_DEBUG
#define VGGT_IN_RANGE(cond, site) ((cond) ? true : ::vggt::record_bounds_failure(site))
#else
#define VGGT_IN_RANGE(cond, site) true
#endif
