// hg_check.cuh -- range checks of the checked build.
//
// Built with -DHASHGRID_CHECKED (libhashgrid_checked.so), every global-memory access of the
// kernels is tested against the extent of the buffer it belongs to. Before each launch the
// host records, per buffer role, the byte range the call may touch; an access outside its
// role's range sets that role's bit in a device status word and is skipped (a load reads
// zeros), so a wrong index becomes an error code instead of a fault. After the kernel the
// host reads the word back on the call's stream, clears it and returns
// HASHGRID_ERR_DEVICE_CHECK naming the roles. The checked build is synchronous (each call
// waits for its kernel) and slower; it exists to run the parity tests under it. In the
// regular build in_bounds() is the constant true and every check compiles away.
#pragma once

#include <stdint.h>

namespace hg {

enum CheckRole {
    kChkX = 0,      // point coordinates (read)
    kChkTable = 1,  // feature table (read; Adam also writes it)
    kChkOut = 2,    // encoding, dL/dx, MLP output or index export (written)
    kChkDout = 3,   // upstream gradient rows (read)
    kChkGrad = 4,   // table gradient (reduced into; Adam reads and may clear it)
    kChkM = 5,      // Adam first moment
    kChkV = 6,      // Adam second moment
    kChkRoles = 7
};

struct CheckRanges {
    uint64_t lo[kChkRoles];
    uint64_t hi[kChkRoles];  // one past the last byte; lo == hi: the role is not used
};

#ifdef HASHGRID_CHECKED
__device__ CheckRanges g_check_ranges;
__device__ unsigned int g_check_flags;

template <int R>
__device__ __forceinline__ bool in_bounds(const void* p, uint32_t bytes) {
    const uint64_t a = (uint64_t)(uintptr_t)p;
    if (a >= g_check_ranges.lo[R] && a + bytes <= g_check_ranges.hi[R]) return true;
    atomicOr(&g_check_flags, 1u << R);
    return false;
}
#else
template <int R>
__device__ __forceinline__ constexpr bool in_bounds(const void*, uint32_t) {
    return true;
}
#endif

}  // namespace hg
