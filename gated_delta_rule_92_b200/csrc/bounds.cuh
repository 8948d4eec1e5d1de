// bounds.cuh -- device-side range checks of the debug build (GDN2_DEBUG_BOUNDS).
//
// The debug library (libgdn2_debug.so, the same sources compiled with
// -DGDN2_DEBUG_BOUNDS) checks every per-thread global load and store of the
// kernels against the extent of the argument buffer it belongs to.  Before
// each launch the host entry points write those extents -- computed from the
// call's pointers, sizes and the layouts gdn2.h documents, independently of the
// kernels' own index arithmetic -- into a per-device table on the launch's
// stream.  A check that fails does not trap: it records GDN2_ERR_OUT_OF_BOUNDS
// in the device status word and the first failing site (buffer, source line)
// in a second word, and the access is skipped (a load yields zero).  TMA copies
// are bounded by their tensor maps, which the host encodes from the same sizes.
//
// In the release build GDN2_IN_BOUNDS is the constant true and every check
// compiles away.  The debug table is one per device: calls that run at the
// same time on different streams of one device overwrite each other's
// extents, so the debug build expects one call in flight per device.
#pragma once
#include <stdint.h>

namespace gdn2 {

enum BufId : int {
    kBufQ = 0, kBufK, kBufV, kBufLA, kBufB, kBufW, kBufC,   // token tensors
    kBufS0, kBufST, kBufO,                                  // states, output
    kBufGate, kBufNW, kBufCU,                               // epilogue gate, norm weight, cu_seqlens
    kBufCount
};

constexpr int kStatusBounds = 6;   // == GDN2_ERR_OUT_OF_BOUNDS

struct BoundsTable {
    unsigned long long lo[kBufCount], hi[kBufCount];   // [lo, hi) in bytes; lo == hi: no buffer
};

#ifdef GDN2_DEBUG_BOUNDS
__device__ BoundsTable g_bounds;
__device__ unsigned int g_bounds_site = 0u;   // (buffer + 1) << 16 | line of the first failed check

__device__ __noinline__ bool in_bounds(int buf, const void *p, unsigned long long bytes, int line) {
    const unsigned long long a = reinterpret_cast<unsigned long long>(p);
    const unsigned long long lo = g_bounds.lo[buf], hi = g_bounds.hi[buf];
    if (a >= lo && a <= hi && bytes <= hi - a) return true;
    atomicCAS(&g_bounds_site, 0u, (static_cast<unsigned int>(buf + 1) << 16) | (static_cast<unsigned int>(line) & 0xffffu));
    atomicExch(&g_device_status, kStatusBounds);
    return false;
}
#define GDN2_IN_BOUNDS(buf, p, bytes) (::gdn2::in_bounds((buf), (p), (bytes), __LINE__))
#else
#define GDN2_IN_BOUNDS(buf, p, bytes) (true)
#endif

}  // namespace gdn2
