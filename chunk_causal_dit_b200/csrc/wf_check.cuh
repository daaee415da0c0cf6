// wf_check.cuh -- bounds checks of the debug build (compiled with -DWF_CHECK).
//
// The kernels' global accesses come in two kinds:
// - TMA tensor loads, clipped to their tensor maps by the hardware;
// - plain loads and stores at addresses computed from the plan's arithmetic (ring
//   slots, token rows, heads, table entries).
// WF_BOUNDS guards the second kind (WF_CHECKED re-tests a condition that a
// WF_BOUNDS already recorded).  In the debug build a failed check sets
// kStatusBounds in the plan's status word, records the site (first one wins) and
// the access is skipped: nothing traps, and wf_sync_status reports
// WF_ERR_BOUNDS.  In the normal build the macro is the constant true, so the
// guarded code is what it would be without it.
//
// The attention kernels' remaining computed accesses are their O and lse stores:
// row c*L + q_row with q_row < L guarded, c < W and h < H by the unit decoding.
// They are left unchecked so that those kernels stay as profiled.
#pragma once
#include "wf_internal.h"

namespace wf {

constexpr uint32_t kStatusBounds = 2u;      // status bit: a debug-build bounds check failed

enum : uint32_t {
    kSiteAppend = 0x101,
    kSiteQuantRows = 0x201,
    kSiteQuantTiles = 0x202,
    kSiteLayerNorm = 0x301,
    kSiteGemmStore = 0x401,
    kSiteGemmQkv = 0x402,
    kSiteGemmTable = 0x403,
};

#ifdef WF_CHECK
__device__ __forceinline__ bool bounds_ok(bool ok, DeviceWords *words, uint32_t site)
{
    if (!ok && words != nullptr) {
        atomicOr(&words->status, kStatusBounds);
        atomicCAS(&words->timeout_where, 0u, site);
    }
    return ok;
}
#define WF_BOUNDS(cond, words, site) ::wf::bounds_ok((cond), (words), (site))
#define WF_CHECKED(cond) (cond)
#else
#define WF_BOUNDS(cond, words, site) true
#define WF_CHECKED(cond) true
#endif

}  // namespace wf
