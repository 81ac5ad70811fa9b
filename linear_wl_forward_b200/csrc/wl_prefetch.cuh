// Cross-call L2 prefetch: the CTAs of a launch pull a list of device ranges
// (normally the weights of the call that follows in the stream) into L2 while
// this call runs, so that call starts from L2 instead of HBM.
#pragma once

#include "wl_common.cuh"
#include "wl_internal.h"

namespace wl {

// CTA c of `grid` issues its 1/grid share of the list's bytes (the ranges laid
// end to end, shares cut at 16-byte multiples) as bulk prefetches of at most
// kPrefetchPiece bytes.  One thread calls it.  A prefetch only moves data into
// L2, the device's point of coherence, so it never changes what any kernel
// reads; it may be issued before the wait for the previous kernel.
__device__ __forceinline__ void l2_prefetch_share(const PrefetchList &pf, unsigned c, unsigned grid) {
    if (pf.n <= 0 || grid == 0) return;
    const uint64_t lo = (pf.total * c / grid) & ~uint64_t(15);
    const uint64_t hi = c + 1 == grid ? pf.total : (pf.total * (c + 1) / grid) & ~uint64_t(15);
    uint64_t b0 = 0;
    for (int i = 0; i < pf.n && b0 < hi; ++i) {
        const uint64_t b1 = b0 + pf.bytes[i];
        uint64_t s = lo > b0 ? lo : b0;
        const uint64_t e = hi < b1 ? hi : b1;
        while (s < e) {
            const uint64_t left = e - s;
            const uint32_t n = left < kPrefetchPiece ? (uint32_t)left : kPrefetchPiece;
            bulk_prefetch_l2(pf.ptr[i] + (s - b0), n);
            s += n;
        }
        b0 = b1;
    }
}

}  // namespace wl
