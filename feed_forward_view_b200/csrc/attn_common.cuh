// attn_common.cuh -- pieces shared by the two attention kernels (attn_fwd.cu,
// bf16; attn_fwd_f32.cu, the fp32 mode): bounded mbarrier waits and the
// tensor maps their TMA loads read.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "pdl.cuh"
#include "sm100.cuh"
#include "vggt_internal.h"

namespace vggt {
namespace attn {

// Bounded wait that also gives up once this CTA or any other CTA reported a
// timeout; records a timeout of its own. The barrier is polled back to back
// (try_wait itself suspends the thread for a while); the abort flag, the clock
// and the global status word are only looked at every 256 polls, so that a
// phase that completes is noticed within one poll and not one global-memory
// round trip later.
struct Waiter {
    long long limit;
    volatile int* abort;
    int* status;

    __device__ __forceinline__ bool operator()(uint32_t bar, uint32_t parity) const {
        if (mbar_try_wait(bar, parity)) return true;
        const long long t0 = clock64();
        for (uint32_t it = 1;; ++it) {
            if (mbar_try_wait(bar, parity)) return true;
            if ((it & 255u) == 0) {
                if (*abort) return false;
                if (*reinterpret_cast<volatile int*>(status) & kStatusTimeout) {
                    *abort = 1;
                    return false;
                }
                if (clock64() - t0 > limit) {
                    *abort = 1;
                    atomicOr(status, kStatusTimeout);
                    return false;
                }
            }
        }
    }
};

// Wait used while draining on the way out: ignores the abort flags.
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity, long long limit) {
    if (mbar_try_wait(bar, parity)) return;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > limit) return;
    }
}

// The constant [1, 0, ..., 0] key rows of the PV MMA's ones column, in the
// 128-byte-swizzled layout the MMA reads: the 16-byte chunk c of row r sits
// at chunk c ^ (r % 8), so element 0 of row r lies at byte r * 128 + (r % 8)
// * 16. All threads of the block call it; `bytes` is the tile's size.
__device__ __forceinline__ void fill_ones_tile(uint8_t* tile, int bytes, int nthreads) {
    for (int i = threadIdx.x; i < bytes / 16; i += nthreads) {
        const int r = i >> 3, chunk = i & 7;
        uint4 w = make_uint4(0u, 0u, 0u, 0u);
        if (chunk == (r & 7)) w.x = 0x3F80u;  // bf16 1.0 in the low half
        reinterpret_cast<uint4*>(tile)[i] = w;
    }
}

// 3-D bf16 tensor map with a {64, box1, box2} box and 128-byte swizzling
// (host). False if the driver entry point is missing or encoding failed.
bool make_map(CUtensorMap* map, const void* base, uint64_t d1, uint64_t d2, uint64_t stride1_bytes,
              uint64_t stride2_bytes, uint32_t box1, uint32_t box2);

}  // namespace attn
}  // namespace vggt
