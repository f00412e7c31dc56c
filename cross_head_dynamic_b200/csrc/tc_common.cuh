// tc_common.cuh -- pieces shared by the tcgen05 kernels: thread roles, bounded
// waits with a CTA-wide abort flag, named barriers, band geometry.
#pragma once

#include "common.cuh"
#include "tc_ptx.cuh"

namespace dc {
namespace tc {

// 8 compute warps (two per TMEM lane quarter) + 1 producer warp (TMA + MMA issue).
constexpr int kComputeWarps = 8;
constexpr int kComputeThreads = kComputeWarps * 32;
constexpr int kThreads = kComputeThreads + 32;
constexpr int kProducerWarp = kComputeWarps;
constexpr uint64_t kWaitNs = 2000000000ull;   // a legitimate wait lasts microseconds
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Bounded wait on an mbarrier phase.  After the first timeout anywhere in the
// CTA every later wait returns immediately (false) so the CTA drains to its
// teardown instead of hanging; the status word records the event.
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, volatile int *abort_flag) {
    if (*abort_flag) return false;
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = ptx::globaltimer();
    while (true) {
        for (int i = 0; i < 32; ++i)
            if (ptx::mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (ptx::globaltimer() - t0 > kWaitNs) {
            *abort_flag = 1;
            raise_status(DC_DEVERR_TIMEOUT);
            return false;
        }
    }
}

// Named barrier among `nthreads` threads (barrier 0 is __syncthreads).
__device__ __forceinline__ void named_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
// The two compute warps that share TMEM lane quarter q.
__device__ __forceinline__ void pair_sync(int q) { named_sync(1 + q, 64); }
// All compute warps.
__device__ __forceinline__ void compute_sync() { named_sync(5, kComputeThreads); }

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&v);
}

// Byte offset of element (row, col) of a K-major, 128-byte-swizzled bf16 tile
// made of 64-column blocks of 128 rows (16 KiB each).
__device__ __forceinline__ uint32_t sw128_offset(int row, int col) {
    return (uint32_t)((col >> 6) * 16384 + row * 128 + ((((col & 63) >> 3) ^ (row & 7)) << 4) + ((col & 7) << 1));
}

// Column band of TMEM lane quarter q in a [128 x span] score tile whose column
// c holds key kbase + c (kbase = block start - (W - 1)): rows 32q .. 32q+31
// (those below `rows`) need columns [32q, 32q + rows_q - 1 + W - 1].  Split in
// 8-column chunks between the two warps of the quarter.
struct Band {
    int cb;      // first column of the quarter's band
    int nch;     // chunks of 8 columns in the band
    int c0;      // first chunk of this thread's half
    int mync;    // chunks in this thread's half
};

__device__ __forceinline__ Band make_band(int q, int split, int rows, int W, int span) {
    Band b;
    b.cb = 32 * q;
    const int rows_q = min(32, rows - 32 * q);
    if (rows_q <= 0) {
        b.nch = 0;
    } else {
        int ce = b.cb + rows_q - 1 + W;          // one past the last column used
        ce = (ce + 7) & ~7;
        if (ce > span) ce = span;
        b.nch = (ce - b.cb) >> 3;
    }
    const int half = (b.nch + 1) >> 1;
    b.c0 = split * half;
    b.mync = max(0, min(b.nch - b.c0, half));
    return b;
}

}  // namespace tc
}  // namespace dc
