// tc_common.cuh -- pieces shared by the tcgen05 kernels: thread roles, bounded
// waits with a CTA-wide abort flag, named barriers, band geometry.
#pragma once

#include "common.cuh"
#include "tc_ptx.cuh"

namespace dc {
namespace tc {

// Four warpgroups: warpgroups 0-2 are the 12 compute warps, three per TMEM lane
// quarter (warp w reads lanes 32*(w%4) .. +31 and takes part w/4 of the
// quarter's columns); warp 12 (warpgroup 3) issues TMA and MMA, warps 13-15
// only lend their registers.  The kernels launch with 128 registers per thread
// (512 threads fill the 64K register file); warpgroup 3 then drops to
// kRegsProducer and the compute warpgroups rise to kRegsCompute, which sums to
// the launch budget (a larger sum would make setmaxnreg.inc wait forever).
// The build checks that ptxas gives every tcgen05 kernel exactly kLaunchRegs.
constexpr int kSplits = 3;
constexpr int kComputeWarps = 4 * kSplits;
constexpr int kComputeThreads = kComputeWarps * 32;
constexpr int kThreads = kComputeThreads + 128;
constexpr int kProducerWarp = kComputeWarps;
constexpr int kLaunchRegs = 128;
constexpr int kRegsProducer = 80;
constexpr int kRegsCompute = 144;
static_assert(kThreads * kLaunchRegs <= 65536, "launch register budget exceeds the register file");
static_assert(kComputeThreads * kRegsCompute + (kThreads - kComputeThreads) * kRegsProducer <= kThreads * kLaunchRegs,
              "register split exceeds the launch budget");
static_assert(kRegsCompute % 8 == 0 && kRegsProducer % 8 == 0 && kRegsProducer >= 24 && kRegsCompute <= 256,
              "setmaxnreg counts must be multiples of 8 in [24, 256]");

__device__ __forceinline__ void regs_producer() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsProducer));
}
__device__ __forceinline__ void regs_compute() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsCompute));
}
constexpr uint32_t kWaitNs = 2000000000u;   // default limit; a legitimate wait lasts microseconds
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Per-CTA control words in shared memory: ctl[0] is the abort flag, ctl[1] the
// wait limit in nanoseconds (copied from Shape::wait_ns by the thread that
// initialises the mbarriers).
__device__ __forceinline__ void init_ctl(volatile int *ctl, uint32_t wait_ns) {
    ctl[0] = 0;
    ctl[1] = (int)wait_ns;
}

// Bounded wait on an mbarrier phase.  After the first timeout anywhere in the
// CTA every later wait returns immediately (false) so the CTA drains to its
// teardown instead of hanging; the status word records the event.
// The loop is compact and not unrolled: it is inlined at every wait of every
// kernel, and small code keeps instruction-cache misses down.  The abort flag and
// the clock are looked at every 64 polls.
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, volatile int *abort_flag) {
    if (*abort_flag) return false;
    uint32_t t0 = 0;
#pragma unroll 1
    for (uint32_t n = 1;; ++n) {
        if (ptx::mbar_try_wait(bar, parity)) return true;
        if ((n & 63) == 0) {
            if (n == 64) t0 = ptx::globaltimer_lo();
            if (*abort_flag || ptx::globaltimer_lo() - t0 > (uint32_t)abort_flag[1]) break;
        }
    }
    *abort_flag = 1;   // after a timeout anywhere in the CTA every later wait returns at once
    raise_status(DC_DEVERR_TIMEOUT);
    return false;
}

// Named barrier among `nthreads` threads (barrier 0 is __syncthreads).
__device__ __forceinline__ void named_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
// The compute warps that share TMEM lane quarter q.
__device__ __forceinline__ void pair_sync(int q) { named_sync(1 + q, 32 * kSplits); }
// All compute warps.
__device__ __forceinline__ void compute_sync() { named_sync(5, kComputeThreads); }

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&v);
}

// w = bf16(old + mult * acc) for 16 consecutive values: old read from `src` (16-byte
// aligned), acc the fp32 accumulator words.  Used where a window segment adds its share
// to an output that an earlier segment wrote.
__device__ __forceinline__ void add_bf16x16(uint32_t w[8], const __nv_bfloat16 *src, float mult, const uint32_t acc[16]) {
    const uint4 o0 = *(const uint4 *)src, o1 = *(const uint4 *)(src + 8);
    const uint32_t old[8] = {o0.x, o0.y, o0.z, o0.w, o1.x, o1.y, o1.z, o1.w};
#pragma unroll
    for (int e = 0; e < 8; ++e)
        w[e] = pack_bf16x2(__uint_as_float(old[e] << 16) + mult * __uint_as_float(acc[2 * e]),
                           __uint_as_float(old[e] & 0xFFFF0000u) + mult * __uint_as_float(acc[2 * e + 1]));
}

// Byte offset of element (row, col) of a K-major, 128-byte-swizzled bf16 tile
// made of 64-column blocks of 128 rows (16 KiB each).
__device__ __forceinline__ uint32_t sw128_offset(int row, int col) {
    return (uint32_t)((col >> 6) * 16384 + row * 128 + ((((col & 63) >> 3) ^ (row & 7)) << 4) + ((col & 7) << 1));
}

// Column band of TMEM lane quarter q in a [128 x span] score tile whose column
// c holds key kbase + c, with kbase = block start - (W - 1) - off: row i's window
// is columns [i + off, i + off + W - 1], so rows 32q .. 32q+31 (those below `rows`)
// need columns [32q + off, 32q + off + rows_q - 1 + W - 1].  The band starts at
// the 8-column boundary at or before that and is split in 8-column chunks between
// the kSplits warps of the quarter.
struct Band {
    int cb;      // first column of the quarter's band
    int nch;     // chunks of 8 columns in the band
    int c0;      // first chunk of this thread's part
    int mync;    // chunks in this thread's part
};

__device__ __forceinline__ Band make_band(int q, int split, int rows, int W, int span, int off = 0) {
    Band b;
    b.cb = (32 * q + off) & ~7;
    const int rows_q = min(32, rows - 32 * q);
    if (rows_q <= 0) {
        b.nch = 0;
    } else {
        int ce = 32 * q + off + rows_q - 1 + W;  // one past the last column used
        ce = (ce + 7) & ~7;
        if (ce > span) ce = span;
        b.nch = (ce - b.cb) >> 3;
    }
    const int per = (b.nch + kSplits - 1) / kSplits;
    b.c0 = split * per;
    b.mync = max(0, min(b.nch - b.c0, per));
    return b;
}

// Zero the columns of tile row `row` outside its quarter's band (split 0 takes the
// columns before the band, the last split those after it).
__device__ __forceinline__ void zero_outside_band(uint8_t *tile, int row, int split, const Band &bd, int span) {
    const uint4 z4 = make_uint4(0, 0, 0, 0);
    const int ce = bd.cb + bd.nch * 8;
    if (split == 0) {
        for (int col = 0; col < bd.cb && col < span; col += 8) *(uint4 *)(tile + sw128_offset(row, col)) = z4;
    } else if (split == kSplits - 1) {
        for (int col = (ce > bd.cb ? ce : bd.cb); col < span; col += 8) *(uint4 *)(tile + sw128_offset(row, col)) = z4;
    }
}

// Window segments.  A window wider than the tile geometry allows (W > 129) is cut into
// segments of at most 128 keys counted back from the query: segment k of query t holds
// keys t - shift - Wseg + 1 .. t - shift (shift = 128 k), inside t's document.  Each
// segment runs the kernels with W = Wseg; pmap and the dP band keep rows of the full
// width `wrow`, where the segment's keys start at column wofs = wrow - shift - Wseg.
struct Seg {
    int shift;   // keys of the segment end `shift` tokens before the query
    int wrow;    // row length of pmap and the dP band (the full window W)
    int wofs;    // first column of the segment in those rows
    int mode;    // what this launch of the kernel does (per-kernel enum)
};

// Keys [lo, hi] of query t in the segment (Wseg = s.W); false when it holds none.
__device__ __forceinline__ bool seg_window(const Shape &s, int64_t t, int shift, int64_t &lo, int64_t &hi) {
    int64_t a = __ldg(s.cu + doc_index(s.cu, s.num_docs, t));
    if (a < 0) a = 0;
    hi = t - shift;
    lo = hi - s.W + 1;
    if (lo < a) lo = a;
    return hi >= lo;
}

// 16-column chunks [begin, end) of a D-column accumulator row drained by this split.
__device__ __forceinline__ void acc_split(int split, int nchunk16, int &begin, int &end) {
    const int per = (nchunk16 + kSplits - 1) / kSplits;
    begin = min(split * per, nchunk16);
    end = min(begin + per, nchunk16);
}

// Prefetch into L2 the 16-column chunks of a D-column bf16 output row that this split
// drains: a segment that adds into an output reads them just before its stores.
template <int D>
__device__ __forceinline__ void prefetch_drain_row(const __nv_bfloat16 *row, int split) {
    int cb16, ce16;
    acc_split(split, D / 16, cb16, ce16);
    for (int c = cb16; c < ce16; ++c) ptx::prefetch_l2(row + c * 16);
}

}  // namespace tc
}  // namespace dc
