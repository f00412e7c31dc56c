// tc_fwd.cuh -- tcgen05 forward kernel of Lightweight DC attention (bf16 in,
// fp32 accumulate).
//
// One CTA per block of BM (<= 128) consecutive packed query tokens, all heads.
// Keys of the block live in one tile of span = round16(BM + W - 1) rows that
// starts W - 1 tokens before the block; tile column c is key kbase + c.
//
// Phase 1, per head h (double-buffered Q/K tiles in smem):
//   TMA     Q_h [128 x d], K_h [span x d]          (128-byte swizzle)
//   MMA     S_h = Q_h K_h^T  -> TMEM columns [0, span) fp32
//   SIMT    pull the row band of S_h into registers (which frees the S columns
//           for the next head's MMA), mask to the causal window inside the
//           document, softmax per row, P += c[t,h] * p_h with P accumulated in
//           registers (the H maps never leave the chip)
// Phase 2:
//   SIMT    P -> bf16 tile in smem (K-major, swizzled); the block's pmap rows
//           -> smem -> one bulk copy to global
//   per head: TMA V_h [span x d]; MMA U_h = P V_h -> TMEM [128 x d] (two
//           buffers); SIMT o_h = g[t,h] * U_h -> bf16 -> global (32-byte stores)
//
// Warps 0-11 do the SIMT work: warp w reads TMEM lanes 32*(w%4).. (rows of
// the tile) and part w/4 of its quarter's column band.  Warp 12 lane 0
// issues every TMA and MMA.  All waits are bounded (see wait_bar).
#pragma once

#include "tc_common.cuh"

namespace dc {
namespace tc {

template <int D>
struct FwdLayout {
    static constexpr uint32_t kQBytes = 128u * D * 2;        // Q_h tile: D/64 boxes of 128 rows x 128 B
    static constexpr uint32_t kKHalf = 256u * 128;           // one 64-column box of a K/V tile (<= 256 rows)
    static constexpr uint32_t kKBytes = (D / 64) * kKHalf;   // K_h or V_h tile
    static constexpr uint32_t kPBytes = 4u * 16384;          // P tile: 4 blocks of 64 columns x 128 rows
    static constexpr uint32_t kQ0 = 0;
    static constexpr uint32_t kQ1 = kQBytes;
    static constexpr uint32_t kK0 = 2 * kQBytes;
    static constexpr uint32_t kK1 = kK0 + kKBytes;
    // the P tile reuses the Q buffers when they are large enough (free after the last S MMA)
    static constexpr uint32_t kP = (2 * kQBytes >= kPBytes) ? 0u : kK1 + kKBytes;
    static constexpr uint32_t kRed = (kP == 0 ? kK1 + kKBytes : kP + kPBytes);
    // per-row (max, sum) of each split, double-buffered by head parity: [2][kSplits][128] float2
    static constexpr uint32_t kBars = kRed + 2 * kSplits * 128 * 8;
    // pmap rows of the block, contiguous as in global memory, written out by one bulk copy
    static constexpr uint32_t kStage = kBars + 256;
    static constexpr uint32_t kStageBytes = 27u * 1024 + 512;
    static constexpr uint32_t kBytes = kStage + kStageBytes;
    static constexpr uint32_t kAlloc = kBytes + 1024;        // slack to align the base to 1 KiB
    static_assert(kAlloc <= 227u * 1024, "forward tile layout exceeds shared memory");
};

struct FwdArgs {
    Shape s;
    int BM;
    int span;
    const float *c;
    const float *g;
    __nv_bfloat16 *o;
    float *lse;
    __nv_bfloat16 *pmap;
    Seg seg;      // window segment (segmented instantiation only)
};

// Launches of the segmented forward, in order: the far segment's LSE into lse (phase 1
// only); the near segment, which merges its own LSE with it (the whole window's LSE, kept
// in lse), composes its part of P with that and writes o; the far segment again, which
// composes its part with the whole window's LSE and adds its share to o.
enum : int { kFwdSegStats = 1, kFwdSegNear = 2, kFwdSegFarApply = 3 };

// mbarrier slots
enum : int { kBarQK = 0, kBarSFull = 2, kBarSFree = 3, kBarV = 4, kBarUFull = 6, kBarUFree = 8, kBarP = 10,
             kNumBars = 11 };

template <int D, int MAXC, bool SEG = false>
__global__ void __launch_bounds__(kThreads, 1)
fwd_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
           const __grid_constant__ CUtensorMap map_v, const FwdArgs a) {
    using L = FwdLayout<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint64_t *bars = (uint64_t *)(sm + L::kBars);
    uint32_t *tmem_slot = (uint32_t *)(bars + 16);
    volatile int *abort_flag = (volatile int *)(tmem_slot + 1);
    float2 *red = (float2 *)(sm + L::kRed);       // [2][kSplits][128] (max, sum)

    const Shape &s = a.s;
    const int H = s.H, W = s.W, BM = a.BM, span = a.span;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t0 = (int64_t)blockIdx.x * BM;
    const int64_t kbase = SEG ? t0 - a.seg.shift - (W - 1) : t0 - (W - 1);
    // the segmented LSE launch stops after phase 1
    const bool stats_only = SEG && a.seg.mode == kFwdSegStats;

    validate_seqlens(s);
    if (threadIdx.x == 0) {
        for (int i = 0; i < kNumBars; ++i) {
            uint32_t cnt = 1;
            if (i == kBarSFree || i == kBarUFree || i == kBarUFree + 1 || i == kBarP)
                cnt = kComputeThreads;
            ptx::mbar_init(&bars[i], cnt);
        }
        init_ctl(abort_flag, s.wait_ns);
        ptx::fence_mbar_init();
    }
    if (warp == 0) {
        ptx::tmem_alloc(tmem_slot, 512);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp >= kProducerWarp) {
        regs_producer();
        if (warp == kProducerWarp && lane == 0) {
            ptx::prefetch_tensormap(&map_q);
            ptx::prefetch_tensormap(&map_k);
            ptx::prefetch_tensormap(&map_v);
            const uint32_t qk_bytes = L::kQBytes + (D / 64) * span * 128;
            const uint32_t v_bytes = (D / 64) * span * 128;
            auto issue_qk = [&](int h) {
                const int b = h & 1;
                uint8_t *q = sm + (b ? L::kQ1 : L::kQ0);
                uint8_t *k = sm + (b ? L::kK1 : L::kK0);
                ptx::mbar_arrive_expect_tx(&bars[kBarQK + b], qk_bytes);
                for (int kb = 0; kb < D / 64; ++kb) {
                    ptx::tma_load_2d(q + kb * 16384, &map_q, h * D + kb * 64, (int)t0, &bars[kBarQK + b]);
                    ptx::tma_load_2d(k + kb * L::kKHalf, &map_k, h * D + kb * 64, (int)kbase, &bars[kBarQK + b]);
                }
            };
            auto issue_v = [&](int h) {
                const int b = h & 1;
                uint8_t *v = sm + (b ? L::kK1 : L::kK0);
                ptx::mbar_arrive_expect_tx(&bars[kBarV + b], v_bytes);
                for (int kb = 0; kb < D / 64; ++kb)
                    ptx::tma_load_2d(v + kb * L::kKHalf, &map_v, h * D + kb * 64, (int)kbase, &bars[kBarV + b]);
            };
            const uint32_t id_s = ptx::idesc_bf16_f32(128, span, 0, 0);
            const uint32_t id_pv = ptx::idesc_bf16_f32(128, D, 0, 1);

            // ---- phase 1: S_h = Q_h K_h^T into the single S buffer (TMEM columns 0..)
            // (test hook: with s.inject the first CTA never issues head 0's loads, so the
            // wait for them runs out and the CTA takes the abort path; nothing is in flight)
            for (int h = 0; h < H && h < 2; ++h)
                if (!(h == 0 && s.inject && blockIdx.x == 0)) issue_qk(h);
            for (int h = 0; h < H; ++h) {
                const int b = h & 1;
                bool ok = wait_bar(&bars[kBarQK + b], (uint32_t)(h >> 1) & 1, abort_flag);
                if (h >= 1) ok = wait_bar(&bars[kBarSFree], (uint32_t)(h - 1) & 1, abort_flag) && ok;
                ptx::tc_fence_after();
                if (ok) {
                    const uint32_t qa = ptx::smem_u32(sm + (b ? L::kQ1 : L::kQ0));
                    const uint32_t ka = ptx::smem_u32(sm + (b ? L::kK1 : L::kK0));
#pragma unroll
                    for (int k = 0; k < D / 16; ++k) {
                        const uint64_t ad = ptx::smem_desc_sw128(qa + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024);
                        const uint64_t bd = ptx::smem_desc_sw128(ka + (k >> 2) * L::kKHalf + (k & 3) * 32, 16, 1024);
                        ptx::mma_bf16(tmem, ad, bd, id_s, k > 0);
                    }
                }
                ptx::mma_commit(&bars[kBarSFull]);
                if (h + 2 < H) {
                    if (wait_bar(&bars[kBarSFull], (uint32_t)h & 1, abort_flag)) issue_qk(h + 2);
                }
            }
            // ---- phase 2: U_h = P V_h.  V_h reuses the K buffer of the same parity once
            // the last S MMA that read it has completed.
            if (!stats_only && wait_bar(&bars[kBarSFull], (uint32_t)(H - 1) & 1, abort_flag)) {   // every S MMA done
                for (int b = 0; b < 2 && b < H; ++b) issue_v(b);
            }
            bool p_ok = !stats_only && wait_bar(&bars[kBarP], 0, abort_flag);
            const uint32_t pa = ptx::smem_u32(sm + L::kP);
            for (int h = 0; h < (stats_only ? 0 : H); ++h) {
                const int b = h & 1;
                const uint32_t n = (uint32_t)(h >> 1);
                bool ok = wait_bar(&bars[kBarV + b], n & 1, abort_flag) && p_ok;
                if (h >= 2) ok = wait_bar(&bars[kBarUFree + b], (n - 1) & 1, abort_flag) && ok;
                ptx::tc_fence_after();
                if (ok) {
                    const uint32_t va = ptx::smem_u32(sm + (b ? L::kK1 : L::kK0));
                    for (int k = 0; k < span / 16; ++k) {
                        const uint64_t ad = ptx::smem_desc_sw128(pa + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024);
                        const uint64_t bd = ptx::smem_desc_sw128(va + k * 2048, L::kKHalf, 1024);
                        ptx::mma_bf16(tmem + b * 256, ad, bd, id_pv, k > 0);
                    }
                }
                ptx::mma_commit(&bars[kBarUFull + b]);
                if (h + 2 < H) {
                    if (wait_bar(&bars[kBarUFull + b], n & 1, abort_flag)) issue_v(h + 2);
                }
            }
        }
        __syncwarp();
    } else {
        regs_compute();
        // ---------------------------------------------------------------- compute warps
        const int q = warp & 3, split = warp >> 2;
        const int i = 32 * q + lane;                   // tile row = TMEM lane
        const int64_t t = t0 + i;
        const bool valid = (i < BM) && (t < s.N);
        int clo = 1, chi = 0;                           // valid columns of this row: [clo, chi]
        if (valid) {
            if constexpr (SEG) {
                int64_t lo, hi;
                if (seg_window(s, t, a.seg.shift, lo, hi)) {
                    clo = (int)(lo - kbase);
                    chi = (int)(hi - kbase);
                }
            } else {
                clo = (int)(window_lo(s, t) - kbase);
                chi = (int)(t - kbase);
            }
        }
        const Band bd = make_band(q, split, BM, W, span);
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        const float sl2 = s.scale * kLog2e;

        const uint32_t s_cols = tmem + lane_base;          // S_h, columns [0, span)

        // c (phase 1) and g (epilogue) of this row are read once per head.  A first read
        // that misses L2 costs microseconds while every CTA streams its tiles, so the rows
        // are brought into L2 now and each head's value is loaded one head ahead.
        if (valid && split == 0) {
            ptx::prefetch_l2(a.c + t * H);
            ptx::prefetch_l2(a.c + t * H + H - 1);
            ptx::prefetch_l2(a.g + t * H);
            ptx::prefetch_l2(a.g + t * H + H - 1);
        }
        float c_next = valid ? __ldg(a.c + t * H) : 0.f;

        // composed map of this thread's band, accumulated over heads in registers
        float P[MAXC][8];
#pragma unroll
        for (int cc = 0; cc < MAXC; ++cc)
#pragma unroll
            for (int e = 0; e < 8; ++e) P[cc][e] = 0.f;
        // column c is in this row's window iff (unsigned)(c - span_lo) <= span_n; a row with an
        // empty window (clo > chi: past the block or past N) gets span_lo = ~0u, so no c passes
        const uint32_t span_lo = (chi >= clo) ? (uint32_t)clo : ~0u;
        const uint32_t span_n = (chi >= clo) ? (uint32_t)(chi - clo) : 0u;

        for (int h = 0; h < H; ++h) {
            const float ch = c_next;
            if (h + 1 < H) c_next = valid ? __ldg(a.c + t * H + h + 1) : 0.f;
            wait_bar(&bars[kBarSFull], (uint32_t)h & 1, abort_flag);
            ptx::tc_fence_after();
            // pull this thread's band of S_h into registers with one wait
            uint32_t xr[MAXC][8];
#pragma unroll
            for (int cc = 0; cc < MAXC; ++cc)
                if (cc < bd.mync) ptx::tmem_ld8_issue(s_cols + bd.cb + (bd.c0 + cc) * 8, xr[cc]);
            ptx::tmem_wait_ld();
            float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};   // independent chains
#pragma unroll
            for (int cc = 0; cc < MAXC; ++cc) {
                if (cc < bd.mync) {
                    ptx::reg_fence8(xr[cc]);
                    const uint32_t col = (uint32_t)(bd.cb + (bd.c0 + cc) * 8);
                    // chunks inside every lane's window (most of the band) skip the mask
                    if (__all_sync(0xffffffffu, col - span_lo <= span_n && col + 7 - span_lo <= span_n)) {
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const float v = __uint_as_float(xr[cc][e]) * sl2;
                            xr[cc][e] = __float_as_uint(v);
                            mx[e & 3] = fmaxf(mx[e & 3], v);
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            float v = __uint_as_float(xr[cc][e]) * sl2;
                            v = (col + e - span_lo <= span_n) ? v : -INFINITY;
                            xr[cc][e] = __float_as_uint(v);
                            mx[e & 3] = fmaxf(mx[e & 3], v);
                        }
                    }
                }
            }
            ptx::tc_fence_before();
            ptx::mbar_arrive(&bars[kBarSFree]);   // S columns free for the next head's MMA
            if constexpr (SEG) {
                if (a.seg.mode == kFwdSegFarApply) {   // p_h = 2^(s log2e - lse log2e), whole window's LSE
                    const float lref = valid ? __ldg(a.lse + t * H + h) * kLog2e : 0.f;
                    const float coef = ch;
#pragma unroll
                    for (int cc = 0; cc < MAXC; ++cc)
                        if (cc < bd.mync)
#pragma unroll
                            for (int e = 0; e < 8; ++e)
                                P[cc][e] = fmaf(coef, ex2(__uint_as_float(xr[cc][e]) - lref), P[cc][e]);
                    continue;
                }
            }
            // Softmax with this split's own maximum; the splits' (max, sum) pairs are then
            // combined in one exchange: Z = sum_s Z_s 2^(m_s - m), p = e_s 2^(m_s - m) / Z.
            const float mloc = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
            const bool any = mloc != -INFINITY;   // this split has a column in the row's window
            const float mref = any ? mloc : 0.f;
            float zs[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int cc = 0; cc < MAXC; ++cc) {
                if (cc < bd.mync) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float ev = ex2(__uint_as_float(xr[cc][e]) - mref);
                        xr[cc][e] = __float_as_uint(ev);
                        zs[e & 3] += ev;
                    }
                }
            }
            // near segment: the far segment's LSE (log2 units), read before any split of this
            // row writes the merged value
            float lfar2 = 0.f;
            if constexpr (SEG) lfar2 = (valid && !stats_only) ? a.lse[t * H + h] * kLog2e : 0.f;
            float2 *rd = red + (h & 1) * (kSplits * 128);
            rd[split * 128 + i] = make_float2(mloc, (zs[0] + zs[1]) + (zs[2] + zs[3]));
            pair_sync(q);
            float2 ms[kSplits];
#pragma unroll
            for (int sp = 0; sp < kSplits; ++sp) ms[sp] = rd[sp * 128 + i];
            float m = ms[0].x;
#pragma unroll
            for (int sp = 1; sp < kSplits; ++sp) m = fmaxf(m, ms[sp].x);
            if (!valid) m = 0.f;
            float Z = 0.f;
#pragma unroll
            for (int sp = 0; sp < kSplits; ++sp) Z += ms[sp].y > 0.f ? ms[sp].y * ex2(ms[sp].x - m) : 0.f;
            if constexpr (SEG) {
                // log2 of this segment's normalizer (-inf: no key of the row in it)
                const float l2 = Z > 0.f ? m + __log2f(Z) : -INFINITY;
                if (stats_only) {   // far segment's LSE
                    if (split == 0 && valid) a.lse[t * H + h] = l2 * kLn2;
                    continue;
                }
                // near segment: the whole window's normalizer, log2(2^l2 + 2^lfar2)
                const float hi = fmaxf(l2, lfar2), lo = fminf(l2, lfar2);
                const float lw2 = (lo == -INFINITY) ? hi : hi + __log2f(1.f + ex2(lo - hi));
                const float coef = (valid && any) ? ch * ex2(mref - lw2) : 0.f;
#pragma unroll
                for (int cc = 0; cc < MAXC; ++cc)
                    if (cc < bd.mync)
#pragma unroll
                        for (int e = 0; e < 8; ++e) P[cc][e] = fmaf(coef, __uint_as_float(xr[cc][e]), P[cc][e]);
                if (split == 0 && valid) a.lse[t * H + h] = lw2 * kLn2;
                continue;
            }
            const float coef = (valid && any) ? ch * ex2(mref - m) / Z : 0.f;
#pragma unroll
            for (int cc = 0; cc < MAXC; ++cc)
                if (cc < bd.mync)
#pragma unroll
                    for (int e = 0; e < 8; ++e) P[cc][e] = fmaf(coef, __uint_as_float(xr[cc][e]), P[cc][e]);
            if (split == 0 && valid && a.lse) a.lse[t * H + h] = (m + __log2f(Z)) * kLn2;
        }

        if (!stats_only) {   // phase 2 (the segmented LSE launch stops here)
            float g_next = valid ? __ldg(a.g + t * H) : 0.f;   // head 0's scale, loaded ahead
            // the far segment adds to o: bring the rows it reads into L2 two heads ahead
            const bool o_add = SEG && a.seg.mode == kFwdSegFarApply && valid;
            if (o_add)
                for (int h = 0; h < H && h < 2; ++h) prefetch_drain_row<D>(a.o + t * s.so + h * D, split);
            // ---- P tile (bf16, K-major, swizzled) in smem; zero the columns outside the band
            uint8_t *ptile = sm + L::kP;
            uint32_t Pb[MAXC][4];   // P rounded to bf16 pairs, also the pmap values
#pragma unroll
            for (int cc = 0; cc < MAXC; ++cc) {
                if (cc < bd.mync) {
                    const int col = bd.cb + (bd.c0 + cc) * 8;
#pragma unroll
                    for (int e = 0; e < 4; ++e) Pb[cc][e] = pack_bf16x2(P[cc][2 * e], P[cc][2 * e + 1]);
                    *(uint4 *)(ptile + sw128_offset(i, col)) = make_uint4(Pb[cc][0], Pb[cc][1], Pb[cc][2], Pb[cc][3]);
                }
            }
            zero_outside_band(ptile, i, split, bd, span);
            ptx::fence_proxy_async_smem();
            ptx::mbar_arrive(&bars[kBarP]);

            // ---- pmap[t][w] = P(t, t-W+1+w) = P at tile column i + w.  The block's rows are one
            // contiguous run of pmap: build it in shared memory from the registers (passes of
            // `rpp` rows when it does not fit) and write it with one bulk copy per pass.
            // A segment owns only columns wofs .. wofs + W - 1 of each row: plain stores.
            if (SEG && a.pmap) {
                if (valid) {
                    uint16_t *prow = (uint16_t *)a.pmap + t * a.seg.wrow + a.seg.wofs;   // prow[w], w < W
#pragma unroll
                    for (int cc = 0; cc < MAXC; ++cc) {
                        if (cc < bd.mync) {
                            const int col = bd.cb + (bd.c0 + cc) * 8;
#pragma unroll
                            for (int e = 0; e < 8; ++e) {
                                const uint32_t w = (uint32_t)(col + e - i);
                                if (w < (uint32_t)W) prow[w] = (uint16_t)(Pb[cc][e >> 1] >> (16 * (e & 1)));
                            }
                        }
                    }
                }
            } else if (a.pmap) {
                const int rows_blk = (int)min((int64_t)BM, s.N - t0);
                const int rpp = min(BM, (int)(L::kStageBytes / (uint32_t)(2 * W)) & ~7);   // rows per pass
                uint16_t *stage = (uint16_t *)(sm + L::kStage);
                for (int r0 = 0; r0 < rows_blk; r0 += rpp) {
                    const int nr = min(rpp, rows_blk - r0);
                    if (i >= r0 && i < r0 + nr) {
                        uint16_t *srow = stage + (i - r0) * W - i;   // srow[col] = pmap[t][col - i]
#pragma unroll
                        for (int cc = 0; cc < MAXC; ++cc) {
                            if (cc < bd.mync) {
                                const int col = bd.cb + (bd.c0 + cc) * 8;
#pragma unroll
                                for (int e = 0; e < 8; ++e) {
                                    const uint32_t w = (uint32_t)(col + e - i);
                                    if (w < (uint32_t)W) srow[col + e] = (uint16_t)(Pb[cc][e >> 1] >> (16 * (e & 1)));
                                }
                            }
                        }
                    }
                    ptx::fence_proxy_async_smem();
                    compute_sync();
                    if (threadIdx.x == 0) {
                        const uint32_t bytes = (uint32_t)nr * W * 2;
                        uint8_t *dst = (uint8_t *)(a.pmap + (t0 + r0) * W);
                        const uint32_t main = bytes & ~15u;
                        for (uint32_t x = main; x < bytes; x += 2)   // ragged end of the tensor
                            *(uint16_t *)(dst + x) = *(const uint16_t *)((const uint8_t *)stage + x);
                        if (main) ptx::bulk_store(dst, stage, main);
                        ptx::bulk_commit();
                        if (r0 + rpp < rows_blk) ptx::bulk_wait_read();
                    }
                    if (r0 + rpp < rows_blk) compute_sync();
                }
            }

            // ---- epilogue: o_h = g[t,h] * U_h; this split drains 16-column chunks [cb16, ce16)
            int cb16, ce16;
            acc_split(split, D / 16, cb16, ce16);
            constexpr int kMaxC16 = (D / 16 + kSplits - 1) / kSplits;
            const bool o_aligned32 = (((uintptr_t)a.o | (uintptr_t)(s.so * 2)) & 31) == 0;
            for (int h = 0; h < H; ++h) {
                const int b = h & 1;
                const uint32_t n = (uint32_t)(h >> 1);
                if (o_add && h + 2 < H) prefetch_drain_row<D>(a.o + t * s.so + (h + 2) * D, split);
                const float gh = g_next;
                if (h + 1 < H) g_next = valid ? __ldg(a.g + t * H + h + 1) : 0.f;
                wait_bar(&bars[kBarUFull + b], n & 1, abort_flag);
                ptx::tc_fence_after();
                uint32_t ur[kMaxC16][16];
#pragma unroll
                for (int c = 0; c < kMaxC16; ++c)
                    if (cb16 + c < ce16) ptx::tmem_ld16_issue(tmem + lane_base + b * 256 + (cb16 + c) * 16, ur[c]);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < kMaxC16; ++c) {
                    if (cb16 + c < ce16) {
                        ptx::reg_fence16(ur[c]);
                        if (valid) {
                            uint32_t w[8];
#pragma unroll
                            for (int e = 0; e < 8; ++e)
                                w[e] = pack_bf16x2(gh * __uint_as_float(ur[c][2 * e]), gh * __uint_as_float(ur[c][2 * e + 1]));
                            if constexpr (SEG) {   // later segments add their share to o
                                if (a.seg.mode == kFwdSegFarApply)
                                    add_bf16x16(w, a.o + t * s.so + h * D + (cb16 + c) * 16, gh, ur[c]);
                            }
                            ptx::st_global_32b(a.o + t * s.so + h * D + (cb16 + c) * 16, w, o_aligned32);
                        }
                    }
                }
                ptx::tc_fence_before();
                ptx::mbar_arrive(&bars[kBarUFree + b]);
            }
        }
    }

    if (threadIdx.x == 0) ptx::bulk_wait_all();   // the pmap copy has left shared memory
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, 512);
    }
}

}  // namespace tc
}  // namespace dc
