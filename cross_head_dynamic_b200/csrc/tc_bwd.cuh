// tc_bwd.cuh -- tcgen05 backward kernels of Lightweight DC attention (bf16 in,
// fp32 accumulate).  The gradients are the chain rule of
//   p_h = softmax(sigma q_h k_h^T) on the window, P = sum_h c_h p_h, o_h = g_h P v_h:
//   E_h = dO_h v_h^T, dP = sum_h g_h E_h, dg_h = sum_j P E_h, dc_h = sum_j dP p_h,
//   ds_h = c_h p_h (dP - dc_h), dq_h = sigma ds_h k_h, dk_h = sigma ds_h^T q_h,
//   dv_h = P^T (g_h dO_h).
//
// Query side (one CTA per block of BM query tokens, all heads):
//   phase 1, per head: MMA E_h = dO_h V_h^T -> TMEM; SIMT dP += g_h E_h
//            (registers), dg_h = sum_j P E_h with P from the forward's pmap
//            (the CTA's pmap rows arrive by one bulk load and are kept in
//            registers); dP is then written, by one bulk store, as a band [N][W]
//            in the workspace for the key side, which must see exactly the dP
//            that dc was computed from.
//   phase 2, per head: MMA S_h = Q_h K_h^T -> TMEM; SIMT p_h from lse,
//            dc_h = sum_j dP p_h, ds_h -> bf16 tile in smem; MMA dQ_h = ds_h K_h.
//            With the ds band (DSB), every ds_h(t, j) also goes to the key-major
//            band dsb[h][j][t - j] in the workspace, and no dP band is written.
//            With the ds tile hand-off (DST) the key tile starts BM keys before the
//            block (span = 2 BM), and the ds tile itself, [BM queries x 2 BM keys],
//            goes to the workspace by TMA tensor stores; no dP band either.
// Key side (one CTA per block of BK key tokens; the queries that see them span
// round16(BK + W - 1) rows starting at the block):
//   phase 1, per head: scale the dO_h rows by g_h in smem; MMA dV_h = P^T gdO_h
//            with P^T built once from pmap.
//   phase 2, per head, bwd_key_kernel: the block's rows of the ds band -> ds^T
//            tile; MMA dK_h = ds^T_h Q_h.
//   phase 2, per head, bwd_key_seg_kernel (window segments, or a workspace that
//            holds only the dP band): MMA S^T_h = K_h Q_h^T -> TMEM; SIMT ds^T
//            from lse, c, dc and the query side's dP; MMA dK_h = ds^T_h Q_h.
//   bwd_key_dst_kernel (ds tiles): the key block's ds^T_h arrives by four TMA boxes
//            of the query side's tiles (its own block's and the next block's) and is
//            used as it lands, as an MN-major A operand; the compute warps only build
//            the P tile once, scale dO and drain.
// In both phase-2 loops the gradient MMA of head h runs while the SIMT warps
// work on the scores of head h+1: the producer issues S_{h+1} before dQ_h/dK_h;
// the warps write the next ds tile once that MMA has read the current one and
// then drain its accumulator (two accumulator buffers in TMEM).
// Same thread roles as the forward: warps 0-11 SIMT (three per TMEM lane
// quarter), warp 12 lane 0 issues TMA and MMA; every wait is bounded.
#pragma once

#include "tc_common.cuh"

namespace dc {
namespace tc {

constexpr int kBwdMaxSpan = 240;   // key/query tile rows, keeps both kernels within 227 KiB of smem
// Row length of the ds band for every W <= 129 (129 rounded up to 8): a constant, so that the
// query side's band stores of one head all address from one base register.
constexpr int kDsbRow = 136;

struct BwdArgs {
    Shape s;
    int BM;       // query (or key) block
    int span;     // key (or query) tile rows, multiple of 16, <= kBwdMaxSpan
    const float *c;
    const float *g;
    const float *lse;
    const __nv_bfloat16 *pmap;
    const float *dc_in;    // key side: dc from the query side
    __nv_bfloat16 *dq;     // query side out
    float *dc;
    float *dg;
    float *band;           // dP band [N][W]: written by the query side, read by the key side
    __nv_bfloat16 *dk;     // key side out
    __nv_bfloat16 *dv;
    Seg seg;               // window segment (segmented instantiations only)
    __nv_bfloat16 *dsb;    // ds band [H][N][kDsbRow], key-major (see bwd_key_kernel)
};

// Segmented query side, launched in this order: the far segment's dP band, dg and dc
// (partial sums); the near segment, which completes dg and dc and writes its share of
// dq; the far segment again, which adds its share of dq (it needs the complete dc).
enum : int { kQSegFarPart1 = 1, kQSegNear = 2, kQSegFarPart2 = 3 };
// Segmented key side: the first segment writes dk and dv, the next one adds to them.
enum : int { kKSegWrite = 1, kKSegAdd = 2 };

// Drain this split's 16-column chunks of one row of a [128 x D] fp32 accumulator with one
// TMEM round trip for all of them (for kernels with registers to spare).
template <int D>
__device__ __forceinline__ void drain_row_once(uint32_t taddr, __nv_bfloat16 *dst, float mult, bool store, int split,
                                               bool aligned32) {
    int cb16, ce16;
    acc_split(split, D / 16, cb16, ce16);
    constexpr int kMaxC16 = (D / 16 + kSplits - 1) / kSplits;
    uint32_t r[kMaxC16][16];
#pragma unroll
    for (int c = 0; c < kMaxC16; ++c)
        if (cb16 + c < ce16) ptx::tmem_ld16_issue(taddr + (cb16 + c) * 16, r[c]);
    ptx::tmem_wait_ld();
#pragma unroll
    for (int c = 0; c < kMaxC16; ++c) {
        if (cb16 + c < ce16) {
            ptx::reg_fence16(r[c]);
            if (store) {
                uint32_t w[8];
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    w[e] = pack_bf16x2(mult * __uint_as_float(r[c][2 * e]), mult * __uint_as_float(r[c][2 * e + 1]));
                ptx::st_global_32b(dst + (cb16 + c) * 16, w, aligned32);
            }
        }
    }
}

// Drain this split's 16-column chunks of one row of a [128 x D] fp32 accumulator
// (row base address taddr, output row dst): scale, round to bf16, store when `store`
// (full 32-byte sectors; aligned32 says whether the output buffer allows 256-bit stores).
template <int D, bool ADD = false>
__device__ __forceinline__ void drain_row(uint32_t taddr, __nv_bfloat16 *dst, float mult, bool store, int split,
                                          bool aligned32) {
    int cb16, ce16;
    acc_split(split, D / 16, cb16, ce16);
    constexpr int kMaxC16 = (D / 16 + kSplits - 1) / kSplits;
#pragma unroll
    for (int c = 0; c < kMaxC16; ++c) {
        if (cb16 + c < ce16) {   // one 16-column chunk per TMEM round trip keeps register use low
            uint32_t r[16];
            ptx::tmem_ld16_issue(taddr + (cb16 + c) * 16, r);
            ptx::tmem_wait_ld();
            ptx::reg_fence16(r);
            if (store) {
                uint32_t w[8];
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    w[e] = pack_bf16x2(mult * __uint_as_float(r[2 * e]), mult * __uint_as_float(r[2 * e + 1]));
                if constexpr (ADD) add_bf16x16(w, dst + (cb16 + c) * 16, mult, r);   // dst += mult * acc
                ptx::st_global_32b(dst + (cb16 + c) * 16, w, aligned32);
            }
        }
    }
}

// --------------------------------------------------------------------------- query side
enum : int { kQBarLd = 0, kQBarQ = 2, kQBarK = 3, kQBarXFull = 5, kQBarXFree = 6, kQBarDs = 7, kQBarDqFull = 8,
             kQBarDqFree = 10, kQBarPmap = 12, kQBarDsRead = 13, kQNumBars = 14 };

// Copy `bytes` bytes of global memory to shared memory: a bulk copy of the 16-byte
// multiple (completing on `bar`) and plain copies of the rest.  The caller's arrive on
// `bar` (expect_tx) publishes both.
__device__ __forceinline__ void stage_in(void *sdst, const void *gsrc, uint32_t bytes, uint64_t *bar) {
    const uint32_t main = bytes & ~15u;
    for (uint32_t x = main; x < bytes; x += 2)
        *(uint16_t *)((uint8_t *)sdst + x) = *(const uint16_t *)((const uint8_t *)gsrc + x);
    ptx::mbar_arrive_expect_tx(bar, main);
    if (main) ptx::bulk_load(sdst, gsrc, main, bar);
}

// Copy `bytes` bytes of shared memory to global memory: a bulk copy of the 16-byte
// multiple (committed to this thread's bulk group) and plain copies of the rest.
__device__ __forceinline__ void stage_out(void *gdst, const void *ssrc, uint32_t bytes) {
    const uint32_t main = bytes & ~15u;
    for (uint32_t x = main; x < bytes; x += 2)
        *(uint16_t *)((uint8_t *)gdst + x) = *(const uint16_t *)((const uint8_t *)ssrc + x);
    if (main) ptx::bulk_store(gdst, ssrc, main);
    ptx::bulk_commit();
}

template <int D>
struct QSideLayout {
    uint32_t tile_k;   // K or V tile: D/64 boxes of span rows x 128 B
    uint32_t r0, r1, rq, rd, red, bars, bytes;
    __host__ __device__ QSideLayout(int span) {
        tile_k = (uint32_t)(D / 64) * span * 128;
        r0 = 0;
        r1 = tile_k;
        rq = 2 * tile_k;                  // Q (phase 2) / dO buffer 0 (phase 1)
        rd = rq + 128u * D * 2;           // ds tile (phase 2) / dO buffer 1 (phase 1)
        red = rd + 4u * 16384;
        bars = red + 2 * kSplits * 128 * 4;
        bytes = bars + 512;
    }
};

template <int D, int MAXC, bool SEG = false, bool DSB = false, bool DST = false>
__global__ void __launch_bounds__(kThreads, 1)
bwd_query_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                 const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_do,
                 const __grid_constant__ CUtensorMap map_ds, const BwdArgs a) {
    static_assert(!(DSB && DST) && !(SEG && (DSB || DST)), "one hand-off per instantiation");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const Shape &s = a.s;
    const int H = s.H, W = s.W, BM = a.BM, span = a.span;
    const QSideLayout<D> L(span);
    uint64_t *bars = (uint64_t *)(sm + L.bars);
    uint32_t *tmem_slot = (uint32_t *)(bars + 32);
    volatile int *abort_flag = (volatile int *)(tmem_slot + 1);
    float *red = (float *)(sm + L.red);   // [2 parity][kSplits][128]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t0 = (int64_t)blockIdx.x * BM;
    // DST: the key tile starts BM keys before the block, so that the key blocks of the
    // key side are whole 64-column-aligned column ranges of the ds tile; row i's window
    // then starts at column i + off
    const int off = DST ? BM - (W - 1) : 0;
    const int64_t kbase = SEG ? t0 - a.seg.shift - (W - 1) : t0 - (W - 1) - off;
    const bool do_p1 = !SEG || a.seg.mode != kQSegFarPart2;   // phase 1 (E, dP band, dg)
    const bool do_dq = !SEG || a.seg.mode != kQSegFarPart1;   // ds and dQ
    const int ph0 = do_p1 ? H : 0;                            // X-buffer phases before phase 2

    validate_seqlens(s);
    if (threadIdx.x == 0) {
        for (int i = 0; i < kQNumBars; ++i) {
            const bool many = (i == kQBarXFree || i == kQBarDs || i == kQBarDqFree || i == kQBarDqFree + 1);   // 384
            ptx::mbar_init(&bars[i], many ? kComputeThreads : 1);
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
            const uint32_t q_bytes = 128u * D * 2;
            auto issue_e = [&](int h) {   // phase 1 operands of head h: dO_h and V_h
                const int b = h & 1;
                uint8_t *dst_do = sm + (b ? L.rd : L.rq);
                uint8_t *dst_v = sm + (b ? L.r1 : L.r0);
                ptx::mbar_arrive_expect_tx(&bars[kQBarLd + b], q_bytes + L.tile_k);
                for (int kb = 0; kb < D / 64; ++kb) {
                    ptx::tma_load_2d(dst_do + kb * 16384, &map_do, h * D + kb * 64, (int)t0, &bars[kQBarLd + b]);
                    ptx::tma_load_2d(dst_v + kb * span * 128, &map_v, h * D + kb * 64, (int)kbase,
                                     &bars[kQBarLd + b]);
                }
            };
            auto issue_q = [&](int h) {
                ptx::mbar_arrive_expect_tx(&bars[kQBarQ], q_bytes);
                for (int kb = 0; kb < D / 64; ++kb)
                    ptx::tma_load_2d(sm + L.rq + kb * 16384, &map_q, h * D + kb * 64, (int)t0, &bars[kQBarQ]);
            };
            auto issue_k = [&](int h) {
                const int b = h & 1;
                uint8_t *dst = sm + (b ? L.r1 : L.r0);
                ptx::mbar_arrive_expect_tx(&bars[kQBarK + b], L.tile_k);
                for (int kb = 0; kb < D / 64; ++kb)
                    ptx::tma_load_2d(dst + kb * span * 128, &map_k, h * D + kb * 64, (int)kbase, &bars[kQBarK + b]);
            };
            const uint32_t id_x = ptx::idesc_bf16_f32(128, span, 0, 0);   // E and S: [128 x span]
            const uint32_t id_dq = ptx::idesc_bf16_f32(128, D, 0, 1);     // dQ: [128 x D], B MN-major
            // dQ_h = ds_h K_h into accumulator buffer h & 1 (K_h is MN-major for this product)
            auto mma_dq = [&](int h) {
                const int b = h & 1;
                bool ok = wait_bar(&bars[kQBarDs], (uint32_t)h & 1, abort_flag);
                if (h >= 2) ok = wait_bar(&bars[kQBarDqFree + b], (uint32_t)((h >> 1) - 1) & 1, abort_flag) && ok;
                ptx::tc_fence_after();
                if (ok) {
                    const uint32_t dsa = ptx::smem_u32(sm + L.rd);
                    const uint32_t ka = ptx::smem_u32(sm + (b ? L.r1 : L.r0));
                    for (int k = 0; k < span / 16; ++k) {
                        const uint64_t ad = ptx::smem_desc_sw128(dsa + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024);
                        const uint64_t bd = ptx::smem_desc_sw128(ka + k * 2048, span * 128, 1024);
                        ptx::mma_bf16(tmem + 256 + 128 * b, ad, bd, id_dq, k > 0);
                    }
                }
                ptx::mma_commit(&bars[kQBarDqFull + b]);
                if constexpr (DST) {
                    // the ds tile (its first BM rows, 64-column boxes) to the workspace; the
                    // compute warps rewrite it for the next head once the store has read it
                    // (ds_released, after the producer's refills)
                    if (ok) {
                        for (int cb = 0; cb < span; cb += 64)
                            ptx::tma_store_3d(&map_ds, cb, (int)t0, h, sm + L.rd + (cb >> 6) * 16384);
                    }
                    ptx::bulk_commit();
                }
            };
            auto ds_released = [&]() {
                if constexpr (DST) {
                    ptx::bulk_wait_read();
                    ptx::mbar_arrive(&bars[kQBarDsRead]);
                }
            };

            // the CTA's pmap rows (one contiguous [BM][W] run) into the upper half of the ds
            // tile region, which phase 1 does not use (a segment reads its columns directly)
            if (!SEG)
                stage_in(sm + L.rd + 32768, a.pmap + t0 * W, (uint32_t)(min((int64_t)BM, s.N - t0) * W * 2),
                         &bars[kQBarPmap]);
            if (!do_p1) {   // no phase 1: the phase-2 tiles load at once
                issue_q(0);
                for (int b = 0; b < 2 && b < H; ++b) issue_k(b);
            }
            // ---- phase 1: E_h = dO_h V_h^T
            for (int h = 0; h < (do_p1 ? H : 0) && h < 2; ++h) issue_e(h);
            for (int h = 0; h < (do_p1 ? H : 0); ++h) {
                const int b = h & 1;
                bool ok = wait_bar(&bars[kQBarLd + b], (uint32_t)(h >> 1) & 1, abort_flag);
                if (h >= 1) ok = wait_bar(&bars[kQBarXFree], (uint32_t)(h - 1) & 1, abort_flag) && ok;
                ptx::tc_fence_after();
                if (ok) {
                    const uint32_t da = ptx::smem_u32(sm + (b ? L.rd : L.rq));
                    const uint32_t va = ptx::smem_u32(sm + (b ? L.r1 : L.r0));
#pragma unroll
                    for (int k = 0; k < D / 16; ++k) {
                        const uint64_t ad = ptx::smem_desc_sw128(da + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024);
                        const uint64_t bd = ptx::smem_desc_sw128(va + (k >> 2) * span * 128 + (k & 3) * 32, 16, 1024);
                        ptx::mma_bf16(tmem, ad, bd, id_x, k > 0);
                    }
                }
                ptx::mma_commit(&bars[kQBarXFull]);
                // once E_h has completed its buffers are reused: by dO_{h+2} / V_{h+2}, or, for
                // the last use of buffer b, by the phase-2 tiles K_b (and Q_0 for buffer 0)
                if (wait_bar(&bars[kQBarXFull], (uint32_t)h & 1, abort_flag)) {
                    if (h + 2 < H) {
                        issue_e(h + 2);
                    } else {
                        if (b == 0) issue_q(0);
                        issue_k(b);
                    }
                }
            }
            // ---- phase 2: S_h = Q_h K_h^T; dQ_{h-1} = ds_{h-1} K_{h-1} right after it
            for (int h = 0; h <= H; ++h) {   // h == H only issues dQ_{H-1}
                const uint32_t ph = (uint32_t)(ph0 + h);
                if (h < H) {
                    const int b = h & 1;
                    bool ok = wait_bar(&bars[kQBarQ], (uint32_t)h & 1, abort_flag);
                    ok = wait_bar(&bars[kQBarK + b], (uint32_t)(h >> 1) & 1, abort_flag) && ok;
                    if (ph >= 1) ok = wait_bar(&bars[kQBarXFree], (ph - 1) & 1, abort_flag) && ok;
                    ptx::tc_fence_after();
                    if (ok) {
                        const uint32_t qa = ptx::smem_u32(sm + L.rq);
                        const uint32_t ka = ptx::smem_u32(sm + (b ? L.r1 : L.r0));
#pragma unroll
                        for (int k = 0; k < D / 16; ++k) {
                            const uint64_t ad = ptx::smem_desc_sw128(qa + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024);
                            const uint64_t bd = ptx::smem_desc_sw128(ka + (k >> 2) * span * 128 + (k & 3) * 32, 16, 1024);
                            ptx::mma_bf16(tmem, ad, bd, id_x, k > 0);
                        }
                    }
                    ptx::mma_commit(&bars[kQBarXFull]);
                }
                if (h >= 1 && do_dq) mma_dq(h - 1);
                if (h < H) {
                    // refill: Q_{h+1} once S_h has read Q; K_{h+1} once dQ_{h-1} (or, with no dQ,
                    // S_{h-1}, which completed before S_h) has read K_{h-1}
                    const bool s_done = wait_bar(&bars[kQBarXFull], ph & 1, abort_flag);
                    if (s_done && h + 1 < H) issue_q(h + 1);
                    if (h >= 1 && h + 1 < H &&
                        (do_dq ? wait_bar(&bars[kQBarDqFull + ((h - 1) & 1)], (uint32_t)((h - 1) >> 1) & 1, abort_flag)
                               : s_done))
                        issue_k(h + 1);
                }
                if (h >= 1 && do_dq) ds_released();   // after the refills: they must not wait on it
            }
            if constexpr (DST) ptx::bulk_wait_all();   // the ds tiles have reached global memory
        }
        __syncwarp();
    } else {
        regs_compute();
        // ---------------------------------------------------------------- compute warps
        const int q = warp & 3, split = warp >> 2;
        const int i = 32 * q + lane;
        const int64_t t = t0 + i;
        const bool valid = (i < BM) && (t < s.N);
        int clo = 1, chi = 0;
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
        const Band bd = make_band(q, split, BM, W, span, off);
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        const uint32_t x_cols = tmem + lane_base;
        const float sl2 = s.scale * kLog2e;
        // g (phase 1), lse and c (phase 2) of this row are read once per head.  A first
        // read that misses L2 costs microseconds while every CTA streams its tiles, so the
        // rows are brought into L2 now and each head's value is loaded one head ahead.
        if (valid && split == 0) {
            ptx::prefetch_l2(a.g + t * H);
            ptx::prefetch_l2(a.g + t * H + H - 1);
            ptx::prefetch_l2(a.lse + t * H);
            ptx::prefetch_l2(a.lse + t * H + H - 1);
            ptx::prefetch_l2(a.c + t * H);
            ptx::prefetch_l2(a.c + t * H + H - 1);
        }
        float g_next = (valid && do_p1) ? __ldg(a.g + t * H) : 0.f;
        // head 0's phase-2 values, loaded now: at the start of phase 2 the memory system is
        // at its busiest and a load issued there can take microseconds
        float lse_next = valid ? __ldg(a.lse + t * H) : 0.f;
        float c_next = valid ? __ldg(a.c + t * H) : 0.f;
        // column c is in this row's window iff (unsigned)(c - win_lo) <= win_n (never for a row
        // with an empty window)
        const uint32_t win_lo = (chi >= clo) ? (uint32_t)clo : ~0u;
        const uint32_t win_n = (chi >= clo) ? (uint32_t)(chi - clo) : 0u;
        // ds band row of this query for head h, from the first column of this thread's part of
        // the band: tile column c = c_first + k is element dsrow + k (kDsbRow - 1) (key
        // j = kbase + c, offset t - j = i + W - 1 - c)
        uint16_t *dsrow = nullptr;
        if constexpr (DSB) {
            const int c_first = bd.cb + bd.c0 * 8;
            dsrow = (uint16_t *)a.dsb + (kbase + c_first) * kDsbRow + (i + W - 1 - c_first);
        }

        // P(t, c) = pmap[t][c - i - off] on this thread's band, from the CTA's pmap rows staged by
        // the producer; zero outside the window.  Kept in registers (bf16 pairs) for all heads.
        // A segment reads its columns of the row from global memory.
        uint32_t pvp[MAXC][4];
        if constexpr (SEG) {
            const uint16_t *prow = (const uint16_t *)a.pmap + t * a.seg.wrow + a.seg.wofs - i;   // prow[c], c in window
#pragma unroll
            for (int cc = 0; cc < MAXC; ++cc) {
                if (cc < bd.mync) {
                    const int col = bd.cb + (bd.c0 + cc) * 8;
#pragma unroll
                    for (int e = 0; e < 8; e += 2) {
                        const int c0 = col + e, c1 = c0 + 1;
                        const uint32_t lo = (do_p1 && c0 >= clo && c0 <= chi) ? __ldg(prow + c0) : 0u;
                        const uint32_t hi = (do_p1 && c1 >= clo && c1 <= chi) ? __ldg(prow + c1) : 0u;
                        pvp[cc][e >> 1] = lo | (hi << 16);
                    }
                }
            }
        } else {
            const uint16_t *prow = (const uint16_t *)(sm + L.rd + 32768) + i * W - i - off;
            wait_bar(&bars[kQBarPmap], 0, abort_flag);
#pragma unroll
            for (int cc = 0; cc < MAXC; ++cc) {
                if (cc < bd.mync) {
                    const int col = bd.cb + (bd.c0 + cc) * 8;
#pragma unroll
                    for (int e = 0; e < 8; e += 2) {
                        const int c0 = col + e, c1 = c0 + 1;
                        const uint32_t lo = (c0 >= clo && c0 <= chi) ? prow[c0] : 0u;
                        const uint32_t hi = (c1 >= clo && c1 <= chi) ? prow[c1] : 0u;
                        pvp[cc][e >> 1] = lo | (hi << 16);
                    }
                }
            }
        }
        float dP[MAXC][8];
#pragma unroll
        for (int cc = 0; cc < MAXC; ++cc)
#pragma unroll
            for (int e = 0; e < 8; ++e) dP[cc][e] = 0.f;
        if (SEG && !do_p1) {   // dP from the band the first far-segment launch wrote
            const float *brow = a.band + t * a.seg.wrow + a.seg.wofs - i;   // brow[c], c in window
#pragma unroll
            for (int cc = 0; cc < MAXC; ++cc) {
                if (cc < bd.mync) {
                    const int col = bd.cb + (bd.c0 + cc) * 8;
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int cidx = col + e;
                        if (cidx >= clo && cidx <= chi) dP[cc][e] = __ldg(brow + cidx);
                    }
                }
            }
        }

        // ---- phase 1: dP and dg, three chunks of E_h per TMEM round trip.  dP is left
        // unmasked: outside the window it only ever meets p = 0 (and the key side reads
        // the band inside the window only); P is zero there, so dg needs no mask either.
        for (int h = 0; h < (do_p1 ? H : 0); ++h) {
            const float gh = g_next;
            if (h + 1 < H) g_next = valid ? __ldg(a.g + t * H + h + 1) : 0.f;
            wait_bar(&bars[kQBarXFull], (uint32_t)h & 1, abort_flag);
            ptx::tc_fence_after();
            float dga = 0.f, dgb = 0.f;
            constexpr int G = 3;
#pragma unroll
            for (int g0 = 0; g0 < MAXC; g0 += G) {
                uint32_t er[G][8];
#pragma unroll
                for (int gi = 0; gi < G; ++gi) {
                    const int cc = g0 + gi;
                    if (cc < MAXC && cc < bd.mync) ptx::tmem_ld8_issue(x_cols + bd.cb + (bd.c0 + cc) * 8, er[gi]);
                }
                ptx::tmem_wait_ld();
#pragma unroll
                for (int gi = 0; gi < G; ++gi) {
                    const int cc = g0 + gi;
                    if (cc < MAXC && cc < bd.mync) {
                        ptx::reg_fence8(er[gi]);
#pragma unroll
                        for (int e = 0; e < 8; e += 2) {
                            const float e0 = __uint_as_float(er[gi][e]), e1 = __uint_as_float(er[gi][e + 1]);
                            dP[cc][e] = fmaf(gh, e0, dP[cc][e]);
                            dP[cc][e + 1] = fmaf(gh, e1, dP[cc][e + 1]);
                            dga = fmaf(__uint_as_float(pvp[cc][e >> 1] << 16), e0, dga);
                            dgb = fmaf(__uint_as_float(pvp[cc][e >> 1] & 0xFFFF0000u), e1, dgb);
                        }
                    }
                }
            }
            const float dgp = dga + dgb;
            ptx::tc_fence_before();
            ptx::mbar_arrive(&bars[kQBarXFree]);
            float *rd = red + (h & 1) * (kSplits * 128);
            rd[split * 128 + i] = dgp;
            pair_sync(q);
            if (split == 0 && valid) {
                float sum = rd[i];
#pragma unroll
                for (int sp = 1; sp < kSplits; ++sp) sum += rd[sp * 128 + i];
                if constexpr (SEG) {   // the near segment completes the far segment's partial sum
                    if (a.seg.mode == kQSegNear) sum += a.dg[t * H + h];
                }
                a.dg[t * H + h] = sum;
            }
        }
        // every compute warp has finished phase 1 (and its reads of the staged pmap)
        compute_sync();
        // dP band: band[t][w] = dP(t, t - W + 1 + w) = tile column i + w.  The CTA's rows
        // are one contiguous [BM][W] block of the band: stage it in the ds tile region
        // (free: every E MMA has completed) and write it with one bulk copy.  The row
        // stride W - 1 between lanes is odd for the usual even W, so the staging stores
        // do not conflict.  A segment owns only columns wofs .. wofs + W - 1 of each row: plain
        // stores.
        if constexpr (SEG) {
            if (do_p1 && valid) {
                float *brow = a.band + t * a.seg.wrow + a.seg.wofs;   // brow[w], w < W
#pragma unroll
                for (int cc = 0; cc < MAXC; ++cc) {
                    if (cc < bd.mync) {
                        const int col = bd.cb + (bd.c0 + cc) * 8;
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const uint32_t w = (uint32_t)(col + e - i);
                            if (w < (uint32_t)W) brow[w] = dP[cc][e];
                        }
                    }
                }
            }
        } else if constexpr (!DSB && !DST) {   // (with the ds band or tiles the key side needs no dP)
            float *stage = (float *)(sm + L.rd);
            if (i < BM) {
#pragma unroll
                for (int cc = 0; cc < MAXC; ++cc) {
                    if (cc < bd.mync) {
                        const int col = bd.cb + (bd.c0 + cc) * 8;
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int w = col + e - i;
                            if (w >= 0 && w < W) stage[i * W + w] = dP[cc][e];
                        }
                    }
                }
            }
            ptx::fence_proxy_async_smem();
            compute_sync();
            if (threadIdx.x == 0) stage_out(a.band + t0 * W, stage, (uint32_t)(min((int64_t)BM, s.N - t0) * W * 4));
        }

        // ---- phase 2.  The ds tile region held dO, the pmap rows and the dP band; the band
        // copy reads it while head 0's scores are processed, and it is reused from head 0's
        // ds tile on (columns outside this quarter's band zeroed once).
        uint8_t *dtile = sm + L.rd;
        auto drain_dq = [&](int h) {
            const int b = h & 1;
            wait_bar(&bars[kQBarDqFull + b], (uint32_t)(h >> 1) & 1, abort_flag);
            ptx::tc_fence_after();
            if (SEG && a.seg.mode == kQSegFarPart2)   // adds the far segment's share to dq
                drain_row<D, true>(tmem + lane_base + 256 + 128 * b, a.dq + t * s.sdq + h * D, s.scale, valid, split,
                                   (((uintptr_t)a.dq | (uintptr_t)(s.sdq * 2)) & 31) == 0);
            else
                drain_row<D>(tmem + lane_base + 256 + 128 * b, a.dq + t * s.sdq + h * D, s.scale, valid, split,
                             (((uintptr_t)a.dq | (uintptr_t)(s.sdq * 2)) & 31) == 0);
            ptx::tc_fence_before();
            ptx::mbar_arrive(&bars[kQBarDqFree + b]);
        };
        for (int h = 0; h <= (do_dq ? H : H - 1); ++h) {   // h == H only drains dQ_{H-1}
            if (h < H) {
                const uint32_t ph = (uint32_t)(ph0 + h);
                const float lse2 = lse_next * kLog2e;
                const float ch = c_next;
                if (h + 1 < H) {
                    lse_next = valid ? __ldg(a.lse + t * H + h + 1) : 0.f;
                    c_next = valid ? __ldg(a.c + t * H + h + 1) : 0.f;
                }
                wait_bar(&bars[kQBarXFull], ph & 1, abort_flag);
                ptx::tc_fence_after();
                // p_h and dc_h, the band of S_h in two TMEM round trips
                float dca = 0.f, dcb = 0.f;   // two independent chains
                uint32_t pp[MAXC][4];   // p_h as packed bf16 pairs
                constexpr int G2 = (MAXC + 1) / 2;
#pragma unroll
                for (int g0 = 0; g0 < MAXC; g0 += G2) {
                    uint32_t xr[G2][8];
#pragma unroll
                    for (int gi = 0; gi < G2; ++gi) {
                        const int cc = g0 + gi;
                        if (cc < MAXC && cc < bd.mync) ptx::tmem_ld8_issue(x_cols + bd.cb + (bd.c0 + cc) * 8, xr[gi]);
                    }
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int gi = 0; gi < G2; ++gi) {
                        const int cc = g0 + gi;
                        if (cc < MAXC && cc < bd.mync) {
                            ptx::reg_fence8(xr[gi]);
                            const int col = bd.cb + (bd.c0 + cc) * 8;
                            float p[8];
#pragma unroll
                            for (int e = 0; e < 8; ++e) {
                                const int cidx = col + e;
                                p[e] = (cidx >= clo && cidx <= chi) ? ex2(__uint_as_float(xr[gi][e]) * sl2 - lse2) : 0.f;
                                if (e & 1) dcb = fmaf(dP[cc][e], p[e], dcb);
                                else dca = fmaf(dP[cc][e], p[e], dca);
                            }
#pragma unroll
                            for (int e = 0; e < 4; ++e) pp[cc][e] = pack_bf16x2(p[2 * e], p[2 * e + 1]);
                        }
                    }
                }
                ptx::tc_fence_before();
                ptx::mbar_arrive(&bars[kQBarXFree]);
                float dch;
                if (SEG && a.seg.mode == kQSegFarPart2) {   // dc is complete: the near launch wrote it
                    dch = valid ? a.dc[t * H + h] : 0.f;
                } else {
                    // the near segment adds the far segment's partial dc (read before any split
                    // of this row writes the sum)
                    const float dc_far = (SEG && a.seg.mode == kQSegNear && valid) ? a.dc[t * H + h] : 0.f;
                    float *rd = red + (ph & 1) * (kSplits * 128);
                    rd[split * 128 + i] = dca + dcb;
                    pair_sync(q);
                    dch = rd[i];
#pragma unroll
                    for (int sp = 1; sp < kSplits; ++sp) dch += rd[sp * 128 + i];
                    if constexpr (SEG) dch += dc_far;
                    if (split == 0 && valid) a.dc[t * H + h] = dch;
                }
                if (!do_dq) continue;   // the first far-segment launch stops at dc
                // the previous head's dQ MMA has been running meanwhile; once it has completed the
                // ds tile is free for this head (its accumulator is drained after the tile is handed on)
                if (h >= 1) {
                    wait_bar(&bars[kQBarDqFull + ((h - 1) & 1)], (uint32_t)((h - 1) >> 1) & 1, abort_flag);
                    if constexpr (DST) wait_bar(&bars[kQBarDsRead], (uint32_t)(h - 1) & 1, abort_flag);
                } else {
                    if (!SEG && !DSB && !DST && threadIdx.x == 0) ptx::bulk_wait_read();   // the band copy has left the region
                    compute_sync();
                    zero_outside_band(dtile, i, split, bd, span);
                }
#pragma unroll
                for (int cc = 0; cc < MAXC; ++cc) {
                    if (cc < bd.mync) {
                        const int col = bd.cb + (bd.c0 + cc) * 8;
                        uint32_t w[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float p0 = __uint_as_float(pp[cc][e] << 16), p1 = __uint_as_float(pp[cc][e] & 0xFFFF0000u);
                            w[e] = pack_bf16x2(ch * p0 * (dP[cc][2 * e] - dch), ch * p1 * (dP[cc][2 * e + 1] - dch));
                        }
                        *(uint4 *)(dtile + sw128_offset(i, col)) = make_uint4(w[0], w[1], w[2], w[3]);
                        if constexpr (DSB) {
                            // ds_h(t, j) into the key-major band, dsb[h][j][t - j], for the columns in the
                            // row's window: for one column all lanes (consecutive t) write consecutive
                            // elements.  Column c of this row is element dsrow + c (kDsbRow - 1).
                            uint16_t *pc = dsrow + cc * 8 * (kDsbRow - 1);
                            const uint32_t c0 = (uint32_t)col - win_lo;
                            if (__all_sync(0xffffffffu, c0 <= win_n && c0 + 7 <= win_n)) {
#pragma unroll
                                for (int e = 0; e < 8; ++e) pc[e * (kDsbRow - 1)] = (uint16_t)(w[e >> 1] >> (16 * (e & 1)));
                            } else {
#pragma unroll
                                for (int e = 0; e < 8; ++e)
                                    if (c0 + e <= win_n) pc[e * (kDsbRow - 1)] = (uint16_t)(w[e >> 1] >> (16 * (e & 1)));
                            }
                        }
                    }
                }
                ptx::fence_proxy_async_smem();
                ptx::mbar_arrive(&bars[kQBarDs]);
                if constexpr (DSB) dsrow += s.N * kDsbRow;   // next head's band
            }
            if (h >= 1) drain_dq(h - 1);   // overlaps the dQ_h MMA (other accumulator buffer)
        }
    }

    if (threadIdx.x == 0) ptx::bulk_wait_all();   // the dP band copy has completed
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, 512);
    }
}

// --------------------------------------------------------------------------- key side
enum : int { kKBarLd = 0, kKBarScaled = 2, kKBarPt = 4, kKBarAccFull = 5, kKBarAccFree = 7, kKBarK = 9,
             kKBarXFull = 10, kKBarXFree = 11, kKBarDs = 12, kKBarPmap = 13, kKNumBars = 14 };

template <int D>
struct KSideLayout {
    uint32_t tile_s;   // dO or Q tile over the query span: D/64 boxes of span rows x 128 B
    uint32_t ra, rb0, rb1, rk, colv, bars, bytes, stage, stage_bytes;
    bool stage_in_b1;  // the pmap staging rows fit in buffer 1 + the K/V buffer (dO_0 can load early)
    __host__ __device__ KSideLayout(int span, int W) {
        tile_s = (uint32_t)(D / 64) * span * 128;
        ra = 0;                            // P^T tile (phase 1) / ds^T tile (phase 2): 64 KiB
        rb0 = 4u * 16384;                  // dO buffer 0 (phase 1) / Q buffer 0 (phase 2)
        rb1 = rb0 + tile_s;
        rk = rb1 + tile_s;                 // V_h (phase 1) / K_h (phase 2) of the key block
        colv = rk + 128u * D * 2;          // per-query vectors [2][3][256] fp32
        bars = colv + 2 * 3 * 256 * 4;
        bytes = bars + 512;
        stage_bytes = (uint32_t)span * W * 2;   // pmap rows of the query span, read once
        stage_in_b1 = tile_s + 128u * D * 2 >= stage_bytes;
        stage = stage_in_b1 ? rb1 : rb0;
    }
};

// Key side that recomputes ds^T from S^T (and reads dP from the band): used for window
// segments, and when the workspace cannot hold the ds band.
template <int D, int MAXC, bool SEG = false>
__global__ void __launch_bounds__(kThreads, 1)
bwd_key_seg_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
               const __grid_constant__ CUtensorMap map_do, const BwdArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const Shape &s = a.s;
    const int H = s.H, W = s.W, BK = a.BM, span = a.span;
    const KSideLayout<D> L(span, W);
    uint64_t *bars = (uint64_t *)(sm + L.bars);
    uint32_t *tmem_slot = (uint32_t *)(bars + 32);
    volatile int *abort_flag = (volatile int *)(tmem_slot + 1);
    float *colv = (float *)(sm + L.colv);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t j0 = (int64_t)blockIdx.x * BK;
    // first query of the span: a segment's queries start `shift` tokens after the key block
    const int64_t qbase = SEG ? j0 + a.seg.shift : j0;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kKNumBars; ++i) {
            const bool many = (i == kKBarScaled || i == kKBarScaled + 1 || i == kKBarPt || i == kKBarAccFree ||
                               i == kKBarAccFree + 1 || i == kKBarXFree || i == kKBarDs);
            ptx::mbar_init(&bars[i], many ? kComputeThreads : 1);
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
            // load sequence idx = 0 .. 2H-1 into buffers idx & 1: dO_idx for idx < H, Q_{idx-H} after
            auto issue_ld = [&](int idx) {
                const int b = idx & 1;
                uint8_t *dst = sm + (b ? L.rb1 : L.rb0);
                const CUtensorMap *map = idx < H ? &map_do : &map_q;
                const int h = idx < H ? idx : idx - H;
                ptx::mbar_arrive_expect_tx(&bars[kKBarLd + b], L.tile_s);
                for (int kb = 0; kb < D / 64; ++kb)
                    ptx::tma_load_2d(dst + kb * span * 128, map, h * D + kb * 64, (int)qbase, &bars[kKBarLd + b]);
            };
            auto issue_k = [&](int h) {
                ptx::mbar_arrive_expect_tx(&bars[kKBarK], 128u * D * 2);
                for (int kb = 0; kb < D / 64; ++kb)
                    ptx::tma_load_2d(sm + L.rk + kb * 16384, &map_k, h * D + kb * 64, (int)j0, &bars[kKBarK]);
            };
            const uint32_t id_acc = ptx::idesc_bf16_f32(128, D, 0, 1);     // dV, dK: B MN-major
            const uint32_t id_st = ptx::idesc_bf16_f32(128, span, 0, 0);   // S^T: [128 keys x span]
            const uint32_t ra = ptx::smem_u32(sm + L.ra);
            const uint32_t rk = ptx::smem_u32(sm + L.rk);
            // accumulator product number idx (dV_idx for idx < H, dK_{idx-H} after) into
            // buffer idx & 1: A = the tile in region A (P^T or ds^T), B = load buffer idx & 1
            // (g-scaled dO or Q), MN-major
            auto mma_acc = [&](int idx, bool ok) {
                const int b = idx & 1;
                const uint32_t n = (uint32_t)(idx >> 1);
                if (idx >= 2) ok = wait_bar(&bars[kKBarAccFree + b], (n - 1) & 1, abort_flag) && ok;
                ptx::tc_fence_after();
                if (ok) {
                    const uint32_t ba = ptx::smem_u32(sm + (b ? L.rb1 : L.rb0));
                    for (int k = 0; k < span / 16; ++k) {
                        const uint64_t ad = ptx::smem_desc_sw128(ra + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024);
                        const uint64_t bd2 = ptx::smem_desc_sw128(ba + k * 2048, span * 128, 1024);
                        ptx::mma_bf16(tmem + 256 + 128 * b, ad, bd2, id_acc, k > 0);
                    }
                }
                ptx::mma_commit(&bars[kKBarAccFull + b]);
            };
            // pmap rows j0 .. j0+span-1 (one contiguous run) into the staging area (a segment
            // reads its columns of the rows directly)
            if (!SEG)
                stage_in(sm + L.stage, a.pmap + j0 * W, (uint32_t)(min((int64_t)span, s.N - j0) * W * 2),
                         &bars[kKBarPmap]);
            if (SEG || L.stage_in_b1) issue_ld(0);   // buffer 0 does not overlap the pmap staging rows
            // ---- phase 1: dV_h = P^T (g_h dO_h)
            const bool pt_ok = wait_bar(&bars[kKBarPt], 0, abort_flag);   // staging area consumed
            if (!SEG && !L.stage_in_b1) issue_ld(0);
            issue_ld(1);   // dO_1, or Q_0 when H == 1 (there are 2H >= 2 loads)
            issue_k(0);
            for (int h = 0; h < H; ++h) {
                const int idx = h, b = idx & 1;
                const uint32_t n = (uint32_t)(idx >> 1);
                const bool ok = wait_bar(&bars[kKBarScaled + b], n & 1, abort_flag) && pt_ok;
                mma_acc(idx, ok);
                if (idx + 2 < 2 * H && wait_bar(&bars[kKBarAccFull + b], n & 1, abort_flag)) issue_ld(idx + 2);
            }
            // ---- phase 2: S^T_h = K_h Q_h^T, then dK_{h-1} = ds^T_{h-1} Q_{h-1}
            for (int h = 0; h <= H; ++h) {   // h == H only issues dK_{H-1}
                const int idx = H + h, b = idx & 1;
                if (h < H) {
                    bool ok = wait_bar(&bars[kKBarK], (uint32_t)h & 1, abort_flag);
                    ok = wait_bar(&bars[kKBarLd + b], (uint32_t)(idx >> 1) & 1, abort_flag) && ok;
                    if (h >= 1) ok = wait_bar(&bars[kKBarXFree], (uint32_t)(h - 1) & 1, abort_flag) && ok;
                    ptx::tc_fence_after();
                    if (ok) {
                        const uint32_t qa = ptx::smem_u32(sm + (b ? L.rb1 : L.rb0));
#pragma unroll
                        for (int k = 0; k < D / 16; ++k) {
                            const uint64_t ad = ptx::smem_desc_sw128(rk + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024);
                            const uint64_t bd2 = ptx::smem_desc_sw128(qa + (k >> 2) * span * 128 + (k & 3) * 32, 16, 1024);
                            ptx::mma_bf16(tmem, ad, bd2, id_st, k > 0);
                        }
                    }
                    ptx::mma_commit(&bars[kKBarXFull]);
                }
                if (h >= 1) mma_acc(idx - 1, wait_bar(&bars[kKBarDs], (uint32_t)(h - 1) & 1, abort_flag));
                if (h < H) {
                    // refill: K_{h+1} once S^T_h has read K; Q_{h+1} once dK_{h-1} has read Q_{h-1}
                    if (wait_bar(&bars[kKBarXFull], (uint32_t)h & 1, abort_flag) && h + 1 < H) issue_k(h + 1);
                    if (h >= 1 && idx + 1 < 2 * H &&
                        wait_bar(&bars[kKBarAccFull + ((idx - 1) & 1)], (uint32_t)((idx - 1) >> 1) & 1, abort_flag))
                        issue_ld(idx + 1);
                }
            }
        }
        __syncwarp();
    } else {
        regs_compute();
        // ---------------------------------------------------------------- compute warps
        const int tid = threadIdx.x;   // 0 .. 255
        const int q = warp & 3, split = warp >> 2;
        const int i = 32 * q + lane;                 // key row
        const int64_t j = j0 + i;
        const bool validk = (i < BK) && (j < s.N);
        int clo = 1, chi = 0;                         // query columns c (t = qbase + c) that see key j
        if (validk) {
            const int64_t dend = doc_end(s, j);
            if constexpr (SEG) {   // queries j + shift .. j + shift + W - 1 of j's document
                if (j + a.seg.shift <= dend - 1) {
                    clo = i;
                    int64_t hi = j + a.seg.shift + W - 1;
                    if (hi > dend - 1) hi = dend - 1;
                    chi = (int)(hi - qbase);
                }
            } else {
                clo = i;
                int64_t hi = j + W - 1;
                if (hi > dend - 1) hi = dend - 1;
                chi = (int)(hi - j0);
            }
        }
        // column c is in this row's window iff (unsigned)(c - span_lo) <= span_n; a row with an
        // empty window (clo > chi: past the block or past N) gets span_lo = ~0u, so no c passes
        const uint32_t span_lo = (chi >= clo) ? (uint32_t)clo : ~0u;
        const uint32_t span_n = (chi >= clo) ? (uint32_t)(chi - clo) : 0u;
        const Band bd = make_band(q, split, BK, W, span);
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        const float sl2 = s.scale * kLog2e;

        // ---- pmap rows j0 .. j0+span-1, staged by the producer
        const uint16_t *stage = (const uint16_t *)(sm + L.stage);
        if (!SEG) wait_bar(&bars[kKBarPmap], 0, abort_flag);
        // ---- P^T tile: P^T(i, c) = P(j0 + c, j0 + i) = pmap[j0 + c][i - c + W - 1]
        // (segment: P(qbase + c, j0 + i) = pmap[qbase + c][wofs + i - c + W - 1], from global memory)
        uint8_t *atile = sm + L.ra;
        if constexpr (SEG) {
            const uint16_t *pm = (const uint16_t *)a.pmap + qbase * a.seg.wrow + a.seg.wofs + i + W - 1;
#pragma unroll
            for (int cc = 0; cc < MAXC; ++cc) {
                if (cc < bd.mync) {
                    const int col = bd.cb + (bd.c0 + cc) * 8;
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 8; e += 2) {
                        const uint32_t c0 = (uint32_t)(col + e), c1 = c0 + 1;
                        const uint32_t v0 = (c0 - span_lo <= span_n) ? __ldg(pm + (int64_t)c0 * a.seg.wrow - (int)c0) : 0u;
                        const uint32_t v1 = (c1 - span_lo <= span_n) ? __ldg(pm + (int64_t)c1 * a.seg.wrow - (int)c1) : 0u;
                        w[e >> 1] = v0 | (v1 << 16);
                    }
                    *(uint4 *)(atile + sw128_offset(i, col)) = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
            zero_outside_band(atile, i, split, bd, span);
        } else {
#pragma unroll
            for (int cc = 0; cc < MAXC; ++cc) {
                if (cc < bd.mync) {
                    const int col = bd.cb + (bd.c0 + cc) * 8;
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 8; e += 2) {
                        const uint32_t c0 = (uint32_t)(col + e), c1 = c0 + 1;
                        const uint32_t v0 = (c0 - span_lo <= span_n) ? stage[c0 * W + (i - (int)c0 + W - 1)] : 0u;
                        const uint32_t v1 = (c1 - span_lo <= span_n) ? stage[c1 * W + (i - (int)c1 + W - 1)] : 0u;
                        w[e >> 1] = v0 | (v1 << 16);
                    }
                    *(uint4 *)(atile + sw128_offset(i, col)) = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
            zero_outside_band(atile, i, split, bd, span);
        }
        ptx::fence_proxy_async_smem();
        ptx::mbar_arrive(&bars[kKBarPt]);

        // Scale the rows of dO_h (buffer h & 1) by g[t, h] in place.  Eight threads
        // share one 128-byte row (one 16-byte chunk each), so every quarter warp
        // touches one row: no bank conflicts.  The g values of a thread's rows are
        // fetched together, before the wait for the tile.
        constexpr int kRowsPerPass = kComputeThreads / 8;
        constexpr int kPasses = (kBwdMaxSpan + kRowsPerPass - 1) / kRowsPerPass;
        auto scale_do = [&](int h) {
            const int b = h & 1;
            float gv[kPasses];
#pragma unroll
            for (int it = 0; it < kPasses; ++it) {
                const int r = (tid >> 3) + it * kRowsPerPass;
                gv[it] = (r < span && qbase + r < s.N) ? __ldg(a.g + (qbase + r) * H + h) : 0.f;
            }
            wait_bar(&bars[kKBarLd + b], (uint32_t)(h >> 1) & 1, abort_flag);
            uint8_t *tile = sm + (b ? L.rb1 : L.rb0);
#pragma unroll
            for (int kb = 0; kb < D / 64; ++kb) {
#pragma unroll
                for (int it = 0; it < kPasses; ++it) {
                    const int r = (tid >> 3) + it * kRowsPerPass;
                    if (r < span) {
                        uint4 *p = (uint4 *)(tile + kb * span * 128 + r * 128) + (tid & 7);
                        uint4 v = *p;
                        uint32_t *u = &v.x;
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float f0 = __uint_as_float(u[e] << 16) * gv[it];
                            const float f1 = __uint_as_float(u[e] & 0xFFFF0000u) * gv[it];
                            u[e] = pack_bf16x2(f0, f1);
                        }
                        *p = v;
                    }
                }
            }
            ptx::fence_proxy_async_smem();
            ptx::mbar_arrive(&bars[kKBarScaled + b]);
        };
        auto drain = [&](int idx, __nv_bfloat16 *out, int h, float mult) {
            const int b = idx & 1;
            wait_bar(&bars[kKBarAccFull + b], (uint32_t)(idx >> 1) & 1, abort_flag);
            ptx::tc_fence_after();
            if (SEG && a.seg.mode == kKSegAdd)   // a later segment adds its share
                drain_row<D, true>(tmem + lane_base + 256 + 128 * b, out + j * s.sdq + h * D, mult, validk, split,
                                   (((uintptr_t)out | (uintptr_t)(s.sdq * 2)) & 31) == 0);
            else
                drain_row<D>(tmem + lane_base + 256 + 128 * b, out + j * s.sdq + h * D, mult, validk, split,
                             (((uintptr_t)out | (uintptr_t)(s.sdq * 2)) & 31) == 0);
            ptx::tc_fence_before();
            ptx::mbar_arrive(&bars[kKBarAccFree + b]);
        };

        // Phase-2 inputs that phase 1 does not touch are fetched now, so that their loads run
        // during phase 1: dP(t, j) for this row's band from the query side's workspace, and
        // head 0's per-query vectors.
        float dPT[MAXC][8];
#pragma unroll
        for (int cc = 0; cc < MAXC; ++cc) {
            if (cc < bd.mync) {
                const int col = bd.cb + (bd.c0 + cc) * 8;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const uint32_t cidx = (uint32_t)(col + e);
                    if constexpr (SEG)
                        dPT[cc][e] = (cidx - span_lo <= span_n)
                                         ? __ldg(a.band + (qbase + (int)cidx) * a.seg.wrow + a.seg.wofs + (i - (int)cidx + W - 1))
                                         : 0.f;
                    else
                        dPT[cc][e] = (cidx - span_lo <= span_n)
                                         ? __ldg(a.band + (j0 + (int)cidx) * W + (i - (int)cidx + W - 1)) : 0.f;
                }
            }
        }
        // per-query vectors of head h in colv[h & 1]: [lse * log2e | c | dc], one query column
        // per thread (span <= 256 < kComputeThreads); head h+1's values are fetched while
        // head h is processed
        float nv0 = 0.f, nv1 = 0.f, nv2 = 0.f;
        auto fetch_colv = [&](int h) {
            const int64_t tq = qbase + tid;
            const bool ok = tid < span && tq < s.N;
            nv0 = ok ? __ldg(a.lse + tq * H + h) * kLog2e : 0.f;
            nv1 = ok ? __ldg(a.c + tq * H + h) : 0.f;
            nv2 = ok ? __ldg(a.dc_in + tq * H + h) : 0.f;
        };
        auto store_colv = [&](int h) {
            float *cv = colv + (h & 1) * 768;
            if (tid < 256) {
                cv[tid] = nv0;
                cv[256 + tid] = nv1;
                cv[512 + tid] = nv2;
            }
        };
        fetch_colv(0);
        store_colv(0);   // published by the first phase-2 compute_sync

        // ---- phase 1: dV (scaling dO_h runs ahead of draining dV_{h-1}; one copy of each)
        for (int h = 0; h <= H; ++h) {
            if (h < H) scale_do(h);
            if (h >= 1) drain(h - 1, a.dv, h - 1, 1.f);
        }

        // ---- phase 2: dK
        uint8_t *dtile = sm + L.ra;   // ds^T tile reuses the P^T region (every dV MMA has completed)
        for (int h = 0; h <= H; ++h) {   // h == H only drains dK_{H-1}
            if (h < H) {
                const float *cv = colv + (h & 1) * 768;
                compute_sync();   // colv[h & 1] written; every warp is done with head h - 1
                if (h + 1 < H) fetch_colv(h + 1);
                wait_bar(&bars[kKBarXFull], (uint32_t)h & 1, abort_flag);
                ptx::tc_fence_after();
                uint32_t dsp[MAXC][4];   // ds^T as packed bf16 pairs
                constexpr int G2 = (MAXC + 1) / 2;   // the band of S^T_h in two TMEM round trips
#pragma unroll
                for (int g0 = 0; g0 < MAXC; g0 += G2) {
                    uint32_t xr[G2][8];
#pragma unroll
                    for (int gi = 0; gi < G2; ++gi) {
                        const int cc = g0 + gi;
                        if (cc < MAXC && cc < bd.mync)
                            ptx::tmem_ld8_issue(tmem + lane_base + bd.cb + (bd.c0 + cc) * 8, xr[gi]);
                    }
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int gi = 0; gi < G2; ++gi) {
                        const int cc = g0 + gi;
                        if (cc < MAXC && cc < bd.mync) {
                            ptx::reg_fence8(xr[gi]);
                            const int col = bd.cb + (bd.c0 + cc) * 8;   // the same for every lane
                            float lv[8], cvv[8], dcv[8];
                            *(float4 *)&lv[0] = *(const float4 *)(cv + col);
                            *(float4 *)&lv[4] = *(const float4 *)(cv + col + 4);
                            *(float4 *)&cvv[0] = *(const float4 *)(cv + 256 + col);
                            *(float4 *)&cvv[4] = *(const float4 *)(cv + 256 + col + 4);
                            *(float4 *)&dcv[0] = *(const float4 *)(cv + 512 + col);
                            *(float4 *)&dcv[4] = *(const float4 *)(cv + 512 + col + 4);
#pragma unroll
                            for (int e = 0; e < 8; e += 2) {
                                float dsv[2];
#pragma unroll
                                for (int u = 0; u < 2; ++u) {
                                    const uint32_t cidx = (uint32_t)(col + e + u);
                                    const float p = ex2(__uint_as_float(xr[gi][e + u]) * sl2 - lv[e + u]);
                                    const float v = cvv[e + u] * p * (dPT[cc][e + u] - dcv[e + u]);
                                    dsv[u] = (cidx - span_lo <= span_n) ? v : 0.f;
                                }
                                dsp[cc][e >> 1] = pack_bf16x2(dsv[0], dsv[1]);
                            }
                        }
                    }
                }
                ptx::tc_fence_before();
                ptx::mbar_arrive(&bars[kKBarXFree]);
                // the previous head's dK MMA (running while this head's S^T was computed) must have
                // read the ds^T tile before it is overwritten; its accumulator is drained afterwards
                if (h >= 1)
                    wait_bar(&bars[kKBarAccFull + ((H + h - 1) & 1)], (uint32_t)((H + h - 1) >> 1) & 1, abort_flag);
#pragma unroll
                for (int cc = 0; cc < MAXC; ++cc) {
                    if (cc < bd.mync) {
                        const int col = bd.cb + (bd.c0 + cc) * 8;
                        *(uint4 *)(dtile + sw128_offset(i, col)) = make_uint4(dsp[cc][0], dsp[cc][1], dsp[cc][2], dsp[cc][3]);
                    }
                }
                ptx::fence_proxy_async_smem();
                ptx::mbar_arrive(&bars[kKBarDs]);
            }
            if (h >= 1) drain(H + h - 1, a.dk, h - 1, s.scale);   // overlaps the dK_h MMA
            if (h + 1 < H) store_colv(h + 1);
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, 512);
    }
}

// --------------------------------------------------------------------------- key side, ds from the band
// The query side wrote every ds_h(t, j) it used for dQ into the key-major band
// dsb[h][j][t - j] (bf16).  A key block's rows of it are one contiguous [BK][wp] run per
// head: one bulk copy brings them to shared memory, and each key row's band of ds^T is
// read from there.  No S^T product, no K tile, no dP band and no per-query vectors.
//   phase 1, per head: scale the dO_h rows by g_h in smem; MMA dV_h = P^T gdO_h.
//   phase 2, per head: ds^T_h tile from the staged rows; MMA dK_h = ds^T_h Q_h, drained
//            while the next head's tile is built.
enum : int { kDBarLd = 0, kDBarScaled = 2, kDBarPt = 4, kDBarAccFull = 5, kDBarAccFree = 7, kDBarDsIn = 9,
             kDBarDs = 10, kDBarPmap = 11, kDBarRowsRead = 12, kDNumBars = 13 };

template <int D>
struct DSideLayout {
    uint32_t tile_s;   // dO or Q tile over the query span: D/64 boxes of span rows x 128 B
    uint32_t ra, rb0, rb1, rs, bars, bytes, stage, stage_bytes;
    bool stage_in_b1;  // the pmap staging rows fit in buffer 1 (dO_0 can load early)
    __host__ __device__ DSideLayout(int span, int W, int BK, int wp) {
        tile_s = (uint32_t)(D / 64) * span * 128;
        ra = 0;                                  // P^T tile (phase 1) / ds^T tile (phase 2): 64 KiB
        rb0 = 4u * 16384;                        // dO buffer 0 (phase 1) / Q buffer 0 (phase 2)
        rb1 = rb0 + tile_s;
        rs = rb1 + tile_s;                       // ds rows of the key block [BK][wp] bf16
        bars = rs + (((uint32_t)BK * wp * 2 + 127) & ~127u);
        bytes = bars + 512;
        stage_bytes = (uint32_t)span * W * 2;    // pmap rows of the query span, read once
        stage_in_b1 = tile_s >= stage_bytes;
        stage = stage_in_b1 ? rb1 : rb0;         // else it spans buffers 0 and 1
    }
};

template <int D, int MAXC>
__global__ void __launch_bounds__(kThreads, 1)
bwd_key_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_do,
               const BwdArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const Shape &s = a.s;
    const int H = s.H, W = s.W, BK = a.BM, span = a.span;
    constexpr int wp = kDsbRow;
    const DSideLayout<D> L(span, W, BK, wp);
    uint64_t *bars = (uint64_t *)(sm + L.bars);
    uint32_t *tmem_slot = (uint32_t *)(bars + 32);
    volatile int *abort_flag = (volatile int *)(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t j0 = (int64_t)blockIdx.x * BK;
    const int rows_blk = (int)min((int64_t)BK, s.N - j0);   // key rows of this block

    if (threadIdx.x == 0) {
        for (int i = 0; i < kDNumBars; ++i) {
            const bool many = (i == kDBarScaled || i == kDBarScaled + 1 || i == kDBarPt || i == kDBarAccFree ||
                               i == kDBarAccFree + 1 || i == kDBarDs || i == kDBarRowsRead);
            ptx::mbar_init(&bars[i], many ? kComputeThreads : 1);
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
            // load sequence idx = 0 .. 2H-1 into buffers idx & 1: dO_idx for idx < H, Q_{idx-H} after
            auto issue_ld = [&](int idx) {
                const int b = idx & 1;
                uint8_t *dst = sm + (b ? L.rb1 : L.rb0);
                const CUtensorMap *map = idx < H ? &map_do : &map_q;
                const int h = idx < H ? idx : idx - H;
                ptx::mbar_arrive_expect_tx(&bars[kDBarLd + b], L.tile_s);
                for (int kb = 0; kb < D / 64; ++kb)
                    ptx::tma_load_2d(dst + kb * span * 128, map, h * D + kb * 64, (int)j0, &bars[kDBarLd + b]);
            };
            // the block's ds rows of head h (contiguous; wp * 2 is a multiple of 16 bytes)
            auto issue_ds = [&](int h) {
                stage_in(sm + L.rs, a.dsb + ((int64_t)h * s.N + j0) * wp, (uint32_t)rows_blk * wp * 2,
                         &bars[kDBarDsIn]);
            };
            const uint32_t id_acc = ptx::idesc_bf16_f32(128, D, 0, 1);     // dV, dK: B MN-major
            const uint32_t ra = ptx::smem_u32(sm + L.ra);
            // accumulator product number idx (dV_idx for idx < H, dK_{idx-H} after) into
            // buffer idx & 1: A = the tile in region A (P^T or ds^T), B = load buffer idx & 1
            // (g-scaled dO or Q), MN-major
            auto mma_acc = [&](int idx, bool ok) {
                const int b = idx & 1;
                const uint32_t n = (uint32_t)(idx >> 1);
                if (idx >= 2) ok = wait_bar(&bars[kDBarAccFree + b], (n - 1) & 1, abort_flag) && ok;
                ptx::tc_fence_after();
                if (ok) {
                    const uint32_t ba = ptx::smem_u32(sm + (b ? L.rb1 : L.rb0));
                    for (int k = 0; k < span / 16; ++k) {
                        const uint64_t ad = ptx::smem_desc_sw128(ra + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024);
                        const uint64_t bd2 = ptx::smem_desc_sw128(ba + k * 2048, span * 128, 1024);
                        ptx::mma_bf16(tmem + 256 + 128 * b, ad, bd2, id_acc, k > 0);
                    }
                }
                ptx::mma_commit(&bars[kDBarAccFull + b]);
            };
            // pmap rows j0 .. j0+span-1 (one contiguous run) into the staging area; head 0's ds rows
            stage_in(sm + L.stage, a.pmap + j0 * W, (uint32_t)(min((int64_t)span, s.N - j0) * W * 2),
                     &bars[kDBarPmap]);
            issue_ds(0);
            if (L.stage_in_b1) issue_ld(0);   // buffer 0 does not overlap the pmap staging rows
            // ---- phase 1: dV_h = P^T (g_h dO_h)
            const bool pt_ok = wait_bar(&bars[kDBarPt], 0, abort_flag);   // staging area consumed
            if (!L.stage_in_b1) issue_ld(0);
            issue_ld(1);   // dO_1, or Q_0 when H == 1 (there are 2H >= 2 loads)
            for (int h = 0; h < H; ++h) {
                const int idx = h, b = idx & 1;
                const uint32_t n = (uint32_t)(idx >> 1);
                const bool ok = wait_bar(&bars[kDBarScaled + b], n & 1, abort_flag) && pt_ok;
                mma_acc(idx, ok);
                if (idx + 2 < 2 * H && wait_bar(&bars[kDBarAccFull + b], n & 1, abort_flag)) issue_ld(idx + 2);
            }
            // ---- phase 2: dK_h = ds^T_h Q_h
            for (int h = 0; h < H; ++h) {
                const int idx = H + h, b = idx & 1;
                const uint32_t n = (uint32_t)(idx >> 1);
                // the next head's rows load as soon as this head's have been read into registers
                if (h + 1 < H && wait_bar(&bars[kDBarRowsRead], (uint32_t)h & 1, abort_flag)) issue_ds(h + 1);
                bool ok = wait_bar(&bars[kDBarDs], (uint32_t)h & 1, abort_flag);   // tile h written
                ok = wait_bar(&bars[kDBarLd + b], n & 1, abort_flag) && ok;        // Q_h
                mma_acc(idx, ok);
                if (idx + 2 < 2 * H && wait_bar(&bars[kDBarAccFull + b], n & 1, abort_flag)) issue_ld(idx + 2);
            }
        }
        __syncwarp();
    } else {
        regs_compute();
        // ---------------------------------------------------------------- compute warps
        const int tid = threadIdx.x;   // 0 .. 383
        const int q = warp & 3, split = warp >> 2;
        const int i = 32 * q + lane;                 // key row
        const int64_t j = j0 + i;
        const bool validk = (i < BK) && (j < s.N);
        int clo = 1, chi = 0;                         // query columns c (t = j0 + c) that see key j
        if (validk) {
            clo = i;
            const int64_t dend = doc_end(s, j);
            int64_t hi = j + W - 1;
            if (hi > dend - 1) hi = dend - 1;
            chi = (int)(hi - j0);
        }
        // column c is in this row's window iff (unsigned)(c - span_lo) <= span_n; a row with an
        // empty window (clo > chi: past the block or past N) gets span_lo = ~0u, so no c passes
        const uint32_t span_lo = (chi >= clo) ? (uint32_t)clo : ~0u;
        const uint32_t span_n = (chi >= clo) ? (uint32_t)(chi - clo) : 0u;
        const Band bd = make_band(q, split, BK, W, span);
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;

        // ---- P^T tile: P^T(i, c) = P(j0 + c, j0 + i) = pmap[j0 + c][i - c + W - 1]
        const uint16_t *stage = (const uint16_t *)(sm + L.stage);
        wait_bar(&bars[kDBarPmap], 0, abort_flag);
        uint8_t *atile = sm + L.ra;
#pragma unroll
        for (int cc = 0; cc < MAXC; ++cc) {
            if (cc < bd.mync) {
                const int col = bd.cb + (bd.c0 + cc) * 8;
                uint32_t w[4];
#pragma unroll
                for (int e = 0; e < 8; e += 2) {
                    const uint32_t c0 = (uint32_t)(col + e), c1 = c0 + 1;
                    const uint32_t v0 = (c0 - span_lo <= span_n) ? stage[c0 * W + (i - (int)c0 + W - 1)] : 0u;
                    const uint32_t v1 = (c1 - span_lo <= span_n) ? stage[c1 * W + (i - (int)c1 + W - 1)] : 0u;
                    w[e >> 1] = v0 | (v1 << 16);
                }
                *(uint4 *)(atile + sw128_offset(i, col)) = make_uint4(w[0], w[1], w[2], w[3]);
            }
        }
        zero_outside_band(atile, i, split, bd, span);
        ptx::fence_proxy_async_smem();
        ptx::mbar_arrive(&bars[kDBarPt]);

        // Scale the rows of dO_h (buffer h & 1) by g[t, h] in place.  Eight threads
        // share one 128-byte row (one 16-byte chunk each), so every quarter warp
        // touches one row: no bank conflicts.  The g values of a thread's rows are
        // fetched together, before the wait for the tile.
        constexpr int kRowsPerPass = kComputeThreads / 8;
        constexpr int kPasses = (kBwdMaxSpan + kRowsPerPass - 1) / kRowsPerPass;
        auto scale_do = [&](int h) {
            const int b = h & 1;
            float gv[kPasses];
#pragma unroll
            for (int it = 0; it < kPasses; ++it) {
                const int r = (tid >> 3) + it * kRowsPerPass;
                gv[it] = (r < span && j0 + r < s.N) ? __ldg(a.g + (j0 + r) * H + h) : 0.f;
            }
            wait_bar(&bars[kDBarLd + b], (uint32_t)(h >> 1) & 1, abort_flag);
            uint8_t *tile = sm + (b ? L.rb1 : L.rb0);
#pragma unroll
            for (int kb = 0; kb < D / 64; ++kb) {
#pragma unroll
                for (int it = 0; it < kPasses; ++it) {
                    const int r = (tid >> 3) + it * kRowsPerPass;
                    if (r < span) {
                        uint4 *p = (uint4 *)(tile + kb * span * 128 + r * 128) + (tid & 7);
                        uint4 v = *p;
                        uint32_t *u = &v.x;
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float f0 = __uint_as_float(u[e] << 16) * gv[it];
                            const float f1 = __uint_as_float(u[e] & 0xFFFF0000u) * gv[it];
                            u[e] = pack_bf16x2(f0, f1);
                        }
                        *p = v;
                    }
                }
            }
            ptx::fence_proxy_async_smem();
            ptx::mbar_arrive(&bars[kDBarScaled + b]);
        };
        auto drain = [&](int idx, __nv_bfloat16 *out, int h, float mult) {
            const int b = idx & 1;
            wait_bar(&bars[kDBarAccFull + b], (uint32_t)(idx >> 1) & 1, abort_flag);
            ptx::tc_fence_after();
            drain_row<D>(tmem + lane_base + 256 + 128 * b, out + j * s.sdq + h * D, mult, validk, split,
                         (((uintptr_t)out | (uintptr_t)(s.sdq * 2)) & 31) == 0);
            ptx::tc_fence_before();
            ptx::mbar_arrive(&bars[kDBarAccFree + b]);
        };

        // ---- phase 1: dV (scaling dO_h runs ahead of draining dV_{h-1}; one copy of each)
        for (int h = 0; h <= H; ++h) {
            if (h < H) scale_do(h);
            if (h >= 1) drain(h - 1, a.dv, h - 1, 1.f);
        }

        // ---- phase 2: dK.  ds^T(i, c) = ds(j0 + c, j0 + i) = dsb[h][j0 + i][c - i], row i of the
        // staged rows (stride wp); the tile reuses the P^T region (every dV MMA has completed).
        const uint16_t *dsr = (const uint16_t *)(sm + L.rs) + i * wp - i;   // dsr[c], c in window
        for (int h = 0; h <= H; ++h) {   // h == H only drains dK_{H-1}
            if (h < H) {
                wait_bar(&bars[kDBarDsIn], (uint32_t)h & 1, abort_flag);
                uint32_t dsp[MAXC][4];
#pragma unroll
                for (int cc = 0; cc < MAXC; ++cc) {
                    if (cc < bd.mync) {
                        const int col = bd.cb + (bd.c0 + cc) * 8;
#pragma unroll
                        for (int e = 0; e < 8; e += 2) {
                            const uint32_t c0 = (uint32_t)(col + e), c1 = c0 + 1;
                            const uint32_t v0 = (c0 - span_lo <= span_n) ? dsr[c0] : 0u;
                            const uint32_t v1 = (c1 - span_lo <= span_n) ? dsr[c1] : 0u;
                            dsp[cc][e >> 1] = v0 | (v1 << 16);
                        }
                    }
                }
                ptx::mbar_arrive(&bars[kDBarRowsRead]);   // the staged rows may be replaced
                // the previous head's dK MMA must have read the tile before it is overwritten
                if (h >= 1)
                    wait_bar(&bars[kDBarAccFull + ((H + h - 1) & 1)], (uint32_t)((H + h - 1) >> 1) & 1, abort_flag);
#pragma unroll
                for (int cc = 0; cc < MAXC; ++cc) {
                    if (cc < bd.mync) {
                        const int col = bd.cb + (bd.c0 + cc) * 8;
                        *(uint4 *)(atile + sw128_offset(i, col)) = make_uint4(dsp[cc][0], dsp[cc][1], dsp[cc][2], dsp[cc][3]);
                    }
                }
                ptx::fence_proxy_async_smem();
                ptx::mbar_arrive(&bars[kDBarDs]);
            }
            if (h >= 1) drain(H + h - 1, a.dk, h - 1, s.scale);   // overlaps the dK_h MMA
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, 512);
    }
}

// --------------------------------------------------------------------------- key side, ds tiles
// Key block [j0, j0 + BK) with BK the query side's BM; the queries that see its keys are
// t in [j0, j0 + 2 BK) (W - 1 <= BK): the rows of this block's ds tile and of the next
// block's.  In a query block's tile, column c is key t0 - BM + c, so the key block's keys
// are columns BK .. 2 BK - 1 of its own block's tile and columns 0 .. BK - 1 of the next
// block's: whole 64-column boxes for TMA.
//   phase 1, per head: scale the dO_h rows by g_h in smem; MMA dV_h = P^T gdO_h with
//            A = the P tile [span queries x 128 keys] (MN-major), built once from pmap.
//   phase 2, per head: four TMA boxes land ds_h(t, j) for the block's keys as a
//            [span queries x 128 keys] tile, which is A = ds^T_h (MN-major) as it is;
//            MMA dK_h = ds^T_h Q_h, drained while the next head's product runs.
// The compute warps build the P tile, scale dO and drain; they never touch ds.
enum : int { kTBarLd = 0, kTBarScaled = 2, kTBarPt = 4, kTBarAccFull = 5, kTBarAccFree = 7, kTBarDs = 9,
             kTBarPmap = 11, kTNumBars = 12 };

template <int D>
struct TSideLayout {
    uint32_t tile_a;   // P tile or ds^T tile: 2 boxes of 64 key columns x span rows
    uint32_t tile_s;   // dO or Q tile over the query span: D/64 boxes of span rows x 128 B
    uint32_t ra0, ra1, rb0, rb1, bars, bytes;
    __host__ __device__ TSideLayout(int span) {
        tile_a = 2u * (uint32_t)span * 128;
        tile_s = (uint32_t)(D / 64) * span * 128;
        ra0 = 0;                  // P tile (phase 1) / ds^T of odd heads (phase 2)
        ra1 = ra0 + tile_a;       // pmap rows of the query span (start) / ds^T of even heads
        rb0 = ra1 + tile_a;       // dO buffer 0 (phase 1) / Q buffer 0 (phase 2)
        rb1 = rb0 + tile_s;       // dO buffer 1 / Q buffer 1
        bars = rb1 + tile_s;
        bytes = bars + 512;
    }
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
bwd_key_dst_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_do,
                   const __grid_constant__ CUtensorMap map_ds, const BwdArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const Shape &s = a.s;
    const int H = s.H, W = s.W, BK = a.BM, span = a.span;   // span = 2 BK
    const TSideLayout<D> L(span);
    uint64_t *bars = (uint64_t *)(sm + L.bars);
    uint32_t *tmem_slot = (uint32_t *)(bars + 32);
    volatile int *abort_flag = (volatile int *)(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t j0 = (int64_t)blockIdx.x * BK;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kTNumBars; ++i) {
            const bool many = (i == kTBarScaled || i == kTBarScaled + 1 || i == kTBarPt || i == kTBarAccFree ||
                               i == kTBarAccFree + 1);
            ptx::mbar_init(&bars[i], many ? kComputeThreads : 1);
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
            // load sequence idx = 0 .. 2H-1 into buffers idx & 1: dO_idx for idx < H, Q_{idx-H} after
            auto issue_ld = [&](int idx) {
                const int b = idx & 1;
                uint8_t *dst = sm + (b ? L.rb1 : L.rb0);
                const CUtensorMap *map = idx < H ? &map_do : &map_q;
                const int h = idx < H ? idx : idx - H;
                ptx::mbar_arrive_expect_tx(&bars[kTBarLd + b], L.tile_s);
                for (int kb = 0; kb < D / 64; ++kb)
                    ptx::tma_load_2d(dst + kb * span * 128, map, h * D + kb * 64, (int)j0, &bars[kTBarLd + b]);
            };
            // ds^T_h: this block's tile, columns BK + 64 c (its rows -> tile rows 0 .. BK-1), and
            // the next block's, columns 64 c (-> tile rows BK .. 2 BK - 1); even heads into ra1,
            // odd heads into ra0.  Rows past N and columns past span arrive as zeros.
            auto issue_ds = [&](int h) {
                uint8_t *dst = sm + ((h & 1) ? L.ra0 : L.ra1);
                uint64_t *bar = &bars[kTBarDs + (h & 1)];
                ptx::mbar_arrive_expect_tx(bar, 4u * (uint32_t)BK * 128);
                for (int c = 0; c < 2; ++c) {
                    ptx::tma_load_3d(dst + c * span * 128, &map_ds, BK + 64 * c, (int)j0, h, bar);
                    ptx::tma_load_3d(dst + c * span * 128 + BK * 128, &map_ds, 64 * c, (int)(j0 + BK), h, bar);
                }
            };
            const uint32_t id_acc = ptx::idesc_bf16_f32(128, D, 1, 1);   // A and B MN-major
            // accumulator product idx (dV_idx for idx < H, dK_{idx-H} after) into TMEM buffer idx & 1:
            // A = the [span x 128] tile at abase, B = load buffer idx & 1 (g-scaled dO or Q)
            auto mma_acc = [&](int idx, uint32_t abase, bool ok) {
                const int b = idx & 1;
                const uint32_t n = (uint32_t)(idx >> 1);
                if (idx >= 2) ok = wait_bar(&bars[kTBarAccFree + b], (n - 1) & 1, abort_flag) && ok;
                ptx::tc_fence_after();
                if (ok) {
                    const uint32_t ba = ptx::smem_u32(sm + (b ? L.rb1 : L.rb0));
                    for (int k = 0; k < span / 16; ++k) {
                        const uint64_t ad = ptx::smem_desc_sw128(abase + k * 2048, span * 128, 1024);
                        const uint64_t bd2 = ptx::smem_desc_sw128(ba + k * 2048, span * 128, 1024);
                        ptx::mma_bf16(tmem + 256 + 128 * b, ad, bd2, id_acc, k > 0);
                    }
                }
                ptx::mma_commit(&bars[kTBarAccFull + b]);
            };
            // pmap rows j0 .. j0 + span - 1 (one contiguous run) into ra1; dO_0, dO_1 (or Q_0)
            stage_in(sm + L.ra1, a.pmap + j0 * W, (uint32_t)(min((int64_t)span, s.N - j0) * W * 2),
                     &bars[kTBarPmap]);
            issue_ld(0);
            issue_ld(1);   // dO_1, or Q_0 when H == 1 (there are 2H >= 2 loads)
            // ---- phase 1: dV_h = P^T (g_h dO_h)
            const bool pt_ok = wait_bar(&bars[kTBarPt], 0, abort_flag);   // P tile built, staging consumed
            if (pt_ok) issue_ds(0);
            const uint32_t pa = ptx::smem_u32(sm + L.ra0);
            for (int h = 0; h < H; ++h) {
                const int idx = h, b = idx & 1;
                const uint32_t n = (uint32_t)(idx >> 1);
                const bool ok = wait_bar(&bars[kTBarScaled + b], n & 1, abort_flag) && pt_ok;
                mma_acc(idx, pa, ok);
                if (wait_bar(&bars[kTBarAccFull + b], n & 1, abort_flag)) {
                    if (idx + 2 < 2 * H) issue_ld(idx + 2);
                    if (h == H - 1 && H >= 2) issue_ds(1);   // every dV MMA has read the P tile
                }
            }
            // ---- phase 2: dK_h = ds^T_h Q_h
            for (int h = 0; h < H; ++h) {
                const int idx = H + h, b = idx & 1;
                const uint32_t n = (uint32_t)(idx >> 1);
                bool ok = wait_bar(&bars[kTBarDs + (h & 1)], (uint32_t)(h >> 1) & 1, abort_flag);
                ok = wait_bar(&bars[kTBarLd + b], n & 1, abort_flag) && ok;   // Q_h
                mma_acc(idx, ptx::smem_u32(sm + ((h & 1) ? L.ra0 : L.ra1)), ok);
                if (wait_bar(&bars[kTBarAccFull + b], n & 1, abort_flag)) {   // operands read
                    if (h + 2 < H) issue_ds(h + 2);
                    if (idx + 2 < 2 * H) issue_ld(idx + 2);
                }
            }
        }
        __syncwarp();
    } else {
        regs_compute();
        // ---------------------------------------------------------------- compute warps
        const int tid = threadIdx.x;   // 0 .. 383
        const int q = warp & 3, split = warp >> 2;
        const int i = 32 * q + lane;                 // key row of the accumulators
        const int64_t j = j0 + i;
        const bool validk = (i < BK) && (j < s.N);
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;

        // ---- P tile: element (r, c) = P(j0 + r, j0 + c) = pmap[j0 + r][c - r + W - 1] for key
        // columns c < BK inside row r's window, else 0.  MN-major, 128-byte swizzle: column c
        // is in box c / 64, 16-byte chunk (c % 64) / 8 of row r, swizzled with r & 7.  Each
        // unit is one chunk: 8 consecutive keys of one query row, one 16-byte store.  The
        // lanes of a warp take consecutive rows of one chunk column: their staged reads are
        // W - 1 elements apart (spread over the banks) and their stores fill whole 128-byte
        // rows.
        wait_bar(&bars[kTBarPmap], 0, abort_flag);
        {
            const uint16_t *stage = (const uint16_t *)(sm + L.ra1);
            const int rows_q = (int)min((int64_t)span, s.N - j0);   // staged query rows
            uint8_t *ptile = sm + L.ra0;
            for (int u = tid; u < span * 16; u += kComputeThreads) {
                const int k = u / span, r = u - k * span;
                uint32_t w[4];
#pragma unroll
                for (int e = 0; e < 8; e += 2) {
                    const int c0 = k * 8 + e;
                    const uint32_t x0 = (uint32_t)(c0 - r + W - 1), x1 = x0 + 1;   // pmap columns
                    const bool row_ok = r < rows_q;
                    const uint32_t v0 = (row_ok && c0 < BK && x0 < (uint32_t)W) ? stage[r * W + (int)x0] : 0u;
                    const uint32_t v1 = (row_ok && c0 + 1 < BK && x1 < (uint32_t)W) ? stage[r * W + (int)x1] : 0u;
                    w[e >> 1] = v0 | (v1 << 16);
                }
                *(uint4 *)(ptile + (k >> 3) * (span * 128) + r * 128 + (((k & 7) ^ (r & 7)) << 4)) =
                    make_uint4(w[0], w[1], w[2], w[3]);
            }
        }
        ptx::fence_proxy_async_smem();
        ptx::mbar_arrive(&bars[kTBarPt]);

        // Scale the rows of dO_h (buffer h & 1) by g[t, h] in place.  Eight threads
        // share one 128-byte row (one 16-byte chunk each), so every quarter warp
        // touches one row: no bank conflicts.  The g values of a thread's rows are
        // loaded one head ahead (a load issued just before its use waits on L2).
        constexpr int kRowsPerPass = kComputeThreads / 8;
        constexpr int kPasses = (256 + kRowsPerPass - 1) / kRowsPerPass;
        float gnext[kPasses];
        auto load_g = [&](int h) {
#pragma unroll
            for (int it = 0; it < kPasses; ++it) {
                const int r = (tid >> 3) + it * kRowsPerPass;
                gnext[it] = (h < H && r < span && j0 + r < s.N) ? __ldg(a.g + (j0 + r) * H + h) : 0.f;
            }
        };
        load_g(0);
        auto scale_do = [&](int h) {
            const int b = h & 1;
            float gv[kPasses];
#pragma unroll
            for (int it = 0; it < kPasses; ++it) gv[it] = gnext[it];
            load_g(h + 1);
            wait_bar(&bars[kTBarLd + b], (uint32_t)(h >> 1) & 1, abort_flag);
            uint8_t *tile = sm + (b ? L.rb1 : L.rb0);
#pragma unroll
            for (int kb = 0; kb < D / 64; ++kb) {
#pragma unroll
                for (int it = 0; it < kPasses; ++it) {
                    const int r = (tid >> 3) + it * kRowsPerPass;
                    if (r < span) {
                        uint4 *p = (uint4 *)(tile + kb * span * 128 + r * 128) + (tid & 7);
                        uint4 v = *p;
                        uint32_t *u = &v.x;
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float f0 = __uint_as_float(u[e] << 16) * gv[it];
                            const float f1 = __uint_as_float(u[e] & 0xFFFF0000u) * gv[it];
                            u[e] = pack_bf16x2(f0, f1);
                        }
                        *p = v;
                    }
                }
            }
            ptx::fence_proxy_async_smem();
            ptx::mbar_arrive(&bars[kTBarScaled + b]);
        };
        auto drain = [&](int idx, __nv_bfloat16 *out, int h, float mult) {
            const int b = idx & 1;
            wait_bar(&bars[kTBarAccFull + b], (uint32_t)(idx >> 1) & 1, abort_flag);
            ptx::tc_fence_after();
            drain_row_once<D>(tmem + lane_base + 256 + 128 * b, out + j * s.sdq + h * D, mult, validk, split,
                              (((uintptr_t)out | (uintptr_t)(s.sdq * 2)) & 31) == 0);
            ptx::tc_fence_before();
            ptx::mbar_arrive(&bars[kTBarAccFree + b]);
        };

        // ---- phase 1: dV (scaling dO_h runs ahead of draining dV_{h-1}; one copy of each)
        for (int h = 0; h <= H; ++h) {
            if (h < H) scale_do(h);
            if (h >= 1) drain(h - 1, a.dv, h - 1, 1.f);
        }
        // ---- phase 2: dK, each head drained while the next head's product runs
        for (int h = 0; h < H; ++h) drain(H + h, a.dk, h, s.scale);
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, 512);
    }
}

}  // namespace tc
}  // namespace dc
