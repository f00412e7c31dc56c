// tc_bwd.cuh -- tcgen05 backward kernels of Lightweight DC attention (bf16 in,
// fp32 accumulate).  The gradients are the chain rule of
//   p_h = softmax(sigma q_h k_h^T) on the window, P = sum_h c_h p_h, o_h = g_h P v_h:
//   E_h = dO_h v_h^T, dP = sum_h g_h E_h, dg_h = sum_j P E_h, dc_h = sum_j dP p_h,
//   ds_h = c_h p_h (dP - dc_h), dq_h = sigma ds_h k_h, dk_h = sigma ds_h^T q_h,
//   dv_h = P^T (g_h dO_h).
//
// Query side (one CTA per block of BM query tokens, all heads):
//   phase 1, per head: MMA E_h = dO_h V_h^T -> TMEM; SIMT dP += g_h E_h
//            (registers), dg_h = sum_j P E_h with P from the forward's pmap;
//            dP is then stored as a band [N][W] in the workspace.
//   phase 2, per head: MMA S_h = Q_h K_h^T -> TMEM; SIMT p_h from lse,
//            dc_h = sum_j dP p_h, ds_h -> bf16 tile in smem; MMA dQ_h = ds_h K_h.
// Key side (one CTA per block of BK key tokens; the queries that see them span
// round16(BK + W - 1) rows starting at the block):
//   phase 1, per head: scale the dO_h rows by g_h in smem; MMA dV_h = P^T gdO_h
//            with P^T built once from pmap.
//   phase 2, per head: MMA S^T_h = K_h Q_h^T -> TMEM; SIMT ds^T from lse, c,
//            dc and the stored dP; MMA dK_h = ds^T_h Q_h.
// Same thread roles as the forward: warps 0-7 SIMT (two per TMEM lane
// quarter), warp 8 lane 0 issues TMA and MMA; every wait is bounded.
#pragma once

#include "tc_common.cuh"

namespace dc {
namespace tc {

constexpr int kBwdMaxSpan = 240;   // key/query tile rows, keeps both kernels within 227 KiB of smem

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
};

// --------------------------------------------------------------------------- query side
enum : int { kQBarLd = 0, kQBarQ = 2, kQBarK = 3, kQBarXFull = 5, kQBarXFree = 6, kQBarDs = 7, kQBarDqFull = 8,
             kQBarDqFree = 10, kQNumBars = 12 };

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
        bars = red + 2 * 2 * 128 * 4;
        bytes = bars + 512;
    }
};

template <int D, int MAXC>
__global__ void __launch_bounds__(kThreads, 1)
bwd_query_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                 const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_do,
                 const BwdArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const Shape &s = a.s;
    const int H = s.H, W = s.W, BM = a.BM, span = a.span;
    const QSideLayout<D> L(span);
    uint64_t *bars = (uint64_t *)(sm + L.bars);
    uint32_t *tmem_slot = (uint32_t *)(bars + 32);
    volatile int *abort_flag = (volatile int *)(tmem_slot + 1);
    float *red = (float *)(sm + L.red);   // [2 parity][2 split][128]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t0 = (int64_t)blockIdx.x * BM;
    const int64_t kbase = t0 - (W - 1);

    validate_seqlens(s);
    if (threadIdx.x == 0) {
        for (int i = 0; i < kQNumBars; ++i) {
            const bool many = (i == kQBarXFree || i == kQBarDs || i == kQBarDqFree || i == kQBarDqFree + 1);
            ptx::mbar_init(&bars[i], many ? kComputeThreads : 1);
        }
        *abort_flag = 0;
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

    if (warp == kProducerWarp) {
        if (lane == 0) {
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

            // ---- phase 1: E_h = dO_h V_h^T
            for (int h = 0; h < H && h < 2; ++h) issue_e(h);
            for (int h = 0; h < H; ++h) {
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
                if (h + 2 < H && wait_bar(&bars[kQBarXFull], (uint32_t)h & 1, abort_flag)) issue_e(h + 2);
            }
            // ---- phase 2: S_h = Q_h K_h^T, then dQ_h = ds_h K_h
            if (wait_bar(&bars[kQBarXFull], (uint32_t)(H - 1) & 1, abort_flag)) {   // all E MMAs done
                issue_q(0);
                for (int h = 0; h < H && h < 2; ++h) issue_k(h);
            }
            for (int h = 0; h < H; ++h) {
                const int b = h & 1;
                const uint32_t ph = (uint32_t)(H + h);
                bool ok = wait_bar(&bars[kQBarQ], (uint32_t)h & 1, abort_flag);
                ok = wait_bar(&bars[kQBarK + b], (uint32_t)(h >> 1) & 1, abort_flag) && ok;
                ok = wait_bar(&bars[kQBarXFree], (ph - 1) & 1, abort_flag) && ok;
                ptx::tc_fence_after();
                const uint32_t ka = ptx::smem_u32(sm + (b ? L.r1 : L.r0));
                if (ok) {
                    const uint32_t qa = ptx::smem_u32(sm + L.rq);
#pragma unroll
                    for (int k = 0; k < D / 16; ++k) {
                        const uint64_t ad = ptx::smem_desc_sw128(qa + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024);
                        const uint64_t bd = ptx::smem_desc_sw128(ka + (k >> 2) * span * 128 + (k & 3) * 32, 16, 1024);
                        ptx::mma_bf16(tmem, ad, bd, id_x, k > 0);
                    }
                }
                ptx::mma_commit(&bars[kQBarXFull]);
                if (wait_bar(&bars[kQBarXFull], ph & 1, abort_flag) && h + 1 < H) issue_q(h + 1);
                ok = wait_bar(&bars[kQBarDs], (uint32_t)h & 1, abort_flag);
                if (h >= 2) ok = wait_bar(&bars[kQBarDqFree + b], (uint32_t)((h >> 1) - 1) & 1, abort_flag) && ok;
                ptx::tc_fence_after();
                if (ok) {
                    const uint32_t dsa = ptx::smem_u32(sm + L.rd);
                    for (int k = 0; k < span / 16; ++k) {
                        const uint64_t ad = ptx::smem_desc_sw128(dsa + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024);
                        const uint64_t bd = ptx::smem_desc_sw128(ka + k * 2048, span * 128, 1024);
                        ptx::mma_bf16(tmem + 256 + 128 * b, ad, bd, id_dq, k > 0);
                    }
                }
                ptx::mma_commit(&bars[kQBarDqFull + b]);
                if (h + 2 < H && wait_bar(&bars[kQBarDqFull + b], (uint32_t)(h >> 1) & 1, abort_flag)) issue_k(h + 2);
            }
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- compute warps
        const int q = warp & 3, split = warp >> 2;
        const int i = 32 * q + lane;
        const int64_t t = t0 + i;
        const bool valid = (i < BM) && (t < s.N);
        int clo = 1, chi = 0;
        if (valid) {
            clo = (int)(window_lo(s, t) - kbase);
            chi = (int)(t - kbase);
        }
        const Band bd = make_band(q, split, BM, W, span);
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        const uint32_t x_cols = tmem + lane_base;
        const float sl2 = s.scale * kLog2e;

        // P(t, c) = pmap[t][c - i] for columns c in this row's window (re-read per head;
        // the CTA's pmap rows stay in L1)
        const uint16_t *prow = reinterpret_cast<const uint16_t *>(a.pmap) + t * W - i;
        float dP[MAXC][8];
#pragma unroll
        for (int cc = 0; cc < MAXC; ++cc)
#pragma unroll
            for (int e = 0; e < 8; ++e) dP[cc][e] = 0.f;

        // ---- phase 1: dP and dg
        for (int h = 0; h < H; ++h) {
            wait_bar(&bars[kQBarXFull], (uint32_t)h & 1, abort_flag);
            ptx::tc_fence_after();
            const float gh = valid ? __ldg(a.g + t * H + h) : 0.f;
            float dgp = 0.f;
#pragma unroll
            for (int cc = 0; cc < MAXC; ++cc) {
                if (cc < bd.mync) {
                    const int col = bd.cb + (bd.c0 + cc) * 8;
                    float E[8];
                    ptx::tmem_ld8(x_cols + col, E);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int cidx = col + e;
                        const bool in = cidx >= clo && cidx <= chi;
                        const float ev = in ? E[e] : 0.f;
                        const float pv = in ? __uint_as_float((uint32_t)__ldg(prow + cidx) << 16) : 0.f;
                        dP[cc][e] = fmaf(gh, ev, dP[cc][e]);
                        dgp = fmaf(pv, ev, dgp);
                    }
                }
            }
            ptx::tc_fence_before();
            ptx::mbar_arrive(&bars[kQBarXFree]);
            float *rd = red + (h & 1) * 256;
            rd[split * 128 + i] = dgp;
            pair_sync(q);
            if (split == 0 && valid) a.dg[t * H + h] = rd[i] + rd[128 + i];
        }
        // dP band: band[t][w] = dP(t, t - W + 1 + w), tile column i + w
        if (valid) {
            float *brow = a.band + t * W - i;
#pragma unroll
            for (int cc = 0; cc < MAXC; ++cc) {
                if (cc < bd.mync) {
                    const int col = bd.cb + (bd.c0 + cc) * 8;
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int cidx = col + e;
                        if (cidx >= i && cidx < i + W) brow[cidx] = dP[cc][e];
                    }
                }
            }
        }

        // ---- phase 2: the ds tile region held dO in phase 1; every E MMA has
        // completed (waited above), so zero its columns outside this quarter's band once.
        uint8_t *dtile = sm + L.rd;
        {
            const uint4 z4 = make_uint4(0, 0, 0, 0);
            const int ce = bd.cb + bd.nch * 8;
            if (split == 0) {
                for (int col = 0; col < bd.cb && col < span; col += 8) *(uint4 *)(dtile + sw128_offset(i, col)) = z4;
            } else {
                for (int col = (ce > bd.cb ? ce : bd.cb); col < span; col += 8)
                    *(uint4 *)(dtile + sw128_offset(i, col)) = z4;
            }
        }
        for (int h = 0; h < H; ++h) {
            const uint32_t ph = (uint32_t)(H + h);
            wait_bar(&bars[kQBarXFull], ph & 1, abort_flag);
            ptx::tc_fence_after();
            const float lse2 = valid ? __ldg(a.lse + t * H + h) * kLog2e : 0.f;
            // pass 1: p_h and dc_h; p is parked (bf16) in this thread's own slots of the
            // ds tile, whose previous contents the dQ MMA of head h-1 has finished reading
            float dcp = 0.f;
#pragma unroll
            for (int cc = 0; cc < MAXC; ++cc) {
                if (cc < bd.mync) {
                    const int col = bd.cb + (bd.c0 + cc) * 8;
                    float x[8];
                    ptx::tmem_ld8(x_cols + col, x);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int cidx = col + e;
                        const float p = (cidx >= clo && cidx <= chi) ? ex2(x[e] * sl2 - lse2) : 0.f;
                        x[e] = p;
                        dcp = fmaf(dP[cc][e], p, dcp);
                    }
                    *(uint4 *)(dtile + sw128_offset(i, col)) =
                        make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                                   pack_bf16x2(x[6], x[7]));
                }
            }
            ptx::tc_fence_before();
            ptx::mbar_arrive(&bars[kQBarXFree]);
            float *rd = red + (ph & 1) * 256;
            rd[split * 128 + i] = dcp;
            pair_sync(q);
            const float dch = rd[i] + rd[128 + i];
            if (split == 0 && valid) a.dc[t * H + h] = dch;
            const float ch = valid ? __ldg(a.c + t * H + h) : 0.f;
            // pass 2: ds_h = c_h p_h (dP - dc_h) over the parked p
#pragma unroll
            for (int cc = 0; cc < MAXC; ++cc) {
                if (cc < bd.mync) {
                    const int col = bd.cb + (bd.c0 + cc) * 8;
                    uint4 *slot = (uint4 *)(dtile + sw128_offset(i, col));
                    const uint4 pv = *slot;
                    const uint32_t pw[4] = {pv.x, pv.y, pv.z, pv.w};
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float p0 = __uint_as_float(pw[e] << 16), p1 = __uint_as_float(pw[e] & 0xFFFF0000u);
                        w[e] = pack_bf16x2(ch * p0 * (dP[cc][2 * e] - dch), ch * p1 * (dP[cc][2 * e + 1] - dch));
                    }
                    *slot = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
            ptx::fence_proxy_async_smem();
            ptx::mbar_arrive(&bars[kQBarDs]);

            // drain dQ_h (the next head rewrites the ds tile only after this MMA completed)
            const int b = h & 1;
            wait_bar(&bars[kQBarDqFull + b], (uint32_t)(h >> 1) & 1, abort_flag);
            ptx::tc_fence_after();
            const int cbase = split * (D / 2);
#pragma unroll
            for (int c16 = 0; c16 < D / 32; ++c16) {
                float u[16];
                ptx::tmem_ld16(tmem + lane_base + 256 + 128 * b + cbase + c16 * 16, u);
                if (valid) {
                    uint4 w0, w1;
                    const float sc = s.scale;
                    w0.x = pack_bf16x2(sc * u[0], sc * u[1]);
                    w0.y = pack_bf16x2(sc * u[2], sc * u[3]);
                    w0.z = pack_bf16x2(sc * u[4], sc * u[5]);
                    w0.w = pack_bf16x2(sc * u[6], sc * u[7]);
                    w1.x = pack_bf16x2(sc * u[8], sc * u[9]);
                    w1.y = pack_bf16x2(sc * u[10], sc * u[11]);
                    w1.z = pack_bf16x2(sc * u[12], sc * u[13]);
                    w1.w = pack_bf16x2(sc * u[14], sc * u[15]);
                    uint4 *dst = (uint4 *)(a.dq + (t * H + h) * D + cbase + c16 * 16);
                    dst[0] = w0;
                    dst[1] = w1;
                }
            }
            ptx::tc_fence_before();
            ptx::mbar_arrive(&bars[kQBarDqFree + b]);
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, 512);
    }
}

// --------------------------------------------------------------------------- key side
enum : int { kKBarLd = 0, kKBarScaled = 2, kKBarPt = 4, kKBarAccFull = 5, kKBarAccFree = 7, kKBarK = 9,
             kKBarXFull = 10, kKBarXFree = 11, kKBarDs = 12, kKNumBars = 13 };

template <int D>
struct KSideLayout {
    uint32_t tile_s;   // dO or Q tile over the query span: D/64 boxes of span rows x 128 B
    uint32_t ra, rb0, rb1, rk, colv, bars, bytes;
    __host__ __device__ KSideLayout(int span) {
        tile_s = (uint32_t)(D / 64) * span * 128;
        ra = 0;                            // P^T tile (phase 1) / ds^T tile (phase 2): 64 KiB
        rb0 = 4u * 16384;                  // dO buffer 0 (phase 1) / Q buffer 0 (phase 2)
        rb1 = rb0 + tile_s;
        rk = rb1 + tile_s;                 // K of the key block (phase 2)
        colv = rk + 128u * D * 2;          // per-query vectors [2][3][256] fp32
        bars = colv + 2 * 3 * 256 * 4;
        bytes = bars + 512;
    }
};

template <int D, int MAXC>
__global__ void __launch_bounds__(kThreads, 1)
bwd_key_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
               const __grid_constant__ CUtensorMap map_do, const BwdArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const Shape &s = a.s;
    const int H = s.H, W = s.W, BK = a.BM, span = a.span;
    const KSideLayout<D> L(span);
    uint64_t *bars = (uint64_t *)(sm + L.bars);
    uint32_t *tmem_slot = (uint32_t *)(bars + 32);
    volatile int *abort_flag = (volatile int *)(tmem_slot + 1);
    float *colv = (float *)(sm + L.colv);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t j0 = (int64_t)blockIdx.x * BK;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kKNumBars; ++i) {
            const bool many = (i == kKBarScaled || i == kKBarScaled + 1 || i == kKBarPt || i == kKBarAccFree ||
                               i == kKBarAccFree + 1 || i == kKBarXFree || i == kKBarDs);
            ptx::mbar_init(&bars[i], many ? kComputeThreads : 1);
        }
        *abort_flag = 0;
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

    if (warp == kProducerWarp) {
        if (lane == 0) {
            // load sequence a = 0 .. 2H-1 into buffers a & 1: dO_a for a < H, Q_{a-H} after
            auto issue_ld = [&](int idx) {
                const int b = idx & 1;
                uint8_t *dst = sm + (b ? L.rb1 : L.rb0);
                const CUtensorMap *map = idx < H ? &map_do : &map_q;
                const int h = idx < H ? idx : idx - H;
                ptx::mbar_arrive_expect_tx(&bars[kKBarLd + b], L.tile_s);
                for (int kb = 0; kb < D / 64; ++kb)
                    ptx::tma_load_2d(dst + kb * span * 128, map, h * D + kb * 64, (int)j0, &bars[kKBarLd + b]);
            };
            auto issue_k = [&](int h) {
                ptx::mbar_arrive_expect_tx(&bars[kKBarK], 128u * D * 2);
                for (int kb = 0; kb < D / 64; ++kb)
                    ptx::tma_load_2d(sm + L.rk + kb * 16384, &map_k, h * D + kb * 64, (int)j0, &bars[kKBarK]);
            };
            const uint32_t id_acc = ptx::idesc_bf16_f32(128, D, 0, 1);     // dV, dK: B MN-major
            const uint32_t id_st = ptx::idesc_bf16_f32(128, span, 0, 0);   // S^T: [128 keys x span]
            issue_ld(0);
            if (2 * H > 1) issue_ld(1);
            issue_k(0);
            // ---- phase 1: dV_h = P^T (g_h dO_h)
            bool pt_ok = wait_bar(&bars[kKBarPt], 0, abort_flag);
            const uint32_t ra = ptx::smem_u32(sm + L.ra);
            for (int h = 0; h < H; ++h) {
                const int idx = h, b = idx & 1;
                const uint32_t n = (uint32_t)(idx >> 1);
                bool ok = wait_bar(&bars[kKBarScaled + b], n & 1, abort_flag) && pt_ok;
                if (idx >= 2) ok = wait_bar(&bars[kKBarAccFree + b], (n - 1) & 1, abort_flag) && ok;
                ptx::tc_fence_after();
                if (ok) {
                    const uint32_t da = ptx::smem_u32(sm + (b ? L.rb1 : L.rb0));
                    for (int k = 0; k < span / 16; ++k) {
                        const uint64_t ad = ptx::smem_desc_sw128(ra + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024);
                        const uint64_t bd2 = ptx::smem_desc_sw128(da + k * 2048, span * 128, 1024);
                        ptx::mma_bf16(tmem + 256 + 128 * b, ad, bd2, id_acc, k > 0);
                    }
                }
                ptx::mma_commit(&bars[kKBarAccFull + b]);
                if (idx + 2 < 2 * H && wait_bar(&bars[kKBarAccFull + b], n & 1, abort_flag)) issue_ld(idx + 2);
            }
            // ---- phase 2: S^T_h = K_h Q_h^T, dK_h = ds^T_h Q_h
            for (int h = 0; h < H; ++h) {
                const int idx = H + h, b = idx & 1;
                const uint32_t n = (uint32_t)(idx >> 1);
                bool ok = wait_bar(&bars[kKBarK], (uint32_t)h & 1, abort_flag);
                ok = wait_bar(&bars[kKBarLd + b], n & 1, abort_flag) && ok;
                if (h >= 1) ok = wait_bar(&bars[kKBarXFree], (uint32_t)(h - 1) & 1, abort_flag) && ok;
                ptx::tc_fence_after();
                const uint32_t qa = ptx::smem_u32(sm + (b ? L.rb1 : L.rb0));
                if (ok) {
                    const uint32_t ka = ptx::smem_u32(sm + L.rk);
#pragma unroll
                    for (int k = 0; k < D / 16; ++k) {
                        const uint64_t ad = ptx::smem_desc_sw128(ka + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024);
                        const uint64_t bd2 = ptx::smem_desc_sw128(qa + (k >> 2) * span * 128 + (k & 3) * 32, 16, 1024);
                        ptx::mma_bf16(tmem, ad, bd2, id_st, k > 0);
                    }
                }
                ptx::mma_commit(&bars[kKBarXFull]);
                if (wait_bar(&bars[kKBarXFull], (uint32_t)h & 1, abort_flag) && h + 1 < H) issue_k(h + 1);
                ok = wait_bar(&bars[kKBarDs], (uint32_t)h & 1, abort_flag);
                if (idx >= 2) ok = wait_bar(&bars[kKBarAccFree + b], (n - 1) & 1, abort_flag) && ok;
                ptx::tc_fence_after();
                if (ok) {
                    for (int k = 0; k < span / 16; ++k) {
                        const uint64_t ad = ptx::smem_desc_sw128(ra + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024);
                        const uint64_t bd2 = ptx::smem_desc_sw128(qa + k * 2048, span * 128, 1024);
                        ptx::mma_bf16(tmem + 256 + 128 * b, ad, bd2, id_acc, k > 0);
                    }
                }
                ptx::mma_commit(&bars[kKBarAccFull + b]);
                if (idx + 2 < 2 * H && wait_bar(&bars[kKBarAccFull + b], n & 1, abort_flag)) issue_ld(idx + 2);
            }
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- compute warps
        const int tid = threadIdx.x;   // 0 .. 255
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
        const Band bd = make_band(q, split, BK, W, span);
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        const float sl2 = s.scale * kLog2e;

        // ---- P^T tile: P^T(i, c) = P(j0 + c, j0 + i) = pmap[j0 + c][i - c + W - 1]
        uint8_t *atile = sm + L.ra;
        {
            const uint16_t *pm = reinterpret_cast<const uint16_t *>(a.pmap);
#pragma unroll
            for (int cc = 0; cc < MAXC; ++cc) {
                if (cc < bd.mync) {
                    const int col = bd.cb + (bd.c0 + cc) * 8;
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 8; e += 2) {
                        const int c0 = col + e, c1 = col + e + 1;
                        const uint32_t v0 =
                            (c0 >= clo && c0 <= chi) ? __ldg(pm + (j0 + c0) * W + (i - c0 + W - 1)) : 0u;
                        const uint32_t v1 =
                            (c1 >= clo && c1 <= chi) ? __ldg(pm + (j0 + c1) * W + (i - c1 + W - 1)) : 0u;
                        w[e >> 1] = v0 | (v1 << 16);
                    }
                    *(uint4 *)(atile + sw128_offset(i, col)) = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
            const uint4 z4 = make_uint4(0, 0, 0, 0);
            const int ce = bd.cb + bd.nch * 8;
            if (split == 0) {
                for (int col = 0; col < bd.cb && col < span; col += 8) *(uint4 *)(atile + sw128_offset(i, col)) = z4;
            } else {
                for (int col = (ce > bd.cb ? ce : bd.cb); col < span; col += 8)
                    *(uint4 *)(atile + sw128_offset(i, col)) = z4;
            }
        }
        ptx::fence_proxy_async_smem();
        ptx::mbar_arrive(&bars[kKBarPt]);

        // scale the rows of dO_h (buffer h & 1) by g[t, h] in place
        auto scale_do = [&](int h) {
            const int b = h & 1;
            wait_bar(&bars[kKBarLd + b], (uint32_t)(h >> 1) & 1, abort_flag);
            uint8_t *tile = sm + (b ? L.rb1 : L.rb0);
            const int rows = span * (D / 64);
            for (int hr = tid; hr < rows; hr += kComputeThreads) {
                const int r = hr % span;
                const int64_t tr = j0 + r;
                const float gv = (tr < s.N) ? __ldg(a.g + tr * H + h) : 0.f;
                uint4 *row = (uint4 *)(tile + (hr / span) * span * 128 + r * 128);
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    uint4 v = row[k];
                    uint32_t *u = &v.x;
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float f0 = __uint_as_float(u[e] << 16) * gv;
                        const float f1 = __uint_as_float(u[e] & 0xFFFF0000u) * gv;
                        u[e] = pack_bf16x2(f0, f1);
                    }
                    row[k] = v;
                }
            }
            ptx::fence_proxy_async_smem();
            ptx::mbar_arrive(&bars[kKBarScaled + b]);
        };
        auto drain = [&](int idx, __nv_bfloat16 *out, int h, float mult) {
            const int b = idx & 1;
            wait_bar(&bars[kKBarAccFull + b], (uint32_t)(idx >> 1) & 1, abort_flag);
            ptx::tc_fence_after();
            const int cbase = split * (D / 2);
#pragma unroll
            for (int c16 = 0; c16 < D / 32; ++c16) {
                float u[16];
                ptx::tmem_ld16(tmem + lane_base + 256 + 128 * b + cbase + c16 * 16, u);
                if (validk) {
                    uint4 w0, w1;
                    w0.x = pack_bf16x2(mult * u[0], mult * u[1]);
                    w0.y = pack_bf16x2(mult * u[2], mult * u[3]);
                    w0.z = pack_bf16x2(mult * u[4], mult * u[5]);
                    w0.w = pack_bf16x2(mult * u[6], mult * u[7]);
                    w1.x = pack_bf16x2(mult * u[8], mult * u[9]);
                    w1.y = pack_bf16x2(mult * u[10], mult * u[11]);
                    w1.z = pack_bf16x2(mult * u[12], mult * u[13]);
                    w1.w = pack_bf16x2(mult * u[14], mult * u[15]);
                    uint4 *dst = (uint4 *)(out + (j * H + h) * D + cbase + c16 * 16);
                    dst[0] = w0;
                    dst[1] = w1;
                }
            }
            ptx::tc_fence_before();
            ptx::mbar_arrive(&bars[kKBarAccFree + b]);
        };

        // ---- phase 1: dV
        scale_do(0);
        for (int h = 0; h < H; ++h) {
            if (h + 1 < H) scale_do(h + 1);
            drain(h, a.dv, h, 1.f);
        }

        // ---- phase 2: dK.  dP(t, j) for this row's band from the query side's workspace
        float dPT[MAXC][8];
#pragma unroll
        for (int cc = 0; cc < MAXC; ++cc) {
            if (cc < bd.mync) {
                const int col = bd.cb + (bd.c0 + cc) * 8;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int cidx = col + e;
                    dPT[cc][e] = (cidx >= clo && cidx <= chi) ? __ldg(a.band + (j0 + cidx) * W + (i - cidx + W - 1))
                                                             : 0.f;
                }
            }
        }
        uint8_t *dtile = sm + L.ra;   // ds^T tile reuses the P^T region (every dV MMA has completed)
        for (int h = 0; h < H; ++h) {
            float *cv = colv + (h & 1) * 768;   // [lse * log2e | c | dc] for query columns
            for (int cidx = tid; cidx < span; cidx += kComputeThreads) {
                const int64_t tq = j0 + cidx;
                const bool ok = tq < s.N;
                cv[cidx] = ok ? __ldg(a.lse + tq * H + h) * kLog2e : 0.f;
                cv[256 + cidx] = ok ? __ldg(a.c + tq * H + h) : 0.f;
                cv[512 + cidx] = ok ? __ldg(a.dc_in + tq * H + h) : 0.f;
            }
            compute_sync();
            wait_bar(&bars[kKBarXFull], (uint32_t)h & 1, abort_flag);
            ptx::tc_fence_after();
#pragma unroll
            for (int cc = 0; cc < MAXC; ++cc) {
                if (cc < bd.mync) {
                    const int col = bd.cb + (bd.c0 + cc) * 8;
                    float x[8];
                    ptx::tmem_ld8(tmem + lane_base + col, x);
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 8; e += 2) {
                        float dsv[2];
#pragma unroll
                        for (int u = 0; u < 2; ++u) {
                            const int cidx = col + e + u;
                            float v = 0.f;
                            if (cidx >= clo && cidx <= chi) {
                                const float p = ex2(x[e + u] * sl2 - cv[cidx]);
                                v = cv[256 + cidx] * p * (dPT[cc][e + u] - cv[512 + cidx]);
                            }
                            dsv[u] = v;
                        }
                        w[e >> 1] = pack_bf16x2(dsv[0], dsv[1]);
                    }
                    *(uint4 *)(dtile + sw128_offset(i, col)) = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
            ptx::tc_fence_before();
            ptx::mbar_arrive(&bars[kKBarXFree]);
            ptx::fence_proxy_async_smem();
            ptx::mbar_arrive(&bars[kKBarDs]);
            drain(H + h, a.dk, h, s.scale);
        }
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
