// cg_tc.cuh -- tensor-core forward of the c/g producer for bf16 x (tcgen05, TMA, TMEM).
//
// The producer's forward is the contraction [N x D] . [D x 2H] (form assumed, see cg.cuh).
// One CTA takes a tile of 128 tokens: TMA brings x in [128 tokens][64 columns] blocks
// (128-byte swizzle, K-major A operand), and the CTA's threads write the weight into shared
// memory as the K-major B operand: row n = split * R + o holds split `split` of
// weight[o][.], R = 16 (2H <= 16) or 32 outputs per split, zero for o >= 2H.  The three splits
// are the bf16 terms hi = bf16(w), mid = bf16(w - hi), lo = bf16(w - hi - mid), whose sum is w
// to within 2^-24 |w|, so every product x * split is exact in the fp32 accumulator and the
// result is the fp32 one up to the tensor core's accumulation.  D = 64-column blocks of
// 4 MMAs (M = 128, N = 3R, K = 16) each; the epilogue reads the three split sums of each
// output from TMEM and adds them, then the bias.
//
// Warps 0-3 read TMEM lane quarters 0-3 (one token per thread); warp 4 issues the TMA
// loads (a ring of as many 16 KB stages as shared memory holds, so that most of a tile's
// x is in flight at once); warp 5 allocates TMEM and issues the MMAs.  Every mbarrier
// wait is bounded (wait_bar): a wait that runs out raises DC_DEVERR_TIMEOUT and the CTA
// skips the rest of its work.
#pragma once

#include "cg.cuh"
#include "tc_common.cuh"

namespace dc {
namespace cg {

constexpr int kTcMaxStages = 12;
constexpr int kTcThreads = 192;
constexpr int kTcTile = 128;
constexpr size_t kTcFixed = 1024 + 512;   // base alignment slack; mbarriers, TMEM slot, control words

__host__ __device__ constexpr int tc_rows_per_split(int H) { return 2 * H <= 16 ? 16 : 32; }
__host__ __device__ inline size_t tc_split_bytes(int D, int H) {
    return (size_t)3 * tc_rows_per_split(H) * 128 * ((D + 63) / 64);
}
// Stages of the x ring: as many 16 KB stages as shared memory holds beside the weight
// splits (up to the tile's column blocks and kTcMaxStages); 0 if not even two fit.
inline int tc_stages(int D, int H, size_t smem_max) {
    const size_t w = tc_split_bytes(D, H) + kTcFixed;
    if (w + 2 * 16384 > smem_max) return 0;
    size_t st = (smem_max - w) / 16384;
    const size_t nkb = (size_t)(D + 63) / 64;
    if (st > nkb) st = nkb < 2 ? 2 : nkb;
    return (int)(st > (size_t)kTcMaxStages ? kTcMaxStages : st);
}
inline size_t tc_smem_bytes(int D, int H, int stages) { return kTcFixed + (size_t)stages * 16384 + tc_split_bytes(D, H); }

// The weight splits in the swizzled K-major layout: element (n, k) at byte
// (k / 64) * rows * 128 + n * 128 + (((k % 64) / 8) ^ (n % 8)) * 16 + (k % 8) * 2.
// Work item = (output o < R, 8-column chunk); each writes one 16-byte chunk in each split.
// A thread loads the weights of kBatch items before converting any, so their L2 round
// trips overlap.
constexpr int kBatch = 10;   // 16 outputs x 96 chunks (D = 768) over 160 threads in one round

__device__ __forceinline__ void split3(float v, uint32_t &h, uint32_t &m, uint32_t &l) {
    const __nv_bfloat16 hb = __float2bfloat16_rn(v);
    const float r1 = v - __bfloat162float(hb);   // exact
    const __nv_bfloat16 mb = __float2bfloat16_rn(r1);
    const float r2 = r1 - __bfloat162float(mb);  // exact
    h = __bfloat16_as_ushort(hb);
    m = __bfloat16_as_ushort(mb);
    l = __bfloat16_as_ushort(__float2bfloat16_rn(r2));
}

template <int R>
__device__ __forceinline__ void stage_weight_splits(const CgShape &s, const float *__restrict__ weight, uint8_t *wb,
                                                    int nkb, int tid, int nthreads) {
    constexpr int ROWS = 3 * R;
    const int chunks = nkb * 8;
    const int total = R * chunks;
    for (int i0 = tid; i0 < total; i0 += nthreads * kBatch) {
        float2 v[kBatch][4];
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
            const int i = i0 + b * nthreads;
            const int o = i / chunks, kc = i - o * chunks;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int k = kc * 8 + 2 * u;
                v[b][u] = (i < total && o < 2 * s.H && k < s.D)
                              ? __ldg(reinterpret_cast<const float2 *>(weight + (int64_t)o * s.D + k))
                              : make_float2(0.f, 0.f);
            }
        }
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
            const int i = i0 + b * nthreads;
            if (i >= total) break;
            const int o = i / chunks, kc = i - o * chunks;
            uint32_t w3[3][4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                uint32_t h0, m0, l0, h1, m1, l1;
                split3(v[b][u].x, h0, m0, l0);
                split3(v[b][u].y, h1, m1, l1);
                w3[0][u] = h0 | (h1 << 16);
                w3[1][u] = m0 | (m1 << 16);
                w3[2][u] = l0 | (l1 << 16);
            }
            const int kb = kc >> 3, c16 = kc & 7;
#pragma unroll
            for (int sp = 0; sp < 3; ++sp) {
                const int n = sp * R + o;
                *reinterpret_cast<uint4 *>(wb + kb * ROWS * 128 + n * 128 + ((c16 ^ (n & 7)) << 4)) =
                    make_uint4(w3[sp][0], w3[sp][1], w3[sp][2], w3[sp][3]);
            }
        }
    }
}

template <int R>
__global__ void __launch_bounds__(kTcThreads, 1)
cg_fwd_tc_kernel(const __grid_constant__ CUtensorMap map_x, CgShape s, const float *__restrict__ weight,
                 const uint8_t *__restrict__ splits, const float *__restrict__ bias, float *__restrict__ c,
                 float *__restrict__ g, int nst, uint32_t wait_ns) {
    constexpr int NCOL = 3 * R;                  // MMA N
    constexpr uint32_t TMEM_COLS = NCOL <= 64 ? 64 : 128;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int nkb = (s.D + 63) / 64;
    uint8_t *xs = sm;
    uint8_t *wb = sm + (size_t)nst * 16384;
    uint64_t *bars = (uint64_t *)(wb + (size_t)nkb * NCOL * 128);
    uint64_t *full = bars, *empty = bars + kTcMaxStages, *accfull = bars + 2 * kTcMaxStages;
    uint64_t *wready = accfull + 1;   // the prepared weight image has landed
    uint32_t *tmem_slot = (uint32_t *)(bars + 2 * kTcMaxStages + 2);
    volatile int *abort_flag = (volatile int *)(tmem_slot + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t0 = (int64_t)blockIdx.x * kTcTile;

    // The producer thread sets up the barriers and starts the x loads first; the other
    // threads meanwhile write the weight splits.
    const int first = nkb < nst ? nkb : nst;
    if (warp == 4 && lane == 0) {
        for (int i = 0; i < 2 * kTcMaxStages + 2; ++i) ptx::mbar_init(&bars[i], 1);
        tc::init_ctl(abort_flag, wait_ns);
        ptx::fence_mbar_init();
        ptx::prefetch_tensormap(&map_x);
        if (splits) {   // the weight image first (from L2; the MMAs need all of it), one bulk copy per block
            ptx::mbar_arrive_expect_tx(wready, (uint32_t)(nkb * NCOL * 128));
            for (int kb = 0; kb < nkb; ++kb)
                ptx::bulk_load(wb + kb * NCOL * 128, splits + (size_t)kb * NCOL * 128, NCOL * 128, wready);
        }
        for (int kb = 0; kb < first; ++kb) {
            ptx::mbar_arrive_expect_tx(&full[kb], 16384);
            ptx::tma_load_2d(xs + kb * 16384, &map_x, kb * 64, (int)t0, &full[kb]);
        }
    }
    if (warp == 5) {
        ptx::tmem_alloc(tmem_slot, TMEM_COLS);
        ptx::tmem_relinquish();
    }
    if (warp != 4 && !splits) {
        const int tid = warp < 4 ? threadIdx.x : threadIdx.x - 32;   // warps 0-3 and 5
        stage_weight_splits<R>(s, weight, wb, nkb, tid, kTcThreads - 32);
    }
    ptx::fence_proxy_async_smem();   // the tensor core reads the splits through the async proxy
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 4) {
        if (lane == 0) {
            for (int kb = first; kb < nkb; ++kb) {
                const int st = kb % nst;
                if (!tc::wait_bar(&empty[st], (uint32_t)((kb / nst - 1) & 1), abort_flag)) break;
                ptx::mbar_arrive_expect_tx(&full[st], 16384);
                ptx::tma_load_2d(xs + st * 16384, &map_x, kb * 64, (int)t0, &full[st]);
            }
        }
    } else if (warp == 5) {
        if (lane == 0) {
            const uint32_t idesc = ptx::idesc_bf16_f32(128, NCOL, 0, 0);
            bool ok = !splits || tc::wait_bar(wready, 0, abort_flag);
            for (int kb = 0; kb < nkb && ok; ++kb) {
                const int st = kb % nst;
                ok = tc::wait_bar(&full[st], (uint32_t)((kb / nst) & 1), abort_flag);
                if (!ok) break;
                ptx::tc_fence_after();
                const uint32_t xa = ptx::smem_u32(xs + st * 16384);
                const uint32_t wa = ptx::smem_u32(wb + (size_t)kb * NCOL * 128);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint64_t ad = ptx::smem_desc_sw128(xa + k * 32, 16, 1024);
                    const uint64_t bd = ptx::smem_desc_sw128(wa + k * 32, 16, 1024);
                    ptx::mma_bf16(tmem, ad, bd, idesc, (kb | k) != 0);
                }
                ptx::mma_commit(&empty[st]);
            }
            if (ok) ptx::mma_commit(accfull);
        }
    } else {
        // epilogue: warp w reads TMEM lanes 32w..32w+31, one token per thread
        const bool ok = tc::wait_bar(accfull, 0, abort_flag);
        ptx::tc_fence_after();
        if (ok) {
            const uint32_t base = tmem + ((uint32_t)(warp * 32) << 16);
            uint32_t r[NCOL / 16][16];
#pragma unroll
            for (int b = 0; b < NCOL / 16; ++b) ptx::tmem_ld16_issue(base + b * 16, r[b]);
            ptx::tmem_wait_ld();
            float acc[NCOL];
#pragma unroll
            for (int b = 0; b < NCOL / 16; ++b) {
                ptx::reg_fence16(r[b]);
#pragma unroll
                for (int e = 0; e < 16; ++e) acc[b * 16 + e] = __uint_as_float(r[b][e]);
            }
            const int64_t t = t0 + warp * 32 + lane;
            if (t < s.N) {
#pragma unroll
                for (int o = 0; o < R; ++o) {
                    if (o < 2 * s.H) {
                        const float hi = acc[o];
                        const float mid = acc[R + o];
                        const float lo = acc[2 * R + o];
                        const float v = ((hi + mid) + lo) + __ldg(bias + o);
                        if (o < s.H)
                            c[t * s.H + o] = v;
                        else
                            g[t * s.H + o - s.H] = v;
                    }
                }
            }
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, TMEM_COLS);
    }
}

// ---------------------------------------------------------------------------------------
// dx on the tensor cores (bf16 x and dx, 2H <= 16): dx[t, k] = sum_o e[t, o] weight[o][k] as
// D[128 tokens][k] = A[128][96] . B[96][k], with K = six 16-wide terms pairing the bf16 splits
// of e and of the weight: (e1, w1), (e1, w2), (e2, w1), (e1, w3), (e3, w1), (e2, w2).  The
// dropped products (e2 w3, e3 w2, e3 w3) and the two splits' residuals are below 2^-23 of
// |e w|.  A is K-major (the CTA's threads write each token's row); B is MN-major: the
// forward's split image (rows split * 16 + o, 64-column blocks of 48 x 128 bytes), K16 step j
// pointing at the 16 rows of the weight split it pairs with.  The
// columns go in chunks of up to 256 (6 MMAs each) into two alternating TMEM buffers, so the
// epilogue of one chunk (TMEM -> bf16 -> 32-byte stores of each token's row) overlaps the
// products of the next.
// ---------------------------------------------------------------------------------------

constexpr int kDxThreads = 288;    // warps 0-3: A rows and epilogue; 5-8: epilogue; warp 4: TMEM, MMAs
constexpr int kDxMaxChunks = 8;    // 256-column chunks: D <= 2048
constexpr int kDxK = 96;           // six 16-wide terms
// B in shared memory holds the three splits only, rows split * 16 + o of each 64-column
// block (the forward's image, byte for byte); K16 step j of the six terms reads the 16 rows
// of split dx_term_b(j)
constexpr int kDxBRow = 3 * 16 * 128;   // bytes of one 64-column block of B
constexpr size_t kDxFixed = 1024 + 2 * 16384 + 256;   // alignment slack, A (two 64-wide K blocks), barriers

inline size_t dx_tc_smem_bytes(int D) { return kDxFixed + (size_t)kDxBRow * ((D + 63) / 64); }

// split of e or of the weight used by term j (0 = hi, 1 = mid, 2 = lo), for A and for B
__host__ __device__ constexpr int dx_term_a(int j) { return j == 2 || j == 5 ? 1 : j == 4 ? 2 : 0; }
__host__ __device__ constexpr int dx_term_b(int j) { return j == 1 || j == 5 ? 1 : j == 3 ? 2 : 0; }

__global__ void __launch_bounds__(kDxThreads, 1)
cg_bwd_dx_tc_kernel(CgShape s, const float *__restrict__ weight, const uint8_t *__restrict__ splits,
                    const float *__restrict__ dc, const float *__restrict__ dg, __nv_bfloat16 *__restrict__ dx,
                    uint32_t wait_ns) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int nblk = (s.D + 63) / 64;
    const int nch = (nblk + 3) / 4;   // column chunks of up to 4 blocks (256 columns)
    uint8_t *as = sm;                 // A: two K blocks of [128 rows][128 bytes]
    uint8_t *wb = sm + 2 * 16384;     // B
    uint64_t *bars = (uint64_t *)(wb + (size_t)nblk * kDxBRow);
    uint64_t *accfull = bars, *tfree = bars + 2, *wready = bars + 4;   // wready[chunk]: its blocks of the image
    uint32_t *tmem_slot = (uint32_t *)(bars + 4 + kDxMaxChunks);
    volatile int *abort_flag = (volatile int *)(tmem_slot + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t0 = (int64_t)blockIdx.x * kTcTile;

    if (threadIdx.x == 0) {
        ptx::mbar_init(&accfull[0], 1);
        ptx::mbar_init(&accfull[1], 1);
        ptx::mbar_init(&tfree[0], 256);
        ptx::mbar_init(&tfree[1], 256);
        for (int c = 0; c < kDxMaxChunks; ++c) ptx::mbar_init(&wready[c], 1);
        tc::init_ctl(abort_flag, wait_ns);
        ptx::fence_mbar_init();
        if (splits) {   // the weight image, one bulk copy per 64-column block, chunk by chunk
            for (int c = 0; c < nch; ++c) {
                const int nb = nblk - 4 * c < 4 ? nblk - 4 * c : 4;
                ptx::mbar_arrive_expect_tx(&wready[c], (uint32_t)(nb * kDxBRow));
                for (int kb = 4 * c; kb < 4 * c + nb; ++kb)
                    ptx::bulk_load(wb + kb * kDxBRow, splits + (size_t)kb * kDxBRow, kDxBRow, &wready[c]);
            }
        }
    }
    if (warp == 4) {
        ptx::tmem_alloc(tmem_slot, 512);
        ptx::tmem_relinquish();
    }
    if (warp < 4) {
        // this thread's token row of A: e in its three splits, laid out as the six terms
        const int row = threadIdx.x;
        const int64_t t = t0 + row;
        uint32_t sp3[3][8];   // split -> 16 bf16 as 8 words
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            float e0 = 0.f, e1 = 0.f;
            const int o0 = 2 * q, o1 = 2 * q + 1;
            if (t < s.N) {
                if (o0 < 2 * s.H) e0 = o0 < s.H ? __ldg(dc + t * s.H + o0) : __ldg(dg + t * s.H + o0 - s.H);
                if (o1 < 2 * s.H) e1 = o1 < s.H ? __ldg(dc + t * s.H + o1) : __ldg(dg + t * s.H + o1 - s.H);
            }
            uint32_t h0, m0, l0, h1, m1, l1;
            split3(e0, h0, m0, l0);
            split3(e1, h1, m1, l1);
            sp3[0][q] = h0 | (h1 << 16);
            sp3[1][q] = m0 | (m1 << 16);
            sp3[2][q] = l0 | (l1 << 16);
        }
#pragma unroll
        for (int c = 0; c < 16; ++c) {   // 16-byte chunks of the row: K = 8c .. 8c + 7
            const int j = c >> 1, half = c & 1;
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (j < 6) {
                const int sp = dx_term_a(j);
                v = make_uint4(sp3[sp][4 * half], sp3[sp][4 * half + 1], sp3[sp][4 * half + 2], sp3[sp][4 * half + 3]);
            }
            const int blk = c >> 3, c16 = c & 7;
            *reinterpret_cast<uint4 *>(as + blk * 16384 + row * 128 + ((c16 ^ (row & 7)) << 4)) = v;
        }
    }
    if (!splits) stage_weight_splits<16>(s, weight, wb, nblk, threadIdx.x, kDxThreads);
    ptx::fence_proxy_async_smem();
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 4) {
        if (lane == 0) {
            bool ok = true;
            const uint32_t aa = ptx::smem_u32(as), ba = ptx::smem_u32(wb);
            for (int c = 0; c < nch && ok; ++c) {
                const int b = c & 1;
                if (splits) {
                    ok = tc::wait_bar(&wready[c], 0, abort_flag);
                    if (!ok) break;
                }
                if (c >= 2) {
                    ok = tc::wait_bar(&tfree[b], (uint32_t)((c / 2 - 1) & 1), abort_flag);
                    if (!ok) break;
                    ptx::tc_fence_after();
                }
                const int ncols = (nblk - 4 * c < 4 ? nblk - 4 * c : 4) * 64;
                const uint32_t idesc = ptx::idesc_bf16_f32(128, ncols, 0, 1);
#pragma unroll
                for (int k = 0; k < kDxK / 16; ++k) {
                    const uint64_t ad = ptx::smem_desc_sw128(aa + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024);
                    const uint64_t bd =
                        ptx::smem_desc_sw128(ba + 4 * c * kDxBRow + dx_term_b(k) * 16 * 128, kDxBRow, 1024);
                    ptx::mma_bf16(tmem + b * 256, ad, bd, idesc, k != 0);
                }
                ptx::mma_commit(&accfull[b]);
            }
        }
    } else {
        // epilogue: warps 0-3 and 5-8 (warp w reads TMEM lane quarter w % 4); the two sets take
        // alternate pairs of 16-column groups of each chunk
        const int qtr = warp & 3, set = warp < 4 ? 0 : 1;
        const int64_t t = t0 + qtr * 32 + lane;
        __nv_bfloat16 *rowp = dx + (t < s.N ? t : 0) * s.sdx;
        const bool a32 = ((uintptr_t)rowp & 31) == 0;
        for (int c = 0; c < nch; ++c) {
            const int b = c & 1;
            const bool ok = tc::wait_bar(&accfull[b], (uint32_t)((c / 2) & 1), abort_flag);
            ptx::tc_fence_after();
            if (!ok) break;
            const int ncols = (nblk - 4 * c < 4 ? nblk - 4 * c : 4) * 64;
            const uint32_t base = tmem + b * 256 + ((uint32_t)(qtr * 32) << 16);
            for (int g16 = 2 * set; g16 < ncols / 16; g16 += 4) {
                uint32_t r0[16], r1[16];
                ptx::tmem_ld16_issue(base + g16 * 16, r0);
                ptx::tmem_ld16_issue(base + (g16 + 1) * 16, r1);
                ptx::tmem_wait_ld();
                ptx::reg_fence16(r0);
                ptx::reg_fence16(r1);
                auto emit = [&](const uint32_t (&r)[16], int col) {
                    uint32_t w[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const __nv_bfloat162 p2 =
                            __floats2bfloat162_rn(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1]));
                        w[e] = *reinterpret_cast<const uint32_t *>(&p2);
                    }
                    if (t < s.N) {
                        if (col + 16 <= s.D) {
                            ptx::st_global_32b(rowp + col, w, a32);
                        } else {
#pragma unroll
                            for (int e = 0; e < 8; ++e)
                                if (2 * e + col < s.D) reinterpret_cast<uint32_t *>(rowp + col)[e] = w[e];
                        }
                    }
                };
                emit(r0, c * 256 + g16 * 16);
                emit(r1, c * 256 + (g16 + 1) * 16);
            }
            ptx::tc_fence_before();
            ptx::mbar_arrive(&tfree[b]);
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 4) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------------------------------
// dweight on the tensor cores (bf16 x, 2H <= 16): the CTA of partial record b sums its token
// range [b * span, (b + 1) * span) as D[m][k] = sum_t A[t][m] x[t][k] with m = split * 16 + o,
// A[t][m] the bf16 split `split` of e[t][o] (rows m >= 48 zero), so that every product is exact
// and dweight's partial is D[o] + D[16 + o] + D[32 + o], added in that order.  A and x are
// MN-major operands (x straight from TMA in [64 tokens][64 columns] boxes); the columns go in
// groups of up to 256 into two alternating TMEM buffers, each group over all the range's
// 64-token chunks.  Warps 0-1 read TMEM rows 0-63 and write the record, warps 2-3 build the A
// stages, warp 4 issues the TMA loads, warp 5 the MMAs.  dbias's partial is the plain fp32 sum
// of e over the range (threads o < 2H of warp 0, tokens in order).  The record is that of the
// CUDA-core kernel, so the same reduce kernel adds the records.
// ---------------------------------------------------------------------------------------

constexpr int kDwTcThreads = 192;
constexpr int kDwTcStages = 3;
constexpr int kDwTcChunk = 64;                         // tokens per A / x stage (K)
constexpr int kDwTcXBytes = 4 * 64 * 128;              // 4 column blocks of [64 tokens][128 B]
constexpr int kDwTcABytes = 2 * 64 * 128;              // M blocks 0 (e splits) and 1 (zero)
constexpr int kDwTcStageBytes = kDwTcXBytes + kDwTcABytes;
constexpr int kDwTcXRow = 257;                        // floats per exchange row (odd: rows hit distinct banks)
constexpr size_t kDwTcSmem = 1024 + (size_t)kDwTcStages * kDwTcStageBytes + 32 * kDwTcXRow * 4 + 64 * 17 * 4 + 256;

__global__ void __launch_bounds__(kDwTcThreads, 1)
cg_bwd_dw_tc_kernel(const __grid_constant__ CUtensorMap map_x, CgShape s, int64_t span, const float *__restrict__ dc,
                    const float *__restrict__ dg, float *__restrict__ part, uint32_t wait_ns) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    // rows 0-15: split 2 of outputs 0-15; rows 16-31: split 0 + split 1 (one column group)
    float *xchg = (float *)(sm + kDwTcStages * kDwTcStageBytes);
    float *dbpart = xchg + 32 * kDwTcXRow;   // [64 A-builder threads][17]: their sums of e per output
    uint64_t *bars = (uint64_t *)(((uintptr_t)(dbpart + 64 * 17) + 7) & ~(uintptr_t)7);
    uint64_t *full = bars, *aready = bars + kDwTcStages, *empty = bars + 2 * kDwTcStages;
    uint64_t *accfull = bars + 3 * kDwTcStages, *tfree = accfull + 2;
    uint32_t *tmem_slot = (uint32_t *)(tfree + 2);
    volatile int *abort_flag = (volatile int *)(tmem_slot + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int H2 = 2 * s.H;
    const int64_t ta = (int64_t)blockIdx.x * span;
    const int64_t tb = ta + span < s.N ? ta + span : s.N;
    const int nch = tb > ta ? (int)((tb - ta + kDwTcChunk - 1) / kDwTcChunk) : 0;
    const int nblk = (s.D + 63) / 64;
    const int ngr = (nblk + 3) / 4;
    const int items = ngr * nch;
    float *rec = part + (int64_t)blockIdx.x * record_floats(s.D, s.H);

    if (threadIdx.x == 0) {
        for (int i = 0; i < kDwTcStages; ++i) {
            ptx::mbar_init(&full[i], 1);
            ptx::mbar_init(&aready[i], 64);
            ptx::mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(&accfull[i], 1);
            ptx::mbar_init(&tfree[i], 64);
        }
        tc::init_ctl(abort_flag, wait_ns);
        ptx::fence_mbar_init();
    }
    if (warp == 5) {
        ptx::tmem_alloc(tmem_slot, 512);
        ptx::tmem_relinquish();
    }
    // M block 1 of every A stage stays zero
    for (int i = threadIdx.x; i < kDwTcStages * 64 * 128 / 16; i += kDwTcThreads) {
        const int st = i / (64 * 128 / 16), r = i - st * (64 * 128 / 16);
        *reinterpret_cast<uint4 *>(sm + st * kDwTcStageBytes + kDwTcXBytes + 64 * 128 + r * 16) = make_uint4(0u, 0u, 0u, 0u);
    }
    ptx::fence_proxy_async_smem();
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    auto group_blocks = [&](int g) { return nblk - 4 * g < 4 ? nblk - 4 * g : 4; };

    if (warp == 4) {
        if (lane == 0) {
            ptx::prefetch_tensormap(&map_x);
            for (int i = 0; i < items; ++i) {
                const int st = i % kDwTcStages, g = i / nch, ch = i - g * nch;
                if (i >= kDwTcStages && !tc::wait_bar(&empty[st], (uint32_t)((i / kDwTcStages - 1) & 1), abort_flag)) break;
                const int nb = group_blocks(g);
                ptx::mbar_arrive_expect_tx(&full[st], (uint32_t)nb * 8192);
                for (int b = 0; b < nb; ++b)
                    ptx::tma_load_2d(sm + st * kDwTcStageBytes + b * 8192, &map_x, (4 * g + b) * 64,
                                     (int)(ta + (int64_t)ch * kDwTcChunk), &full[st]);
            }
        }
    } else if (warp == 2 || warp == 3) {
        // A stages: thread r builds token row r of the chunk (64 M values, 128 bytes); during the
        // first column group it also sums its tokens' e per output (for dbias)
        const int r = threadIdx.x - 64;
        float dbacc[16];
#pragma unroll
        for (int o = 0; o < 16; ++o) dbacc[o] = 0.f;
        for (int i = 0; i < items; ++i) {
            const int st = i % kDwTcStages, g = i / nch, ch = i - g * nch;
            if (i >= kDwTcStages && !tc::wait_bar(&empty[st], (uint32_t)((i / kDwTcStages - 1) & 1), abort_flag)) break;
            const int64_t t = ta + (int64_t)ch * kDwTcChunk + r;
            uint32_t w[3][8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                float e0 = 0.f, e1 = 0.f;
                const int o0 = 2 * q, o1 = 2 * q + 1;
                if (t < tb) {
                    if (o0 < H2) e0 = o0 < s.H ? __ldg(dc + t * s.H + o0) : __ldg(dg + t * s.H + o0 - s.H);
                    if (o1 < H2) e1 = o1 < s.H ? __ldg(dc + t * s.H + o1) : __ldg(dg + t * s.H + o1 - s.H);
                }
                if (g == 0) {
                    dbacc[o0] += e0;
                    dbacc[o1] += e1;
                }
                uint32_t h0, m0, l0, h1, m1, l1;
                split3(e0, h0, m0, l0);
                split3(e1, h1, m1, l1);
                w[0][q] = h0 | (h1 << 16);
                w[1][q] = m0 | (m1 << 16);
                w[2][q] = l0 | (l1 << 16);
            }
            uint8_t *arow = sm + st * kDwTcStageBytes + kDwTcXBytes + r * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c) {   // 16-byte chunk c holds m = 8c .. 8c + 7
                const int sp = c >> 1, half = c & 1;
                uint4 v = make_uint4(0u, 0u, 0u, 0u);
                if (sp < 3) v = make_uint4(w[sp][4 * half], w[sp][4 * half + 1], w[sp][4 * half + 2], w[sp][4 * half + 3]);
                *reinterpret_cast<uint4 *>(arow + ((c ^ (r & 7)) << 4)) = v;
            }
            ptx::fence_proxy_async_smem();
            ptx::mbar_arrive(&aready[st]);
        }
#pragma unroll
        for (int o = 0; o < 16; ++o) dbpart[r * 17 + o] = dbacc[o];
        tc::named_sync(2, 128);   // warps 0-3: the dbias sums are in dbpart
    } else if (warp == 5) {
        if (lane == 0) {
            bool ok = true;
            for (int i = 0; i < items && ok; ++i) {
                const int st = i % kDwTcStages, g = i / nch, ch = i - g * nch;
                const int b = g & 1;
                if (ch == 0 && g >= 2) {
                    ok = tc::wait_bar(&tfree[b], (uint32_t)((g / 2 - 1) & 1), abort_flag);
                    if (!ok) break;
                }
                ok = tc::wait_bar(&full[st], (uint32_t)((i / kDwTcStages) & 1), abort_flag) &&
                     tc::wait_bar(&aready[st], (uint32_t)((i / kDwTcStages) & 1), abort_flag);
                if (!ok) break;
                ptx::tc_fence_after();
                const uint32_t xa = ptx::smem_u32(sm + st * kDwTcStageBytes);
                const uint32_t aa = xa + kDwTcXBytes;
                const uint32_t idesc = ptx::idesc_bf16_f32(128, group_blocks(g) * 64, 1, 1);
#pragma unroll
                for (int k = 0; k < kDwTcChunk / 16; ++k) {
                    const uint64_t ad = ptx::smem_desc_sw128(aa + k * 2048, 64 * 128, 1024);
                    const uint64_t bd = ptx::smem_desc_sw128(xa + k * 2048, 8192, 1024);
                    ptx::mma_bf16(tmem + b * 256, ad, bd, idesc, (ch | k) != 0);
                }
                ptx::mma_commit(&empty[st]);
                if (ch == nch - 1) ptx::mma_commit(&accfull[b]);
            }
        }
    } else {
        // warps 0-1: TMEM rows 0-63 (warp 0: split 0 in lanes 0-15, split 1 in 16-31; warp 1:
        // split 2 in lanes 0-15)
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        const int tid64 = threadIdx.x;   // 0..63
        volatile int *verdict = abort_flag + 2;
        // One decision for both warps (the flag may be set by other warps at any time): thread
        // 0 copies it between two barriers of the 64 threads.
        auto collective_abort = [&]() {
            tc::named_sync(1, 64);
            if (tid64 == 0) *verdict = *abort_flag;
            tc::named_sync(1, 64);
            return *verdict != 0;
        };
        for (int g = 0; g < ngr && nch > 0; ++g) {
            const int b = g & 1;
            (void)tc::wait_bar(&accfull[b], (uint32_t)((g / 2) & 1), abort_flag);
            ptx::tc_fence_after();
            if (collective_abort()) break;
            const int ncols = group_blocks(g) * 64;
            for (int c16 = 0; c16 < ncols / 16; ++c16) {
                uint32_t r[16];
                ptx::tmem_ld16_issue(tmem + b * 256 + lane_base + c16 * 16, r);
                ptx::tmem_wait_ld();
                ptx::reg_fence16(r);
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const float own = __uint_as_float(r[e]);
                    const float up = __shfl_down_sync(0xffffffffu, own, 16);   // warp 0: split 1 of the same output
                    if (lane < 16) xchg[(warp == 0 ? 16 + lane : lane) * kDwTcXRow + c16 * 16 + e] = warp == 0 ? own + up : own;
                }
            }
            ptx::tc_fence_before();
            ptx::mbar_arrive(&tfree[b]);   // TMEM buffer b may be overwritten
            tc::named_sync(1, 64);         // the group's sums are in xchg
            for (int o = 0; o < H2; ++o) {
                float *dst = rec + (int64_t)o * s.D + g * 256;
                for (int c = tid64; c < ncols && g * 256 + c < s.D; c += 64)
                    dst[c] = xchg[(16 + o) * kDwTcXRow + c] + xchg[o * kDwTcXRow + c];   // (split 0 + split 1) + split 2
            }
            tc::named_sync(1, 64);   // xchg is free for the next group
        }
        tc::named_sync(2, 128);   // warps 0-3: the A builders' dbias sums are in dbpart
        if (nch == 0) {   // an empty range: zero record
            for (int64_t i = tid64; i < record_floats(s.D, s.H); i += 64) rec[i] = 0.f;
        } else if (tid64 < H2) {
            // dbias: the 64 builder threads' sums (each over its tokens in order), added in order
            float acc = dbpart[tid64];
            for (int i = 1; i < 64; ++i) acc += dbpart[i * 17 + tid64];
            rec[(int64_t)H2 * s.D + tid64] = acc;
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------------------------------
// The weight's bf16 split image, written once per weight: 3R rows x 128 bytes per 64-column
// block, byte for byte what the forward (K-major B) and dx (MN-major B, 2H <= 16) otherwise
// build in shared memory, so results are identical with or without it.
// ---------------------------------------------------------------------------------------
__host__ __device__ inline size_t prep_fwd_bytes(int D, int H) { return tc_split_bytes(D, H); }


template <int R>
__global__ void __launch_bounds__(256) cg_prepare_kernel(CgShape s, const float *__restrict__ weight,
                                                        uint8_t *__restrict__ img) {
    const int nkb = (s.D + 63) / 64;
    const int tid = blockIdx.x * blockDim.x + threadIdx.x, nth = gridDim.x * blockDim.x;
    stage_weight_splits<R>(s, weight, img, nkb, tid, nth);
}

}  // namespace cg
}  // namespace dc
