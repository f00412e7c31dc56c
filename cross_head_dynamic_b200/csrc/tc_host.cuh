// tc_host.cuh -- host side of the tcgen05/TMA path: shape support, block-size
// choice, TMA descriptors (cuTensorMapEncodeTiled through the runtime's
// driver entry point, so the library does not link libcuda), launches.
#pragma once

#include <cuda.h>
#include <mutex>

#include "common.cuh"
#include "simt.cuh"
#include "tc_fwd.cuh"
#include "tc_bwd.cuh"

namespace dc {
namespace tc {

constexpr int kMaxWindow = 129;      // BM = 128 keeps the key tile (BM + W - 1 rows) within 256
constexpr int kSegWidth = 128;       // wider windows run as segments of this many keys
constexpr int kMaxSegWindow = 2 * kSegWidth;

inline bool supports(const Shape &s) {
    return (s.d == 64 || s.d == 128) && s.W >= 1 && s.W <= kMaxSegWindow && s.H >= 1 && s.H <= 16 &&
           s.N <= (int64_t)INT32_MAX - 512;
}

inline bool segmented(const Shape &s) { return s.W > kMaxWindow; }

// Segment k of a segmented window (k = 0: the kSegWidth keys ending at the query; k = 1:
// the rest): the shape the kernels run with (W = the segment's width) and its Seg.
inline Shape seg_shape(const Shape &s, int k, int mode, Seg *seg) {
    Shape r = s;
    r.W = k == 0 ? kSegWidth : s.W - kSegWidth;
    seg->shift = k * kSegWidth;
    seg->wrow = s.W;
    seg->wofs = s.W - seg->shift - r.W;
    seg->mode = mode;
    return r;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (EncodeTiledFn)p;
    });
    return fn;
}

// 2-D view [N rows][H*d bf16] of a [N][H][d] tensor whose consecutive tokens are `stride`
// elements apart (H * d when contiguous; a multiple of 8); boxes of 64 columns x box_rows
// rows, 128-byte swizzle, zero fill outside the tensor.
inline cudaError_t make_map(CUtensorMap *m, const void *ptr, int64_t N, int H, int d, int64_t stride, int box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    cuuint64_t dims[2] = {(cuuint64_t)H * d, (cuuint64_t)N};
    cuuint64_t strides[1] = {(cuuint64_t)stride * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    cuuint32_t es[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// 3-D view [H][N][cols] of the ds tiles in the workspace (bf16, row stride cols): boxes of 64
// columns x box_rows rows x 1 head, 128-byte swizzle.  Loads outside the tensor read zeros;
// stores outside it are dropped.
inline cudaError_t make_map_ds(CUtensorMap *m, const void *ptr, int64_t N, int H, int cols, int box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)N, (cuuint64_t)H};
    cuuint64_t strides[2] = {(cuuint64_t)cols * 2, (cuuint64_t)N * cols * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
    cuuint32_t es[3] = {1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

inline int sm_count() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

inline int round16(int x) { return (x + 15) & ~15; }

// Query-block size: the candidate (multiple of 16, <= 128, tile span <= 256)
// minimising waves x per-CTA cost, with the per-CTA cost modelled as the tile
// span plus a fixed overhead; one CTA per SM.
inline int choose_block(int64_t N, int W, int sms, int max_span = 256) {
    int best = 64;
    double best_cost = 1e300;
    for (int bm = 128; bm >= 64; bm -= 16) {
        if (round16(bm + W - 1) > max_span) continue;
        const int64_t blocks = (N + bm - 1) / bm;
        const int64_t waves = (blocks + sms - 1) / sms;
        const double cost = (double)waves * (round16(bm + W - 1) + 96);
        if (cost < best_cost - 1e-9) {
            best_cost = cost;
            best = bm;
        }
    }
    return best;
}

// register-array width of the softmax warps: chunks of 8 columns per thread
// (a quarter's band of 31 + W columns split between kSplits warps)
inline int maxc_for(int W) {
    const int need = (((31 + W + 7) / 8) + kSplits - 1) / kSplits;
    if (need <= 3) return 3;
    if (need <= 4) return 4;
    if (need <= 6) return 6;
    return 7;
}

template <typename K>
inline cudaError_t set_smem(K kernel, uint32_t bytes) {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

template <int D, int MAXC, bool SEG = false>
inline cudaError_t launch_fwd(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv, const FwdArgs &a,
                              cudaStream_t st) {
    auto kern = fwd_kernel<D, MAXC, SEG>;
    cudaError_t e = set_smem(kern, FwdLayout<D>::kAlloc);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)((a.s.N + a.BM - 1) / a.BM);
    kern<<<grid, kThreads, FwdLayout<D>::kAlloc, st>>>(mq, mk, mv, a);
    return cudaGetLastError();
}

template <int D>
inline cudaError_t launch_fwd_d(int maxc, const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv,
                                const FwdArgs &a, cudaStream_t st) {
    switch (maxc) {
        case 3: return launch_fwd<D, 3>(mq, mk, mv, a, st);
        case 4: return launch_fwd<D, 4>(mq, mk, mv, a, st);
        case 6: return launch_fwd<D, 6>(mq, mk, mv, a, st);
        default: return launch_fwd<D, 7>(mq, mk, mv, a, st);
    }
}

// Window of more than kMaxWindow keys: the far segment's LSE into lse; the near segment
// merges its own LSE into it, writes its part of pmap and its share of o; the far segment
// writes its part of pmap and adds its share of o (three launches; lse is required).
inline cudaError_t fwd_segmented(const Shape &s, const void *q, const void *k, const void *v, const float *c,
                                 const float *g, void *o, float *lse, void *pmap, cudaStream_t st, int32_t *launches) {
    if (!lse) return cudaErrorInvalidValue;
    const int BM = choose_block(s.N, kSegWidth, sm_count());
    CUtensorMap mq, mk[2], mv[2];
    cudaError_t e = make_map(&mq, q, s.N, s.H, s.d, s.sq, 128);
    for (int sk = 0; sk < 2 && e == cudaSuccess; ++sk) {
        Seg sg;
        const int span = round16(BM + seg_shape(s, sk, 0, &sg).W - 1);
        e = make_map(&mk[sk], k, s.N, s.H, s.d, s.sq, span);
        if (e == cudaSuccess) e = make_map(&mv[sk], v, s.N, s.H, s.d, s.sq, span);
    }
    if (e != cudaSuccess) return e;
    const int order[3][2] = {{1, kFwdSegStats}, {0, kFwdSegNear}, {1, kFwdSegFarApply}};
    for (const auto &step : order) {
        FwdArgs a;
        a.s = seg_shape(s, step[0], step[1], &a.seg);
        a.BM = BM;
        a.span = round16(BM + a.s.W - 1);
        a.c = c;
        a.g = g;
        a.o = (__nv_bfloat16 *)o;
        a.lse = lse;
        a.pmap = (__nv_bfloat16 *)pmap;
        const CUtensorMap &kk = mk[step[0]], &vv = mv[step[0]];
        e = (s.d == 64) ? launch_fwd<64, 7, true>(mq, kk, vv, a, st) : launch_fwd<128, 7, true>(mq, kk, vv, a, st);
        if (e != cudaSuccess) return e;
        ++*launches;
    }
    return cudaSuccess;
}

inline cudaError_t fwd(const Shape &s, const void *q, const void *k, const void *v, const float *c, const float *g,
                       void *o, float *lse, void *pmap, cudaStream_t st, int32_t *launches) {
    if (segmented(s)) return fwd_segmented(s, q, k, v, c, g, o, lse, pmap, st, launches);
    FwdArgs a;
    a.s = s;
    a.BM = choose_block(s.N, s.W, sm_count());
    a.span = round16(a.BM + s.W - 1);
    a.c = c;
    a.g = g;
    a.o = (__nv_bfloat16 *)o;
    a.lse = lse;
    a.pmap = (__nv_bfloat16 *)pmap;
    CUtensorMap mq, mk, mv;
    cudaError_t e = make_map(&mq, q, s.N, s.H, s.d, s.sq, 128);
    if (e == cudaSuccess) e = make_map(&mk, k, s.N, s.H, s.d, s.sq, a.span);
    if (e == cudaSuccess) e = make_map(&mv, v, s.N, s.H, s.d, s.sq, a.span);
    if (e != cudaSuccess) return e;
    const int maxc = maxc_for(s.W);
    e = (s.d == 64) ? launch_fwd_d<64>(maxc, mq, mk, mv, a, st) : launch_fwd_d<128>(maxc, mq, mk, mv, a, st);
    if (e == cudaSuccess) ++*launches;
    return e;
}

template <int D, int MAXC, bool SEG = false, bool DSB = false, bool DST = false>
inline cudaError_t launch_bwd_query(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv,
                                    const CUtensorMap &mdo, const CUtensorMap &mds, const BwdArgs &a,
                                    cudaStream_t st) {
    auto kern = bwd_query_kernel<D, MAXC, SEG, DSB, DST>;
    const uint32_t smem = QSideLayout<D>(a.span).bytes + 1024;
    cudaError_t e = set_smem(kern, smem);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)((a.s.N + a.BM - 1) / a.BM);
    kern<<<grid, kThreads, smem, st>>>(mq, mk, mv, mdo, mds, a);
    return cudaGetLastError();
}

template <int D, int MAXC, bool SEG = false>
inline cudaError_t launch_bwd_key(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mdo,
                                  const BwdArgs &a, cudaStream_t st) {
    auto kern = bwd_key_seg_kernel<D, MAXC, SEG>;
    const KSideLayout<D> L(a.span, a.s.W);
    if (!SEG && L.stage + L.stage_bytes > L.colv) return cudaErrorInvalidValue;   // staging must fit before colv
    const uint32_t smem = L.bytes + 1024;
    cudaError_t e = set_smem(kern, smem);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)((a.s.N + a.BM - 1) / a.BM);
    kern<<<grid, kThreads, smem, st>>>(mq, mk, mdo, a);
    return cudaGetLastError();
}

template <int D, int MAXC>
inline cudaError_t launch_bwd_key_dsb(const CUtensorMap &mq, const CUtensorMap &mdo, const BwdArgs &a,
                                      cudaStream_t st) {
    auto kern = bwd_key_kernel<D, MAXC>;
    const uint32_t smem = DSideLayout<D>(a.span, a.s.W, a.BM, kDsbRow).bytes + 1024;
    cudaError_t e = set_smem(kern, smem);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)((a.s.N + a.BM - 1) / a.BM);
    kern<<<grid, kThreads, smem, st>>>(mq, mdo, a);
    return cudaGetLastError();
}

template <int D>
inline cudaError_t launch_bwd_key_dst(const CUtensorMap &mq, const CUtensorMap &mdo, const CUtensorMap &mds,
                                      const BwdArgs &a, cudaStream_t st) {
    auto kern = bwd_key_dst_kernel<D>;
    const uint32_t smem = TSideLayout<D>(a.span).bytes + 1024;
    cudaError_t e = set_smem(kern, smem);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)((a.s.N + a.BM - 1) / a.BM);
    kern<<<grid, kThreads, smem, st>>>(mq, mdo, mds, a);
    return cudaGetLastError();
}

#define DC_TC_MAXC_SWITCH(maxc, CALL)        \
    switch (maxc) {                          \
        case 3: { constexpr int MC = 3; return CALL; }   \
        case 4: { constexpr int MC = 4; return CALL; }   \
        case 6: { constexpr int MC = 6; return CALL; }   \
        default: { constexpr int MC = 7; return CALL; }  \
    }

inline BwdArgs bwd_args(const Shape &s) {
    BwdArgs a = {};
    a.s = s;
    a.BM = choose_block(s.N, s.W, sm_count(), kBwdMaxSpan);
    a.span = round16(a.BM + s.W - 1);
    return a;
}

// Bytes of the key-major ds band [H][N][kDsbRow] bf16 the query side hands to the key side.
inline size_t dsb_bytes(const Shape &s) { return (size_t)s.H * (size_t)s.N * (size_t)kDsbRow * 2; }

// The ds tile hand-off: query blocks (and key blocks) of kDstBlock tokens, key tiles of
// 2 kDstBlock columns starting kDstBlock keys before the block, tiles [H][N][2 kDstBlock]
// bf16 in the workspace.  It covers windows with W - 1 <= kDstBlock; below kDstMinWindow
// the wider key tile (2 kDstBlock instead of BM + W - 1 columns) costs more than the ds
// band's stores and de-skew (measured: W = 32 and 64 run slower, W = 112 faster).
constexpr int kDstBlock = 112;
constexpr int kDstMinWindow = 97;
inline bool dst_shape(const Shape &s) {
    return !segmented(s) && s.W - 1 <= kDstBlock && s.W >= kDstMinWindow;
}
inline size_t dst_bytes(const Shape &s) { return (size_t)s.H * (size_t)s.N * (size_t)(2 * kDstBlock) * 2; }
inline bool use_dst(const Shape &s, size_t workspace_bytes) {
    if (!dst_shape(s) || workspace_bytes < dst_bytes(s)) return false;
    const uint32_t need = (s.d == 128 ? TSideLayout<128>(2 * kDstBlock).bytes : TSideLayout<64>(2 * kDstBlock).bytes)
                          + 1024;
    return need <= 227u * 1024 && s.W * 2 * kDstBlock * 2 <= (int)TSideLayout<64>(2 * kDstBlock).tile_a;
}
// Register-array width for the DST band: row i's window is columns [i + off, i + off + W - 1]
// with off = kDstBlock - (W - 1), so a lane quarter's band runs from the 8-column boundary at
// or below 32q + off to 32q + off + 31 + W (make_band with that offset).
inline int dst_maxc(int W) {
    const int off = kDstBlock - (W - 1);
    const int nch = (((off + 31 + W) + 7) / 8 * 8 - (off & ~7)) / 8;
    const int need = (nch + kSplits - 1) / kSplits;
    if (need <= 3) return 3;
    if (need <= 4) return 4;
    if (need <= 6) return 6;
    return 7;
}
inline BwdArgs dst_args(const Shape &s) {
    BwdArgs a = {};
    a.s = s;
    a.BM = kDstBlock;
    a.span = 2 * kDstBlock;
    return a;
}

// The backward pair that passes ds through the band (instead of the key side recomputing
// it from S^T and the dP band) runs when the window is one piece, the workspace holds the
// band and the key side's shared-memory layout fits (pmap staging rows before the ds rows).
inline bool use_dsb(const Shape &s, size_t workspace_bytes) {
    if (segmented(s) || workspace_bytes < dsb_bytes(s) || use_dst(s, workspace_bytes)) return false;
    const BwdArgs a = bwd_args(s);
    const bool fits128 = [&] {
        const DSideLayout<128> L(a.span, s.W, a.BM, kDsbRow);
        return L.stage + L.stage_bytes <= L.rs && L.bytes + 1024 <= 227u * 1024;
    }();
    const bool fits64 = [&] {
        const DSideLayout<64> L(a.span, s.W, a.BM, kDsbRow);
        return L.stage + L.stage_bytes <= L.rs && L.bytes + 1024 <= 227u * 1024;
    }();
    return s.d == 128 ? fits128 : fits64;
}

// Segmented query side: far segment (dP band, partial dg and dc), near segment (complete
// dg and dc, its share of dq), far segment again (adds its share of dq).
inline cudaError_t bwd_query_segmented(const Shape &s, const void *q, const void *k, const void *v, const float *c,
                                       const float *g, const void *dO, const float *lse, const void *pmap, void *dq,
                                       float *dc_, float *dg, float *band, cudaStream_t st, int32_t *launches) {
    const int BM = choose_block(s.N, kSegWidth, sm_count(), kBwdMaxSpan);
    CUtensorMap mq, mdo, mk[2], mv[2];
    cudaError_t e = make_map(&mq, q, s.N, s.H, s.d, s.sq, 128);
    if (e == cudaSuccess) e = make_map(&mdo, dO, s.N, s.H, s.d, s.so, 128);
    for (int sk = 0; sk < 2 && e == cudaSuccess; ++sk) {
        Seg sg;
        const int span = round16(BM + seg_shape(s, sk, 0, &sg).W - 1);
        e = make_map(&mk[sk], k, s.N, s.H, s.d, s.sq, span);
        if (e == cudaSuccess) e = make_map(&mv[sk], v, s.N, s.H, s.d, s.sq, span);
    }
    if (e != cudaSuccess) return e;
    const int order[3][2] = {{1, kQSegFarPart1}, {0, kQSegNear}, {1, kQSegFarPart2}};
    for (const auto &step : order) {
        BwdArgs a = {};
        a.s = seg_shape(s, step[0], step[1], &a.seg);
        a.BM = BM;
        a.span = round16(BM + a.s.W - 1);
        a.c = c;
        a.g = g;
        a.lse = lse;
        a.pmap = (const __nv_bfloat16 *)pmap;
        a.dq = (__nv_bfloat16 *)dq;
        a.dc = dc_;
        a.dg = dg;
        a.band = band;
        const CUtensorMap &kk = mk[step[0]], &vv = mv[step[0]];
        e = (s.d == 64) ? launch_bwd_query<64, 7, true>(mq, kk, vv, mdo, mq, a, st)
                        : launch_bwd_query<128, 7, true>(mq, kk, vv, mdo, mq, a, st);
        if (e != cudaSuccess) return e;
        ++*launches;
    }
    return cudaSuccess;
}

inline cudaError_t bwd_query(const Shape &s, const void *q, const void *k, const void *v, const float *c,
                             const float *g, const void *dO, const float *lse, const void *pmap, void *dq, float *dc_,
                             float *dg, void *workspace, size_t workspace_bytes, cudaStream_t st, int32_t *launches) {
    float *band = (float *)workspace;
    if (segmented(s)) return bwd_query_segmented(s, q, k, v, c, g, dO, lse, pmap, dq, dc_, dg, band, st, launches);
    const bool dst = use_dst(s, workspace_bytes);
    const bool dsb = use_dsb(s, workspace_bytes);
    BwdArgs a = dst ? dst_args(s) : bwd_args(s);
    if (dsb) a.dsb = (__nv_bfloat16 *)workspace;
    a.c = c;
    a.g = g;
    a.lse = lse;
    a.pmap = (const __nv_bfloat16 *)pmap;
    a.dq = (__nv_bfloat16 *)dq;
    a.dc = dc_;
    a.dg = dg;
    a.band = band;
    CUtensorMap mq, mk, mv, mdo, mds;
    cudaError_t e = make_map(&mq, q, s.N, s.H, s.d, s.sq, 128);
    if (e == cudaSuccess) e = make_map(&mk, k, s.N, s.H, s.d, s.sq, a.span);
    if (e == cudaSuccess) e = make_map(&mv, v, s.N, s.H, s.d, s.sq, a.span);
    if (e == cudaSuccess) e = make_map(&mdo, dO, s.N, s.H, s.d, s.so, 128);
    if (e == cudaSuccess) e = dst ? make_map_ds(&mds, workspace, s.N, s.H, a.span, a.BM) : make_map(&mds, q, s.N, s.H, s.d, s.sq, 128);
    if (e != cudaSuccess) return e;
    e = [&]() -> cudaError_t {
        if (dst) {
            if (s.d == 64) {
                DC_TC_MAXC_SWITCH(dst_maxc(s.W), (launch_bwd_query<64, MC, false, false, true>(mq, mk, mv, mdo, mds, a, st)));
            }
            DC_TC_MAXC_SWITCH(dst_maxc(s.W), (launch_bwd_query<128, MC, false, false, true>(mq, mk, mv, mdo, mds, a, st)));
        }
        if (dsb) {
            if (s.d == 64) {
                DC_TC_MAXC_SWITCH(maxc_for(s.W), (launch_bwd_query<64, MC, false, true>(mq, mk, mv, mdo, mds, a, st)));
            }
            DC_TC_MAXC_SWITCH(maxc_for(s.W), (launch_bwd_query<128, MC, false, true>(mq, mk, mv, mdo, mds, a, st)));
        }
        if (s.d == 64) {
            DC_TC_MAXC_SWITCH(maxc_for(s.W), (launch_bwd_query<64, MC>(mq, mk, mv, mdo, mds, a, st)));
        }
        DC_TC_MAXC_SWITCH(maxc_for(s.W), (launch_bwd_query<128, MC>(mq, mk, mv, mdo, mds, a, st)));
    }();
    if (e == cudaSuccess) ++*launches;
    return e;
}

// Segmented key side: the near segment's queries write dk and dv, the far segment's add.
inline cudaError_t bwd_key_segmented(const Shape &s, const void *q, const void *k, const float *c, const float *g,
                                     const void *dO, const float *lse, const void *pmap, const float *dc_,
                                     const float *band, void *dk, void *dv, cudaStream_t st, int32_t *launches) {
    const int BK = choose_block(s.N, kSegWidth, sm_count(), kBwdMaxSpan);
    CUtensorMap mk, mq[2], mdo[2];
    cudaError_t e = make_map(&mk, k, s.N, s.H, s.d, s.sq, 128);
    for (int sk = 0; sk < 2 && e == cudaSuccess; ++sk) {
        Seg sg;
        const int span = round16(BK + seg_shape(s, sk, 0, &sg).W - 1);
        e = make_map(&mq[sk], q, s.N, s.H, s.d, s.sq, span);
        if (e == cudaSuccess) e = make_map(&mdo[sk], dO, s.N, s.H, s.d, s.so, span);
    }
    if (e != cudaSuccess) return e;
    const int order[2][2] = {{0, kKSegWrite}, {1, kKSegAdd}};
    for (const auto &step : order) {
        BwdArgs a = {};
        a.s = seg_shape(s, step[0], step[1], &a.seg);
        a.BM = BK;
        a.span = round16(BK + a.s.W - 1);
        a.c = c;
        a.g = g;
        a.lse = lse;
        a.pmap = (const __nv_bfloat16 *)pmap;
        a.dc_in = dc_;
        a.band = const_cast<float *>(band);
        a.dk = (__nv_bfloat16 *)dk;
        a.dv = (__nv_bfloat16 *)dv;
        const CUtensorMap &qq = mq[step[0]], &dd = mdo[step[0]];
        e = (s.d == 64) ? launch_bwd_key<64, 7, true>(qq, mk, dd, a, st) : launch_bwd_key<128, 7, true>(qq, mk, dd, a, st);
        if (e != cudaSuccess) return e;
        ++*launches;
    }
    return cudaSuccess;
}

inline cudaError_t bwd_key(const Shape &s, const void *q, const void *k, const float *c, const float *g,
                           const void *dO, const float *lse, const void *pmap, const float *dc_, const void *workspace,
                           size_t workspace_bytes, void *dk, void *dv, cudaStream_t st, int32_t *launches) {
    const float *band = (const float *)workspace;
    if (segmented(s)) return bwd_key_segmented(s, q, k, c, g, dO, lse, pmap, dc_, band, dk, dv, st, launches);
    if (use_dst(s, workspace_bytes)) {   // ds from the query side's tiles, by TMA
        BwdArgs a = dst_args(s);
        a.pmap = (const __nv_bfloat16 *)pmap;
        a.g = g;
        a.dk = (__nv_bfloat16 *)dk;
        a.dv = (__nv_bfloat16 *)dv;
        CUtensorMap mq, mdo, mds;
        cudaError_t e = make_map(&mq, q, s.N, s.H, s.d, s.sq, a.span);
        if (e == cudaSuccess) e = make_map(&mdo, dO, s.N, s.H, s.d, s.so, a.span);
        if (e == cudaSuccess) e = make_map_ds(&mds, workspace, s.N, s.H, a.span, a.BM);
        if (e != cudaSuccess) return e;
        e = (s.d == 64) ? launch_bwd_key_dst<64>(mq, mdo, mds, a, st) : launch_bwd_key_dst<128>(mq, mdo, mds, a, st);
        if (e == cudaSuccess) ++*launches;
        return e;
    }
    BwdArgs a = bwd_args(s);
    if (use_dsb(s, workspace_bytes)) {   // ds from the query side's band
        a.pmap = (const __nv_bfloat16 *)pmap;
        a.g = g;
        a.dsb = (__nv_bfloat16 *)const_cast<void *>(workspace);
        a.dk = (__nv_bfloat16 *)dk;
        a.dv = (__nv_bfloat16 *)dv;
        CUtensorMap mq, mdo;
        cudaError_t e = make_map(&mq, q, s.N, s.H, s.d, s.sq, a.span);
        if (e == cudaSuccess) e = make_map(&mdo, dO, s.N, s.H, s.d, s.so, a.span);
        if (e != cudaSuccess) return e;
        e = [&]() -> cudaError_t {
            if (s.d == 64) {
                DC_TC_MAXC_SWITCH(maxc_for(s.W), (launch_bwd_key_dsb<64, MC>(mq, mdo, a, st)));
            }
            DC_TC_MAXC_SWITCH(maxc_for(s.W), (launch_bwd_key_dsb<128, MC>(mq, mdo, a, st)));
        }();
        if (e == cudaSuccess) ++*launches;
        return e;
    }
    a.c = c;
    a.g = g;
    a.lse = lse;
    a.pmap = (const __nv_bfloat16 *)pmap;
    a.dc_in = dc_;
    a.band = const_cast<float *>(band);
    a.dk = (__nv_bfloat16 *)dk;
    a.dv = (__nv_bfloat16 *)dv;
    CUtensorMap mq, mk, mdo;
    cudaError_t e = make_map(&mq, q, s.N, s.H, s.d, s.sq, a.span);
    if (e == cudaSuccess) e = make_map(&mk, k, s.N, s.H, s.d, s.sq, 128);
    if (e == cudaSuccess) e = make_map(&mdo, dO, s.N, s.H, s.d, s.so, a.span);
    if (e != cudaSuccess) return e;
    e = [&]() -> cudaError_t {
        if (s.d == 64) {
            DC_TC_MAXC_SWITCH(maxc_for(s.W), (launch_bwd_key<64, MC>(mq, mk, mdo, a, st)));
        }
        DC_TC_MAXC_SWITCH(maxc_for(s.W), (launch_bwd_key<128, MC>(mq, mk, mdo, a, st)));
    }();
    if (e == cudaSuccess) ++*launches;
    return e;
}

}  // namespace tc
}  // namespace dc
