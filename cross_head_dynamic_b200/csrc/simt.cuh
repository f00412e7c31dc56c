// simt.cuh -- CUDA-core kernels for Lightweight DC attention (fp32 arithmetic).
//
// One CTA per query token (forward, backward query side) or per key token
// (backward key side) with one warp per head (up to 8; a warp takes heads w, w + nw, ...
// when there are more).  The sums over heads (the composed map P, dP) are formed by one
// warp in head order, so the results do not depend on the warp count.  These kernels
// cover every supported shape and both storage types; they are the fp32 path
// (tensor cores cannot meet an fp32 tolerance) and the path for bf16 shapes
// the tcgen05 kernels do not take.  Arithmetic is fp32 with expf/logf.
#pragma once

#include "common.cuh"

namespace dc {
namespace simt {

constexpr int kMaxHeads = 16;
constexpr int kMaxWarps = 8;                    // warps per CTA (one per work item up to 8)
constexpr size_t kSmemBudget = 200 * 1024;      // a CTA's shared memory at most

// Floats of the per-warp row tile used by dot_rows32 (32 rows of d + 1).
__host__ __device__ inline size_t tile_floats(int d) { return 32 * ((size_t)d + 1); }

// Shared memory of one CTA with nw warps: a part for the CTA's token (or key tile) and a
// part per warp.
struct SimtSmem {
    size_t per_token, per_warp;   // floats
    size_t bytes(int nw) const { return sizeof(float) * (per_token + (size_t)nw * per_warp); }
};
// Forward: q of every head | lse per head | P over the window | p_h of one 32-key chunk per
// head | the scores of every head over the window when they fit (fwd_keeps_scores) | per
// warp: row tile.
inline bool fwd_keeps_scores(int H, int W) { return (size_t)H * W * sizeof(float) <= 64 * 1024; }
inline SimtSmem fwd_smem(int H, int d, int W) {
    return {(size_t)H * d + kMaxHeads + W + 32 * (size_t)H + (fwd_keeps_scores(H, W) ? (size_t)H * W : 0),
            tile_floats(d)};
}
// Query side: q and dO of every head | P and dP over the window | E_h of one 32-key chunk
// per head | per warp: ds over the window, row tile.
inline SimtSmem bwdq_smem(int H, int d, int W) {
    return {2 * (size_t)H * d + 2 * (size_t)W + 32 * (size_t)H, (size_t)W + tile_floats(d)};
}
// Key side with a tile of TK keys: k of every head of each key | per warp: row tile.
inline SimtSmem bwdk_smem(int H, int d, int TK) { return {(size_t)TK * H * d, tile_floats(d)}; }
// Keys per CTA of the key side: 4 once there are at least 16 keys per SM, else 1.
inline int key_tile(int64_t N) { return N >= 16 * 148 ? 4 : 1; }
// Warps per CTA: one per work item (head, or (head, key) on the key side) up to kMaxWarps,
// fewer when shared memory runs short (0: not even one warp fits).
inline int warps_per_cta(int items, const SimtSmem &m) {
    int nw = items < kMaxWarps ? items : kMaxWarps;
    while (nw > 0 && m.bytes(nw) > kSmemBudget) --nw;
    return nw;
}

// <xs, row(lane)> for up to 32 consecutive rows, row r at rows + r * stride (d = 32 * DPL
// elements, xs in shared memory).  The rows pass through this warp's tile with coalesced
// loads (the warp reads one row at a time), then every lane takes its own row from the
// tile; rows are d + 1 floats apart, so those reads hit 32 distinct banks.  All lanes
// call it; lanes >= cnt get 0.
template <typename T, int DPL>
__device__ __forceinline__ float dot_rows32(const float *xs, const T *rows, int64_t stride, int cnt, float *tile) {
    constexpr int d = 32 * DPL;
    const int lane = threadIdx.x & 31;
    __syncwarp();
    for (int r = 0; r < cnt; ++r) {
        const T *src = rows + r * stride;
#pragma unroll
        for (int i = 0; i < DPL; ++i) tile[r * (d + 1) + lane + 32 * i] = ldf<T>(src + lane + 32 * i);
    }
    __syncwarp();
    float acc = 0.f;
    if (lane < cnt) {
        const float *tr = tile + lane * (d + 1);
#pragma unroll 8
        for (int e = 0; e < d; ++e) acc = fmaf(xs[e], tr[e], acc);
    }
    return acc;
}

// Forward: one CTA per query token, warp w takes heads w, w + nw, ...  lse per head
// (pass 1); the composed map P over the window, 32 keys at a time: every warp writes p_h
// of its heads, then warp 0 adds c_h p_h in head order (pass 2); o_h = g_h * sum_j P(j)
// v_h(j) per head (pass 3).  With `keep`, pass 1 keeps the scores in shared memory and
// pass 2 reads them back instead of computing them again (the same values).
template <typename T, int DPL>
__global__ void fwd_kernel(Shape s, int keep, const T *__restrict__ q, const T *__restrict__ k,
                           const T *__restrict__ v, const float *__restrict__ c,
                           const float *__restrict__ g, T *__restrict__ o,
                           float *__restrict__ lse, T *__restrict__ pmap, int check_seqlens) {
    constexpr int d = 32 * DPL;
    extern __shared__ float smem[];
    if (check_seqlens) validate_seqlens(s);
    const int H = s.H, W = s.W;
    const int nw = blockDim.x >> 5, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t = blockIdx.x;
    float *qs = smem;
    float *ls = qs + H * d;
    float *Pw = ls + kMaxHeads;
    float *ph = Pw + W;                                     // [H][32]
    float *sc = ph + 32 * H;                                // [H][W] scores (with keep)
    float *tile = sc + (keep ? (size_t)H * W : 0) + (size_t)warp * tile_floats(d);

    for (int i = threadIdx.x; i < H * d; i += blockDim.x) qs[i] = ldf<T>(q + t * s.sq + i);
    __syncthreads();
    const int64_t lo = window_lo(s, t);
    const int n = (int)(t - lo + 1);

    for (int h = warp; h < H; h += nw) {
        float m = -INFINITY, z = 0.f;
        for (int base = 0; base < n; base += 32) {
            const int cnt = min(32, n - base);
            const float x = s.scale * dot_rows32<T, DPL>(qs + h * d, k + (lo + base) * s.sq + h * d, s.sq, cnt, tile);
            if (keep && lane < cnt) sc[h * W + base + lane] = x;
            if (lane < cnt) {
                if (x > m) {
                    z = z * expf(m - x) + 1.f;
                    m = x;
                } else {
                    z += expf(x - m);
                }
            }
        }
        const float M = warp_max(m);
        z = (m == -INFINITY) ? 0.f : z * expf(m - M);
        const float Z = warp_sum(z);
        const float l = M + logf(Z);
        if (lane == 0) {
            ls[h] = l;
            if (lse) lse[t * H + h] = l;
        }
    }
    __syncthreads();
    for (int base = 0; base < n; base += 32) {
        const int cnt = min(32, n - base);
        for (int h = warp; h < H; h += nw) {
            const float x = keep ? (lane < cnt ? sc[h * W + base + lane] : s.scale * 0.f)
                                 : s.scale * dot_rows32<T, DPL>(qs + h * d, k + (lo + base) * s.sq + h * d, s.sq, cnt,
                                                                tile);
            ph[h * 32 + lane] = expf(x - ls[h]);
        }
        __syncthreads();
        if (warp == 0) {
            float P = 0.f;
            for (int h = 0; h < H; ++h) P = fmaf(__ldg(c + t * H + h), ph[h * 32 + lane], P);
            if (lane < cnt) Pw[base + lane] = P;
        }
        __syncthreads();   // Pw written; ph free for the next chunk
    }
    if (pmap) {
        const int64_t w0 = lo - (t - W + 1);   // band index of key lo
        for (int w = threadIdx.x; w < W; w += blockDim.x) stf<T>(pmap + t * W + w, (w >= w0) ? Pw[w - w0] : 0.f);
    }
    for (int h = warp; h < H; h += nw) {
        float acc[DPL];
#pragma unroll
        for (int i = 0; i < DPL; ++i) acc[i] = 0.f;
        for (int jj = 0; jj < n; ++jj) {   // (unrolling it, or four partial sums, measured slower)
            const float P = Pw[jj];
            const T *vr = v + (lo + jj) * s.sq + h * d;
#pragma unroll
            for (int i = 0; i < DPL; ++i) acc[i] = fmaf(P, ldf<T>(vr + lane + 32 * i), acc[i]);
        }
        const float gh = __ldg(g + t * H + h);
#pragma unroll
        for (int i = 0; i < DPL; ++i) stf<T>(o + t * s.so + h * d + lane + 32 * i, gh * acc[i]);
    }
}

// Backward, query side: one CTA per query token, warp w takes heads w, w + nw, ...
// Pass 1 over the window, 32 keys at a time: every warp writes E_h(j) = <dO_h, v_h(j)> of its
// heads and adds P(j) E_h(j) to dg_h; warp 0 then forms dP(j) = sum_h g_h E_h(j) in head order
// (stored to the workspace band).  Pass 2 per head: p_h(j) from lse, dc_h = sum_j dP(j)
// p_h(j), ds_h(j) = c_h p_h(j) (dP(j) - dc_h), dq_h = sigma sum_j ds_h(j) k_h(j).
template <typename T, int DPL>
__global__ void bwd_query_kernel(Shape s, const T *__restrict__ q, const T *__restrict__ k,
                                 const T *__restrict__ v, const float *__restrict__ c,
                                 const float *__restrict__ g, const T *__restrict__ dO,
                                 const float *__restrict__ lse, const T *__restrict__ pmap,
                                 T *__restrict__ dq, float *__restrict__ dc, float *__restrict__ dg,
                                 float *__restrict__ dPband, int check_seqlens) {
    constexpr int d = 32 * DPL;
    extern __shared__ float smem[];
    if (check_seqlens) validate_seqlens(s);
    const int H = s.H, W = s.W;
    const int nw = blockDim.x >> 5, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t = blockIdx.x;
    float *qs = smem;
    float *dos = qs + H * d;
    float *Pw = dos + H * d;
    float *dPw = Pw + W;
    float *eh = dPw + W;                                    // [H][32]
    float *sw = eh + 32 * H + (size_t)warp * (W + tile_floats(d));
    float *tile = sw + W;

    for (int i = threadIdx.x; i < H * d; i += blockDim.x) {
        qs[i] = ldf<T>(q + t * s.sq + i);
        dos[i] = ldf<T>(dO + t * s.so + i);
    }
    const int64_t lo = window_lo(s, t);
    const int n = (int)(t - lo + 1);
    const int w0 = (int)(lo - (t - W + 1));
    for (int jj = threadIdx.x; jj < n; jj += blockDim.x) Pw[jj] = ldf<T>(pmap + t * W + w0 + jj);
    for (int w = threadIdx.x; w < w0; w += blockDim.x) dPband[t * W + w] = 0.f;
    __syncthreads();

    float dgp[kMaxHeads];   // slot u: head warp + u * nw
#pragma unroll
    for (int u = 0; u < kMaxHeads; ++u) dgp[u] = 0.f;
    for (int base = 0; base < n; base += 32) {
        const int cnt = min(32, n - base);
        const int jj = base + lane;
        const float pj = lane < cnt ? Pw[jj] : 0.f;
#pragma unroll
        for (int u = 0; u < kMaxHeads; ++u) {
            const int h = warp + u * nw;
            if (h < H) {
                const float E = dot_rows32<T, DPL>(dos + h * d, v + (lo + base) * s.sq + h * d, s.sq, cnt, tile);
                eh[h * 32 + lane] = E;
                dgp[u] = fmaf(pj, E, dgp[u]);
            }
        }
        __syncthreads();
        if (warp == 0) {
            float dP = 0.f;
            for (int h = 0; h < H; ++h) dP = fmaf(__ldg(g + t * H + h), eh[h * 32 + lane], dP);
            if (lane < cnt) {
                dPw[jj] = dP;
                dPband[t * W + w0 + jj] = dP;
            }
        }
        __syncthreads();   // dPw written; eh free for the next chunk
    }
#pragma unroll
    for (int u = 0; u < kMaxHeads; ++u) {
        const int h = warp + u * nw;
        if (h < H) {
            const float x = warp_sum(dgp[u]);
            if (lane == 0) dg[t * H + h] = x;
        }
    }

    for (int h = warp; h < H; h += nw) {
        const float l = __ldg(lse + t * H + h);
        float dcp = 0.f;
        for (int base = 0; base < n; base += 32) {
            const int cnt = min(32, n - base);
            const float x = s.scale * dot_rows32<T, DPL>(qs + h * d, k + (lo + base) * s.sq + h * d, s.sq, cnt, tile);
            if (lane < cnt) {
                const float p = expf(x - l);
                sw[base + lane] = p;
                dcp = fmaf(dPw[base + lane], p, dcp);
            }
        }
        const float dch = warp_sum(dcp);
        if (lane == 0) dc[t * H + h] = dch;
        const float ch = __ldg(c + t * H + h);
        for (int jj = lane; jj < n; jj += 32) sw[jj] = ch * sw[jj] * (dPw[jj] - dch);
        __syncwarp();
        float acc[DPL];
#pragma unroll
        for (int i = 0; i < DPL; ++i) acc[i] = 0.f;
#pragma unroll 8
        for (int jj = 0; jj < n; ++jj) {
            const float ds = sw[jj];
            const T *kr = k + (lo + jj) * s.sq + h * d;
#pragma unroll
            for (int i = 0; i < DPL; ++i) acc[i] = fmaf(ds, ldf<T>(kr + lane + 32 * i), acc[i]);
        }
#pragma unroll
        for (int i = 0; i < DPL; ++i) stf<T>(dq + t * s.sdq + h * d + lane + 32 * i, s.scale * acc[i]);
        __syncwarp();
    }
}

// Backward, key side: one CTA per tile of TK consecutive key tokens (TK = 4 when there are
// enough keys, so that the query rows the tile's keys share are reused from L1; else 1);
// the warps (one per item up to 8) take the (head, key) items h * TK + kk of the tile in
// turn, so that warps running at the same time share a head and read overlapping query rows.  For key j and the queries
// t whose window holds it, ds_h(t,j) = c[t,h] p_h(t,j) (dP(t,j) - dc[t,h]) with p_h from lse
// and dP from the workspace band, dk_h(j) = sigma sum_t ds_h q_h(t),
// dv_h(j) = sum_t P g_h dO_h(t).
template <typename T, int DPL>
__global__ void bwd_key_kernel(Shape s, int TK, const T *__restrict__ q, const T *__restrict__ k,
                               const float *__restrict__ c, const float *__restrict__ g,
                               const T *__restrict__ dO, const float *__restrict__ lse,
                               const T *__restrict__ pmap, const float *__restrict__ dc,
                               const float *__restrict__ dPband, T *__restrict__ dk,
                               T *__restrict__ dv) {
    constexpr int d = 32 * DPL;
    extern __shared__ float smem[];
    const int H = s.H, W = s.W;
    const int nw = blockDim.x >> 5, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t j0 = (int64_t)blockIdx.x * TK;
    const int tk = (int)min((int64_t)TK, s.N - j0);   // keys of this tile
    float *ks = smem;                                 // [TK][H * d]
    float *tile = ks + (size_t)TK * H * d + (size_t)warp * tile_floats(d);
    for (int i = threadIdx.x; i < tk * H * d; i += blockDim.x) ks[i] = ldf<T>(k + (j0 + i / (H * d)) * s.sq + i % (H * d));
    __syncthreads();

    for (int item = warp; item < H * tk; item += nw) {
        const int h = item / tk, kk = item - h * tk;
        const int64_t j = j0 + kk;
        const float *kh = ks + (size_t)kk * H * d + h * d;
        int64_t hi = j + W - 1;
        const int64_t b = doc_end(s, j);
        if (hi > b - 1) hi = b - 1;
        const int n = (int)(hi - j + 1);
        float ak[DPL], av[DPL];
#pragma unroll
        for (int i = 0; i < DPL; ++i) ak[i] = av[i] = 0.f;
        for (int base = 0; base < n; base += 32) {
            float ds = 0.f, pg = 0.f;
            const int cnt0 = min(32, n - base);
            const float x = s.scale * dot_rows32<T, DPL>(kh, q + (j + base) * s.sq + h * d, s.sq, cnt0, tile);
            if (base + lane < n) {
                const int64_t t = j + base + lane;
                const int64_t w = j - (t - W + 1);
                const float p = expf(x - __ldg(lse + t * H + h));
                ds = __ldg(c + t * H + h) * p * (__ldg(dPband + t * W + w) - __ldg(dc + t * H + h));
                pg = ldf<T>(pmap + t * W + w) * __ldg(g + t * H + h);
            }
            const int cnt = min(32, n - base);
#pragma unroll 8
            for (int l = 0; l < cnt; ++l) {
                const float dsl = __shfl_sync(0xffffffffu, ds, l);
                const float pgl = __shfl_sync(0xffffffffu, pg, l);
                const int64_t t = j + base + l;
                const T *qr = q + t * s.sq + h * d;
                const T *dr = dO + t * s.so + h * d;
#pragma unroll
                for (int i = 0; i < DPL; ++i) {
                    ak[i] = fmaf(dsl, ldf<T>(qr + lane + 32 * i), ak[i]);
                    av[i] = fmaf(pgl, ldf<T>(dr + lane + 32 * i), av[i]);
                }
            }
        }
#pragma unroll
        for (int i = 0; i < DPL; ++i) {
            stf<T>(dk + j * s.sdq + h * d + lane + 32 * i, s.scale * ak[i]);
            stf<T>(dv + j * s.sdq + h * d + lane + 32 * i, av[i]);
        }
    }
}

}  // namespace simt
}  // namespace dc
