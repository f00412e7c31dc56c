// cg.cuh -- producer of the composition weights c and the head scales g, and its
// gradients (CUDA cores, fp32 arithmetic).
//
// The form is an assumption: the m.aitntnews.com post (section "第二刀-砍层内", the
// DCMHA paragraph) says only that the heads' combination is decided dynamically from the
// current input.  The plainest reading is a per-token affine map of the layer's hidden
// state x [N][D].  With weight [2H][D] (row o produces output o) and bias [2H], fp32:
//   c[t,h] = bias[h]     + sum_k x[t,k] weight[h][k]
//   g[t,h] = bias[H + h] + sum_k x[t,k] weight[H + h][k]
// and, for dL/dc = dc, dL/dg = dg, writing e[t] = (dc[t,0..H-1], dg[t,0..H-1]):
//   dx[t,k] = sum_o e[t,o] weight[o][k],  dweight[o][k] = sum_t e[t,o] x[t,k],  dbias[o] = sum_t e[t,o]
//
// The map reads x once (1.5 KB per token at D = 768 in bf16) and does 2H FMAs per element
// of x, an fp32 FMA count on the CUDA cores that takes about as long as the HBM stream at
// 2H = 12, so the kernels spend few instructions per FMA.  The forward and dx use the
// packed fma.rn.f32x2 of sm_100 (two IEEE fp32 FMAs, each rounded to nearest, so the result
// is that of two scalar FMAs in the same order) on pairs of adjacent columns, with the
// weight in shared memory read as broadcasts, and give each lane whole tokens (no
// reduction across lanes).  dweight gives each thread column pairs and walks the tokens
// with scalar FMAs: there the packed form needs each x pair moved into a 64-bit register
// pair, which cost as many instructions as it saved (measured).
//
// Outputs are padded to OUT in {8, 12, 16, 24, 32} (>= 2H; padded weight rows and padded
// entries of e are zero).
//
// dweight and dbias are reduced deterministically: each block of the partial kernel sums
// a fixed token range into its own record of the workspace; the reduce kernel adds the
// records in a fixed order.  The result depends only on N, never on timing.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace dc {
namespace cg {

constexpr int kThreads = 256;             // forward and dx blocks: 8 warps, one per column slice
constexpr int kDwThreads = 384;           // dweight partial blocks: 12 warps, two token groups
constexpr int kDwGroup = kDwThreads / 2;  // threads of one token group
constexpr int kDwStages = 4;              // dweight token stages in flight
__host__ __device__ constexpr int dw_ppt(int OUT) { return OUT <= 16 ? 2 : 1; }   // column pairs per thread, per pass
constexpr size_t kMaxSmem = 227 * 1024;   // dynamic shared memory a block may have
constexpr size_t kDwStageBudget = 48 * 1024;   // one of the dweight kernel's stages
constexpr int kReduceThreads = 512;

struct CgShape {
    int64_t N;
    int D;      // even
    int H;      // 1..16
    int64_t sx;    // elements between tokens of x
    int64_t sdx;   // elements between tokens of dx
};

__host__ __device__ constexpr int out_pad(int H2) { return H2 <= 8 ? 8 : H2 <= 12 ? 12 : H2 <= 16 ? 16 : H2 <= 24 ? 24 : 32; }

// Tokens per stage of the dweight kernel, and its shared memory: kDwStages stages, each the
// x rows then the e rows (fp32); after the last stage the same
// bytes hold one token group's sums for the other ([kDwGroup][pairs per thread][OUT] pairs).
inline int dw_chunk(int D, int H, size_t esize) {
    const size_t per_token = esize * (size_t)D + 4 * (size_t)out_pad(2 * H);
    const size_t c = kDwStageBudget / per_token;
    return (int)(c > 64 ? 64 : c < 1 ? 1 : c);
}
__host__ __device__ inline size_t dw_xbytes(int chunk, int D, size_t esize) {
    return (esize * (size_t)chunk * D + 15) / 16 * 16;   // the e rows follow on a 16-byte boundary
}
__host__ __device__ inline size_t dw_stage_bytes(int chunk, int D, int OUT, size_t esize) {
    return dw_xbytes(chunk, D, esize) + 4 * (size_t)chunk * OUT;   // a multiple of 16 (OUT is one of 4)
}
inline size_t dw_smem_bytes(int D, int H, size_t esize) {
    const int OUT = out_pad(2 * H);
    const size_t stages = kDwStages * dw_stage_bytes(dw_chunk(D, H, esize), D, OUT, esize);
    const size_t xch = 8 * (size_t)kDwGroup * dw_ppt(OUT) * OUT;
    return stages > xch ? stages : xch;
}

// Number of partial records (blocks of the dweight kernel, one wave of one block per SM)
// for N tokens, and the floats in one record: dweight [2H][D] then dbias [2H].
constexpr int kMaxPartials = 148;
inline int partial_blocks(int64_t N) {
    const int64_t want = (N + 63) / 64;
    return (int)(want < 1 ? 1 : want > kMaxPartials ? kMaxPartials : want);
}
__host__ __device__ inline int64_t record_floats(int D, int H) { return (int64_t)2 * H * D + 2 * H; }

// Packed pairs of fp32 live in 64-bit registers (low half first), so that the register
// allocator keeps each pair in an aligned register pair and the packed FMA needs no moves.
typedef unsigned long long f2reg;

// d = (a.lo * b.lo + c.lo, a.hi * b.hi + c.hi), each an IEEE fp32 FMA rounded to nearest even.
__device__ __forceinline__ f2reg ffma2(f2reg a, f2reg b, f2reg c) {
    f2reg d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ f2reg pack2(float lo, float hi) {
    f2reg d;
    asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(lo), "f"(hi));
    return d;
}
__device__ __forceinline__ float2 unpack2(f2reg v) {
    float2 r;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
    return r;
}
// Two consecutive x elements as packed fp32 (bf16 widens exactly).
template <typename T> __device__ __forceinline__ f2reg ldpair(const T *p);
template <> __device__ __forceinline__ f2reg ldpair<float>(const float *p) { return *reinterpret_cast<const f2reg *>(p); }
template <> __device__ __forceinline__ f2reg ldpair<__nv_bfloat16>(const __nv_bfloat16 *p) {
    const unsigned w = *reinterpret_cast<const unsigned *>(p);
    return pack2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}
// Shared-memory loads at 32-bit shared addresses (a loop steps the address by a constant
// instead of recomputing a generic pointer per load).
template <typename T> __device__ __forceinline__ float2 lds_pair(uint32_t a);
template <> __device__ __forceinline__ float2 lds_pair<float>(uint32_t a) {
    float2 v;
    asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(a));
    return v;
}
template <> __device__ __forceinline__ float2 lds_pair<__nv_bfloat16>(uint32_t a) {
    unsigned w;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(w) : "r"(a));
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}
__device__ __forceinline__ float4 lds_f4(uint32_t a) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(a));
    return v;
}
// Asynchronous global -> shared copies (cp.async; completion per thread, by group).
__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
    const unsigned d = (unsigned)__cvta_generic_to_shared(dst);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(d), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(void *dst, const void *src) {
    const unsigned d = (unsigned)__cvta_generic_to_shared(dst);
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(d), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }

// ---------------------------------------------------------------------------------------
// Forward and dx: one lane per token.  A block's 8 warps split the D columns into 8 slices
// (slice_cols each, a multiple of the item width); a tile is the 32 * TPL tokens of one
// block, lane l holding tokens l, l + 32 (TPL = 2, or 1 when OUT > 12).  An item is 32
// bytes of each of the lane's rows (16 bf16 or 8 fp32 columns).  The weight sits in shared
// memory as column pairs, wp[p * OUT + o] = (weight[o][2p], weight[o][2p + 1]); every lane of
// a warp reads the same entry (a broadcast).
// ---------------------------------------------------------------------------------------

__host__ __device__ constexpr int tok_per_lane(int OUT) { return OUT <= 12 ? 2 : 1; }
__host__ __device__ constexpr int tile_tokens(int OUT) { return 32 * tok_per_lane(OUT); }
__host__ __device__ inline int slice_cols(int D, int esize) {
    const int ic = 32 / esize;               // item width in columns
    const int per = (D + 7) / 8;
    return (per + ic - 1) / ic * ic;
}
__host__ __device__ inline size_t wp_bytes(int D, int H) { return sizeof(float) * (size_t)D * out_pad(2 * H); }
// Forward: the weight pairs, then the 8 slices' partial sums of one tile [8][OUT][tile].
__host__ __device__ inline size_t fwd_smem_bytes(int D, int H) {
    const int OUT = out_pad(2 * H);
    return wp_bytes(D, H) + sizeof(float) * 8 * (size_t)OUT * tile_tokens(OUT);
}

// weight [2H][D] into the column-pair layout (outputs 2H..OUT-1 zero); the caller
// synchronizes the block before use.
template <int OUT>
__device__ __forceinline__ void stage_weight_pairs(const CgShape &s, const float *__restrict__ weight, f2reg *wp) {
    const int H2 = 2 * s.H;
    if ((s.D & 3) == 0) {
        const int q4 = s.D / 4;
#pragma unroll
        for (int o = 0; o < OUT; ++o)
            for (int q = threadIdx.x; q < q4; q += blockDim.x) {
                const float4 v = o < H2 ? __ldg(reinterpret_cast<const float4 *>(weight + (int64_t)o * s.D) + q)
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
                wp[2 * q * OUT + o] = pack2(v.x, v.y);
                wp[(2 * q + 1) * OUT + o] = pack2(v.z, v.w);
            }
    } else {
#pragma unroll
        for (int o = 0; o < OUT; ++o)
            for (int q = threadIdx.x; q < s.D / 2; q += blockDim.x) {
                const float2 v = o < H2 ? __ldg(reinterpret_cast<const float2 *>(weight + (int64_t)o * s.D) + q)
                                        : make_float2(0.f, 0.f);
                wp[q * OUT + o] = pack2(v.x, v.y);
            }
    }
}

// 32 bytes of row `row` from column k0 into r[0..7] (zero where t >= N or past column D).
// vec16: the row start is 16-byte aligned and D is a whole number of 16-byte units.
template <typename T>
__device__ __forceinline__ void load_item(const T *__restrict__ row, bool valid, int k0, int D, bool vec16,
                                          uint32_t (&r)[8]) {
    constexpr int E16 = 16 / (int)sizeof(T), E4 = 4 / (int)sizeof(T);
    if (vec16) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (valid && k0 + c * E16 < D) v = __ldg(reinterpret_cast<const uint4 *>(row + k0 + c * E16));
            r[4 * c] = v.x;
            r[4 * c + 1] = v.y;
            r[4 * c + 2] = v.z;
            r[4 * c + 3] = v.w;
        }
    } else {
#pragma unroll
        for (int c = 0; c < 8; ++c)
            r[c] = (valid && k0 + c * E4 < D) ? __ldg(reinterpret_cast<const uint32_t *>(row + k0 + c * E4)) : 0u;
    }
}

// Column pair kp of an item as packed fp32 (x[2kp], x[2kp + 1]).
template <typename T> __device__ __forceinline__ f2reg item_pair(const uint32_t (&r)[8], int kp);
template <> __device__ __forceinline__ f2reg item_pair<__nv_bfloat16>(const uint32_t (&r)[8], int kp) {
    return pack2(__uint_as_float(r[kp] << 16), __uint_as_float(r[kp] & 0xffff0000u));
}
template <> __device__ __forceinline__ f2reg item_pair<float>(const uint32_t (&r)[8], int kp) {
    return pack2(__uint_as_float(r[2 * kp]), __uint_as_float(r[2 * kp + 1]));
}

// c, g.  Warp w accumulates, for each of its lane's tokens and each output o, the packed
// pair (sum over its slice's even columns, sum over its odd columns) of x * weight: one
// packed FMA per (token, output, column pair).  At the end of a tile the 8 slices' sums
// (even + odd) meet in shared memory and are added in slice order, then the bias.  The
// lanes' rows stream from global memory two items ahead of the arithmetic.
template <typename T, int OUT>
__global__ void __launch_bounds__(kThreads, 2) cg_fwd_kernel(CgShape s, const T *__restrict__ x,
                                                            const float *__restrict__ weight,
                                                            const float *__restrict__ bias, float *__restrict__ c,
                                                            float *__restrict__ g, int vec16) {
    constexpr int TPL = tok_per_lane(OUT);
    constexpr int TT = tile_tokens(OUT);
    constexpr int KP = 16 / (int)sizeof(T);   // column pairs per item
    extern __shared__ __align__(16) unsigned char smem[];
    f2reg *wp = reinterpret_cast<f2reg *>(smem);
    float *red = reinterpret_cast<float *>(smem + wp_bytes(s.D, s.H));   // [8][OUT][TT]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int sc = slice_cols(s.D, (int)sizeof(T));
    const int nit = sc / (32 / (int)sizeof(T));
    const int kbase = warp * sc;
    const int64_t ntiles = (s.N + TT - 1) / TT;
    const int64_t items = (int64_t)blockIdx.x < ntiles ? (ntiles - blockIdx.x + gridDim.x - 1) / gridDim.x * nit : 0;
    stage_weight_pairs<OUT>(s, weight, wp);

    // item i -> (tile, step): tiles blockIdx.x, +gridDim.x, ...; steps 0..nit-1
    auto load = [&](int64_t i, uint32_t (&r)[TPL][8]) {
        const int64_t ti = i / nit;
        const int st = (int)(i - ti * nit);
        const int64_t t0 = ((int64_t)blockIdx.x + ti * gridDim.x) * TT + lane;
        const int k0 = kbase + st * (32 / (int)sizeof(T));
#pragma unroll
        for (int j = 0; j < TPL; ++j) {
            const int64_t t = t0 + 32 * j;
            const bool valid = i < items && t < s.N;
            load_item<T>(x + (valid ? t : 0) * s.sx, valid, k0, s.D, vec16 != 0, r[j]);
        }
    };
    f2reg acc[TPL][OUT];
#pragma unroll
    for (int j = 0; j < TPL; ++j)
#pragma unroll
        for (int o = 0; o < OUT; ++o) acc[j][o] = 0ull;
    const int H2 = 2 * s.H;

    auto step = [&](int64_t i, uint32_t (&r)[TPL][8]) {
        const int64_t ti = i / nit;
        const int st = (int)(i - ti * nit);
        const int k0 = kbase + st * (32 / (int)sizeof(T));
#pragma unroll
        for (int kp = 0; kp < KP; ++kp) {
            if (k0 + 2 * kp < s.D) {   // warp-uniform
                const ulonglong2 *w2 = reinterpret_cast<const ulonglong2 *>(wp + ((k0 >> 1) + kp) * OUT);
                f2reg xp[TPL];
#pragma unroll
                for (int j = 0; j < TPL; ++j) xp[j] = item_pair<T>(r[j], kp);
#pragma unroll
                for (int q = 0; q < OUT / 2; ++q) {
                    const ulonglong2 wv = w2[q];
#pragma unroll
                    for (int j = 0; j < TPL; ++j) {
                        acc[j][2 * q] = ffma2(xp[j], wv.x, acc[j][2 * q]);
                        acc[j][2 * q + 1] = ffma2(xp[j], wv.y, acc[j][2 * q + 1]);
                    }
                }
            }
        }
        load(i + 2, r);   // this buffer's next item
        if (st == nit - 1) {   // the tile is done: every warp of the block reaches this together
#pragma unroll
            for (int j = 0; j < TPL; ++j)
#pragma unroll
                for (int o = 0; o < OUT; ++o) {
                    const float2 v = unpack2(acc[j][o]);
                    red[(warp * OUT + o) * TT + lane + 32 * j] = v.x + v.y;
                    acc[j][o] = 0ull;
                }
            __syncthreads();
            const int64_t tb = ((int64_t)blockIdx.x + ti * gridDim.x) * TT;
            for (int e = threadIdx.x; e < TT * H2; e += kThreads) {
                const int tok = e / H2, o = e - tok * H2;
                float sum = red[o * TT + tok];
#pragma unroll
                for (int w = 1; w < 8; ++w) sum += red[(w * OUT + o) * TT + tok];
                const int64_t t = tb + tok;
                if (t < s.N) {
                    const float v = sum + __ldg(bias + o);
                    if (o < s.H)
                        c[t * s.H + o] = v;
                    else
                        g[t * s.H + o - s.H] = v;
                }
            }
            __syncthreads();   // red is free for the next tile
        }
    };

    uint32_t r0[TPL][8], r1[TPL][8];
    load(0, r0);
    load(1, r1);
    __syncthreads();   // the weight pairs are staged
#pragma unroll 1
    for (int64_t i = 0; i < items; i += 2) {
        step(i, r0);
        if (i + 1 < items) step(i + 1, r1);
    }
}

// dx.  Lane per token as in the forward; for each of its tokens a lane holds e as broadcast
// pairs (e[o], e[o]) and forms each column pair of dx as one chain of packed FMAs over the
// outputs o in order: (dx[2p], dx[2p + 1]) = sum_o (e[o], e[o]) * (weight[o][2p], weight[o][2p + 1]).
template <typename T, int OUT>
__global__ void __launch_bounds__(kThreads, 2) cg_bwd_dx_kernel(CgShape s, const float *__restrict__ weight,
                                                               const float *__restrict__ dc,
                                                               const float *__restrict__ dg, T *__restrict__ dx,
                                                               int vec16) {
    constexpr int TPL = tok_per_lane(OUT);
    constexpr int TT = tile_tokens(OUT);
    constexpr int KP = 16 / (int)sizeof(T);
    constexpr int E16 = 16 / (int)sizeof(T), E4 = 4 / (int)sizeof(T);
    extern __shared__ __align__(16) unsigned char smem[];
    f2reg *wp = reinterpret_cast<f2reg *>(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int sc = slice_cols(s.D, (int)sizeof(T));
    const int nit = sc / (32 / (int)sizeof(T));
    const int kbase = warp * sc;
    const int64_t ntiles = (s.N + TT - 1) / TT;
    stage_weight_pairs<OUT>(s, weight, wp);
    __syncthreads();
    const int H2 = 2 * s.H;
#pragma unroll 1
    for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
        f2reg eb[TPL][OUT];
#pragma unroll
        for (int j = 0; j < TPL; ++j) {
            const int64_t t = tile * TT + lane + 32 * j;
#pragma unroll
            for (int o = 0; o < OUT; ++o) {
                float e = 0.f;
                if (t < s.N && o < H2) e = o < s.H ? __ldg(dc + t * s.H + o) : __ldg(dg + t * s.H + o - s.H);
                eb[j][o] = pack2(e, e);
            }
        }
#pragma unroll 1
        for (int st = 0; st < nit; ++st) {
            const int k0 = kbase + st * (32 / (int)sizeof(T));
            uint32_t out[TPL][8];
#pragma unroll
            for (int kp = 0; kp < KP; ++kp) {
                f2reg rr[TPL];
#pragma unroll
                for (int j = 0; j < TPL; ++j) rr[j] = 0ull;
                if (k0 + 2 * kp < s.D) {   // warp-uniform
                    const ulonglong2 *w2 = reinterpret_cast<const ulonglong2 *>(wp + ((k0 >> 1) + kp) * OUT);
#pragma unroll
                    for (int q = 0; q < OUT / 2; ++q) {
                        const ulonglong2 wv = w2[q];
#pragma unroll
                        for (int j = 0; j < TPL; ++j) {
                            rr[j] = ffma2(eb[j][2 * q], wv.x, rr[j]);
                            rr[j] = ffma2(eb[j][2 * q + 1], wv.y, rr[j]);
                        }
                    }
                }
#pragma unroll
                for (int j = 0; j < TPL; ++j) {
                    const float2 v = unpack2(rr[j]);
                    if constexpr (sizeof(T) == 2) {
                        const __nv_bfloat162 b2 = __floats2bfloat162_rn(v.x, v.y);
                        out[j][kp] = *reinterpret_cast<const uint32_t *>(&b2);
                    } else {
                        out[j][2 * kp] = __float_as_uint(v.x);
                        out[j][2 * kp + 1] = __float_as_uint(v.y);
                    }
                }
            }
#pragma unroll
            for (int j = 0; j < TPL; ++j) {
                const int64_t t = tile * TT + lane + 32 * j;
                if (t < s.N) {
                    T *row = dx + t * s.sdx;
                    if (vec16) {
#pragma unroll
                        for (int c = 0; c < 2; ++c)
                            if (k0 + c * E16 < s.D)
                                *reinterpret_cast<uint4 *>(row + k0 + c * E16) =
                                    make_uint4(out[j][4 * c], out[j][4 * c + 1], out[j][4 * c + 2], out[j][4 * c + 3]);
                    } else {
#pragma unroll
                        for (int c = 0; c < 8; ++c)
                            if (k0 + c * E4 < s.D) *reinterpret_cast<uint32_t *>(row + k0 + c * E4) = out[j][c];
                    }
                }
            }
        }
    }
}

// Partial dweight and dbias of the token range [blockIdx.x * span, +span) into record
// blockIdx.x of `part`.  The block's two token groups of kDwGroup threads take the even and
// the odd tokens of every stage; within a group, thread i takes the column pairs
// i + k * kDwGroup (k < dw_ppt(OUT)) of each pass over the columns (a warp's reads of one
// row are then consecutive words), so one broadcast read of four e values feeds
// 4 * 2 * dw_ppt(OUT) scalar FMAs.
// Tokens go through shared memory `chunk` at a time in a ring of kDwStages stages filled
// by asynchronous copies (the x rows and the e rows).  At the end of a pass the odd
// group's sums are added to the even group's in shared memory, in that order.
// dbias: lane o of warp w adds e column o of the tokens w, w + 12, ... of every stage; the
// 12 warp sums are then added in warp order.  Every assignment is fixed, so the record is
// bitwise reproducible.
template <typename T, int OUT>
__global__ void __launch_bounds__(kDwThreads) cg_bwd_dw_partial_kernel(CgShape s, int64_t span, int chunk,
                                                                      const T *__restrict__ x,
                                                                      const float *__restrict__ dc,
                                                                      const float *__restrict__ dg,
                                                                      float *__restrict__ part, int vec16) {
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ float dbred[kDwThreads / 32][32];
    constexpr int PPT = dw_ppt(OUT);
    constexpr int NW = kDwThreads / 32;
    const size_t xbytes = dw_xbytes(chunk, s.D, sizeof(T));
    const size_t sbytes = dw_stage_bytes(chunk, s.D, OUT, sizeof(T));
    auto xs = [&](int b) { return reinterpret_cast<T *>(smem + b * sbytes); };
    auto es = [&](int b) { return reinterpret_cast<float *>(smem + b * sbytes + xbytes); };
    const int H2 = 2 * s.H;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int grp = tid / kDwGroup, tg = tid - grp * kDwGroup;
    const int64_t ta = (int64_t)blockIdx.x * span;
    const int64_t tb = ta + span < s.N ? ta + span : s.N;
    const int64_t ntok = tb > ta ? tb - ta : 0;
    const int nchunks = (int)((ntok + chunk - 1) / chunk);
    float *rec = part + (int64_t)blockIdx.x * record_floats(s.D, s.H);
    const int pairs = s.D / 2;
    auto rows_of = [&](int ci) {
        const int64_t left = ntok - (int64_t)ci * chunk;
        return (int)(left < chunk ? left : chunk);
    };
    // stage ci % kDwStages <- chunk ci (nothing past the last chunk); always one commit group
    auto issue = [&](int ci) {
        if (ci < nchunks) {
            const int64_t tc = ta + (int64_t)ci * chunk;
            const int nt = rows_of(ci);
            T *xd = xs(ci % kDwStages);
            float *ed = es(ci % kDwStages);
            for (int r = warp; r < nt; r += NW) {
                const T *src = x + (tc + r) * s.sx;
                T *dst = xd + r * s.D;
                if (vec16) {
                    constexpr int E = 16 / (int)sizeof(T);
                    for (int q = lane; q < s.D / E; q += 32) cp_async16(dst + q * E, src + q * E);
                } else {
                    constexpr int E = 4 / (int)sizeof(T);
                    for (int q = lane; q < s.D / E; q += 32) cp_async4(dst + q * E, src + q * E);
                }
            }
            for (int i = tid; i < chunk * OUT; i += kDwThreads) {
                const int r = i / OUT, o = i - r * OUT;
                if (r < nt && o < H2)
                    cp_async4(ed + i, o < s.H ? dc + (tc + r) * s.H + o : dg + (tc + r) * s.H + o - s.H);
                else
                    ed[i] = 0.f;
            }
        }
        cp_async_commit();
    };
    float dbacc = 0.f;
    for (int pg = 0; pg < pairs; pg += kDwGroup * PPT) {
        // this thread's pairs; one past the end reads the last pair (always in bounds) and is not written
        int pk[PPT];
#pragma unroll
        for (int k = 0; k < PPT; ++k) pk[k] = min(pg + tg + k * kDwGroup, pairs - 1);
        float acc[PPT][OUT][2];   // (dweight[o][2p], dweight[o][2p + 1]) of pair k
#pragma unroll
        for (int k = 0; k < PPT; ++k)
#pragma unroll
            for (int o = 0; o < OUT; ++o) acc[k][o][0] = acc[k][o][1] = 0.f;
        __syncthreads();   // the previous pass's readers are done with every stage
        for (int ci = 0; ci < kDwStages - 1; ++ci) issue(ci);
#pragma unroll 1
        for (int ci = 0; ci < nchunks; ++ci) {
            issue(ci + kDwStages - 1);
            cp_async_wait<kDwStages - 1>();   // chunk ci has landed (groups complete in order)
            __syncthreads();
            const int nt = rows_of(ci);
            const T *xc = xs(ci % kDwStages);
            const float *ec = es(ci % kDwStages);
            // shared addresses of this group's first token: its x pairs and its e row
            uint32_t xa[PPT];
#pragma unroll
            for (int k = 0; k < PPT; ++k)
                xa[k] = (uint32_t)__cvta_generic_to_shared(xc + grp * s.D + 2 * pk[k]);
            uint32_t ea = (uint32_t)__cvta_generic_to_shared(ec + grp * OUT);
            const uint32_t xstep = 2u * (uint32_t)s.D * (uint32_t)sizeof(T);   // two tokens
#pragma unroll(OUT > 16 ? 1 : 2)
            for (int r = grp; r < nt; r += 2) {
                float2 xv[PPT];
#pragma unroll
                for (int k = 0; k < PPT; ++k) {
                    xv[k] = lds_pair<T>(xa[k]);
                    xa[k] += xstep;
                }
#pragma unroll
                for (int o4 = 0; o4 < OUT / 4; ++o4) {
                    const float4 ev = lds_f4(ea + 16u * o4);
                    const float e[4] = {ev.x, ev.y, ev.z, ev.w};
#pragma unroll
                    for (int j = 0; j < 4; ++j)
#pragma unroll
                        for (int k = 0; k < PPT; ++k) {
                            acc[k][4 * o4 + j][0] = fmaf(e[j], xv[k].x, acc[k][4 * o4 + j][0]);
                            acc[k][4 * o4 + j][1] = fmaf(e[j], xv[k].y, acc[k][4 * o4 + j][1]);
                        }
                }
                ea += 2u * OUT * 4u;
            }
            if (pg == 0 && lane < H2)
                for (int r = warp; r < nt; r += NW) dbacc += ec[r * OUT + lane];
            __syncthreads();   // stage ci % kDwStages is free for chunk ci + kDwStages
        }
        cp_async_wait<0>();   // only empty groups can remain
        __syncthreads();
        // the odd group's sums to shared memory (the stage bytes, [pair k][output o][thread]),
        // then the even group adds them
        float2 *xch = reinterpret_cast<float2 *>(smem);
        if (grp == 1) {
#pragma unroll
            for (int k = 0; k < PPT; ++k)
#pragma unroll
                for (int o = 0; o < OUT; ++o) xch[(k * OUT + o) * kDwGroup + tg] = make_float2(acc[k][o][0], acc[k][o][1]);
        }
        __syncthreads();
        if (grp == 0) {
#pragma unroll
            for (int k = 0; k < PPT; ++k) {
                const int p = pg + tg + k * kDwGroup;
                if (p < pairs) {
#pragma unroll
                    for (int o = 0; o < OUT; ++o) {
                        if (o < H2) {
                            const float2 b = xch[(k * OUT + o) * kDwGroup + tg];
                            *reinterpret_cast<float2 *>(rec + (int64_t)o * s.D + 2 * p) =
                                make_float2(acc[k][o][0] + b.x, acc[k][o][1] + b.y);
                        }
                    }
                }
            }
        }
    }
    dbred[warp][lane] = dbacc;
    __syncthreads();
    if (tid < H2) {
        float tot = dbred[0][tid];
#pragma unroll
        for (int w = 1; w < NW; ++w) tot += dbred[w][tid];
        rec[(int64_t)H2 * s.D + tid] = tot;
    }
}

// dweight, dbias = the sum of the `blocks` records.  A block takes 32 consecutive record
// entries: lane = entry; warp w loads records w, w + 16, ... all at once (a fixed, fully
// predicated batch, absent records read as 0) and adds them in that order; the 16 warp
// sums are then added in warp order.  blocks = 0 writes zeros.
__global__ void __launch_bounds__(kReduceThreads) cg_bwd_dw_reduce_kernel(CgShape s, int blocks,
                                                                         const float *__restrict__ part,
                                                                         float *__restrict__ dweight,
                                                                         float *__restrict__ dbias) {
    constexpr int NW = kReduceThreads / 32;
    constexpr int PER = (kMaxPartials + NW - 1) / NW;
    __shared__ float red[NW][32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t n = record_floats(s.D, s.H);
    const int64_t i = (int64_t)blockIdx.x * 32 + lane;
    float v[PER];
#pragma unroll
    for (int r = 0; r < PER; ++r) {
        const int b = warp + r * NW;
        v[r] = (i < n && b < blocks) ? __ldg(part + (int64_t)b * n + i) : 0.f;
    }
    float sum = v[0];
#pragma unroll
    for (int r = 1; r < PER; ++r) sum += v[r];
    red[warp][lane] = sum;
    __syncthreads();
    if (warp == 0 && i < n) {
        float tot = red[0][lane];
#pragma unroll
        for (int w = 1; w < NW; ++w) tot += red[w][lane];
        const int64_t nw = (int64_t)2 * s.H * s.D;
        if (i < nw)
            dweight[i] = tot;
        else
            dbias[i - nw] = tot;
    }
}

}  // namespace cg
}  // namespace dc
