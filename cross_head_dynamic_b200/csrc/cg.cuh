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
// The map reads x once (1.5 KB per token at D = 768 in bf16) and writes 2H floats: it
// is bound by memory and by fp32 FMA issue (2H FMAs per element of x), not a job for
// the tensor cores.  Every kernel works on pairs of x elements (k = 2 * lane + 64 * i),
// so a warp's loads of one token cover 128 contiguous bytes and its float2 reads of one
// weight row cover 256 contiguous bytes of shared memory without bank conflicts.
//
// Outputs are padded to OUT in {8, 12, 16, 24, 32} (>= 2H; padded rows of the staged
// weight and padded entries of e are zero).  One warp handles TPW = 64 / OUT tokens at
// a time so that its TPW * OUT partial sums fit one 64-slot reduce-scatter.
//
// dweight and dbias are reduced deterministically: each block of the partial kernel
// sums a fixed token range into its own record of the workspace; the reduce kernel
// adds the records in block order.  The result depends only on N, never on timing.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace dc {
namespace cg {

constexpr int kThreads = 256;             // every cg kernel: 8 warps
constexpr int kChunk = 64;                // tokens of e staged at a time by the dweight kernel
constexpr size_t kMaxWeightSmem = 200 * 1024;

struct CgShape {
    int64_t N;
    int D;      // even
    int H;      // 1..16
    int64_t sx;    // elements between tokens of x
    int64_t sdx;   // elements between tokens of dx
};

__host__ __device__ constexpr int out_pad(int H2) { return H2 <= 8 ? 8 : H2 <= 12 ? 12 : H2 <= 16 ? 16 : H2 <= 24 ? 24 : 32; }
__host__ __device__ constexpr int tokens_per_warp(int OUT) { return 64 / OUT; }
__host__ __device__ inline size_t weight_smem_bytes(int D, int H) { return sizeof(float) * (size_t)out_pad(2 * H) * D; }

// Number of partial records (blocks of the dweight kernel) for N tokens, and the floats
// in one record: dweight [2H][D] then dbias [2H].
inline int partial_blocks(int64_t N) {
    const int64_t want = (N + 63) / 64;
    return (int)(want < 1 ? 1 : want > 296 ? 296 : want);
}
__host__ __device__ inline int64_t record_floats(int D, int H) { return (int64_t)2 * H * D + 2 * H; }

template <typename T> __device__ __forceinline__ float2 ld2(const T *p);
template <> __device__ __forceinline__ float2 ld2<float>(const float *p) { return *reinterpret_cast<const float2 *>(p); }
template <> __device__ __forceinline__ float2 ld2<__nv_bfloat16>(const __nv_bfloat16 *p) {
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(p));
}
template <typename T> __device__ __forceinline__ void st2(T *p, float2 v);
template <> __device__ __forceinline__ void st2<float>(float *p, float2 v) { *reinterpret_cast<float2 *>(p) = v; }
template <> __device__ __forceinline__ void st2<__nv_bfloat16>(__nv_bfloat16 *p, float2 v) {
    *reinterpret_cast<__nv_bfloat162 *>(p) = __floats2bfloat162_rn(v.x, v.y);
}

// weight [2H][D] into shared rows [OUT][D]; rows 2H..OUT-1 are zero.
template <int OUT>
__device__ __forceinline__ void stage_weight(const CgShape &s, const float *__restrict__ weight, float *ws) {
    const int n = 2 * s.H * s.D;
    for (int i = threadIdx.x; i < OUT * s.D; i += blockDim.x) ws[i] = i < n ? __ldg(weight + i) : 0.f;
}

// One reduce-scatter step over the warp: lanes that differ in bit HALF/2 exchange halves
// of their first 2 * HALF slots; each keeps the sum of one half in slots [0, HALF).
template <int HALF>
__device__ __forceinline__ void rs_step(float (&v)[64], int lane) {
    const bool up = (lane & (HALF / 2)) != 0;
#pragma unroll
    for (int i = 0; i < HALF; ++i) {
        const float keep = up ? v[i + HALF] : v[i];
        const float send = up ? v[i] : v[i + HALF];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, HALF / 2);
    }
}
// After the five steps lane l holds in v[0], v[1] the warp-wide sums of slots 2l, 2l + 1
// (the halves kept are chosen by the lane's bits from the highest down, so the slot
// index of v[j] is 2 * l + j).  62 shuffles for 64 sums.
__device__ __forceinline__ void reduce_scatter64(float (&v)[64], int lane) {
    rs_step<32>(v, lane);
    rs_step<16>(v, lane);
    rs_step<8>(v, lane);
    rs_step<4>(v, lane);
    rs_step<2>(v, lane);
}

// c, g for TPW tokens per warp at a time (grid-strided).  Slot j * OUT + o of the
// partial sums is token t0 + j, output o.
template <typename T, int OUT>
__global__ void __launch_bounds__(kThreads, 2) cg_fwd_kernel(CgShape s, const T *__restrict__ x,
                                                         const float *__restrict__ weight,
                                                         const float *__restrict__ bias, float *__restrict__ c,
                                                         float *__restrict__ g) {
    constexpr int TPW = tokens_per_warp(OUT);
    extern __shared__ float ws[];
    stage_weight<OUT>(s, weight, ws);
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int H2 = 2 * s.H;
    for (int64_t t0 = ((int64_t)blockIdx.x * (kThreads / 32) + warp) * TPW; t0 < s.N;
         t0 += (int64_t)gridDim.x * (kThreads / 32) * TPW) {
        float acc[64];
#pragma unroll
        for (int i = 0; i < 64; ++i) acc[i] = 0.f;
        const T *xr[TPW];
#pragma unroll
        for (int j = 0; j < TPW; ++j) xr[j] = x + (t0 + j < s.N ? t0 + j : t0) * s.sx;
#pragma unroll 1
        for (int k = 2 * lane; k < s.D; k += 64) {
            float2 xv[TPW];
#pragma unroll
            for (int j = 0; j < TPW; ++j) xv[j] = t0 + j < s.N ? ld2<T>(xr[j] + k) : make_float2(0.f, 0.f);
#pragma unroll
            for (int o = 0; o < OUT; ++o) {
                const float2 wv = *reinterpret_cast<const float2 *>(ws + o * s.D + k);
#pragma unroll
                for (int j = 0; j < TPW; ++j) {
                    acc[j * OUT + o] = fmaf(xv[j].x, wv.x, acc[j * OUT + o]);
                    acc[j * OUT + o] = fmaf(xv[j].y, wv.y, acc[j * OUT + o]);
                }
            }
        }
        reduce_scatter64(acc, lane);
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
            const int slot = 2 * lane + jj;
            const int j = slot / OUT, o = slot - j * OUT;
            const int64_t t = t0 + j;
            if (j < TPW && o < H2 && t < s.N) {
                const float r = acc[jj] + __ldg(bias + o);
                if (o < s.H)
                    c[t * s.H + o] = r;
                else
                    g[t * s.H + o - s.H] = r;
            }
        }
    }
}

// dx for TPW tokens per warp at a time.  The TPW * H values of dc (and of dg) that the
// group needs are contiguous; lane l loads entry l of each and the rest of the warp
// reads them by shuffle.
template <typename T, int OUT>
__global__ void __launch_bounds__(kThreads) cg_bwd_dx_kernel(CgShape s, const float *__restrict__ weight,
                                                            const float *__restrict__ dc,
                                                            const float *__restrict__ dg, T *__restrict__ dx) {
    constexpr int TPW = tokens_per_warp(OUT);
    extern __shared__ float ws[];
    stage_weight<OUT>(s, weight, ws);
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int64_t t0 = ((int64_t)blockIdx.x * (kThreads / 32) + warp) * TPW; t0 < s.N;
         t0 += (int64_t)gridDim.x * (kThreads / 32) * TPW) {
        const int64_t base = t0 * s.H + lane;
        const bool have = lane < TPW * s.H && base < s.N * s.H;
        const float a = have ? __ldg(dc + base) : 0.f;
        const float b = have ? __ldg(dg + base) : 0.f;
        float e[TPW][OUT];
#pragma unroll
        for (int j = 0; j < TPW; ++j)
#pragma unroll
            for (int o = 0; o < OUT; ++o) {
                // Lane indices are warp-uniform; entries past 2H are zero.
                const int src = j * s.H + (o < s.H ? o : o - s.H);
                const float va = __shfl_sync(0xffffffffu, a, src & 31);
                const float vb = __shfl_sync(0xffffffffu, b, src & 31);
                e[j][o] = o < s.H ? va : (o < 2 * s.H ? vb : 0.f);
            }
#pragma unroll 2
        for (int k = 2 * lane; k < s.D; k += 64) {
            float2 acc[TPW];
#pragma unroll
            for (int j = 0; j < TPW; ++j) acc[j] = make_float2(0.f, 0.f);
#pragma unroll
            for (int o = 0; o < OUT; ++o) {
                const float2 wv = *reinterpret_cast<const float2 *>(ws + o * s.D + k);
#pragma unroll
                for (int j = 0; j < TPW; ++j) {
                    acc[j].x = fmaf(e[j][o], wv.x, acc[j].x);
                    acc[j].y = fmaf(e[j][o], wv.y, acc[j].y);
                }
            }
#pragma unroll
            for (int j = 0; j < TPW; ++j)
                if (t0 + j < s.N) st2<T>(dx + (t0 + j) * s.sdx + k, acc[j]);
        }
    }
}

// Partial dweight and dbias of the token range [blockIdx.x * span, +span) into record
// blockIdx.x of `part`.  Work units: u < D/2 is the column pair k = 2u of dweight, u = D/2
// is dbias (x taken as 1).  Each thread holds UPT units; e rows are staged kChunk tokens
// at a time and read as shared-memory broadcasts.
template <typename T, int OUT>
__global__ void __launch_bounds__(kThreads) cg_bwd_dw_partial_kernel(CgShape s, int64_t span,
                                                                    const T *__restrict__ x,
                                                                    const float *__restrict__ dc,
                                                                    const float *__restrict__ dg,
                                                                    float *__restrict__ part) {
    constexpr int UPT = 32 / OUT > 0 ? 32 / OUT : 1;
    __shared__ __align__(16) float es[kChunk][OUT];
    const int H2 = 2 * s.H;
    const int64_t ta = (int64_t)blockIdx.x * span;
    const int64_t tb = ta + span < s.N ? ta + span : s.N;
    const int units = s.D / 2 + 1;
    float *rec = part + (int64_t)blockIdx.x * record_floats(s.D, s.H);
    for (int ug = 0; ug < units; ug += kThreads * UPT) {
        float2 acc[UPT][OUT];
#pragma unroll
        for (int u = 0; u < UPT; ++u)
#pragma unroll
            for (int o = 0; o < OUT; ++o) acc[u][o] = make_float2(0.f, 0.f);
        for (int64_t tc = ta; tc < tb; tc += kChunk) {
            const int nt = (int)(tb - tc < kChunk ? tb - tc : kChunk);
            __syncthreads();   // the previous chunk's readers are done
            for (int i = threadIdx.x; i < kChunk * OUT; i += kThreads) {
                const int r = i / OUT, o = i - r * OUT;
                float v = 0.f;
                if (r < nt && o < H2) v = o < s.H ? __ldg(dc + (tc + r) * s.H + o) : __ldg(dg + (tc + r) * s.H + o - s.H);
                es[r][o] = v;
            }
            __syncthreads();
            for (int r = 0; r < nt; ++r) {
                float e[OUT];
#pragma unroll
                for (int o4 = 0; o4 < OUT / 4; ++o4) {
                    const float4 v = *reinterpret_cast<const float4 *>(&es[r][4 * o4]);
                    e[4 * o4] = v.x;
                    e[4 * o4 + 1] = v.y;
                    e[4 * o4 + 2] = v.z;
                    e[4 * o4 + 3] = v.w;
                }
#pragma unroll
                for (int u = 0; u < UPT; ++u) {
                    const int unit = ug + u * kThreads + threadIdx.x;
                    if (unit < units) {
                        const float2 xv = unit < s.D / 2 ? ld2<T>(x + (tc + r) * s.sx + 2 * unit) : make_float2(1.f, 0.f);
#pragma unroll
                        for (int o = 0; o < OUT; ++o) {
                            acc[u][o].x = fmaf(e[o], xv.x, acc[u][o].x);
                            acc[u][o].y = fmaf(e[o], xv.y, acc[u][o].y);
                        }
                    }
                }
            }
        }
#pragma unroll
        for (int u = 0; u < UPT; ++u) {
            const int unit = ug + u * kThreads + threadIdx.x;
            if (unit < s.D / 2) {
#pragma unroll
                for (int o = 0; o < OUT; ++o)
                    if (o < H2) *reinterpret_cast<float2 *>(rec + (int64_t)o * s.D + 2 * unit) = acc[u][o];
            } else if (unit == s.D / 2) {
#pragma unroll
                for (int o = 0; o < OUT; ++o)
                    if (o < H2) rec[(int64_t)H2 * s.D + o] = acc[u][o].x;
            }
        }
    }
}

// dweight, dbias = the sum of the `blocks` records, added in record order.  A block takes
// 32 consecutive record entries: lane = entry, warp w adds records w, w + 8, ...; the 8
// warp sums are then added in warp order.  blocks = 0 writes zeros.
__global__ void __launch_bounds__(kThreads) cg_bwd_dw_reduce_kernel(CgShape s, int blocks,
                                                                   const float *__restrict__ part,
                                                                   float *__restrict__ dweight,
                                                                   float *__restrict__ dbias) {
    __shared__ float red[kThreads / 32][32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t n = record_floats(s.D, s.H);
    const int64_t i = (int64_t)blockIdx.x * 32 + lane;
    float sum = 0.f;
    if (i < n)
        for (int b = warp; b < blocks; b += kThreads / 32) sum += __ldg(part + (int64_t)b * n + i);
    red[warp][lane] = sum;
    __syncthreads();
    if (warp == 0 && i < n) {
        float tot = red[0][lane];
#pragma unroll
        for (int w = 1; w < kThreads / 32; ++w) tot += red[w][lane];
        const int64_t nw = (int64_t)2 * s.H * s.D;
        if (i < nw)
            dweight[i] = tot;
        else
            dbias[i - nw] = tot;
    }
}

}  // namespace cg
}  // namespace dc
