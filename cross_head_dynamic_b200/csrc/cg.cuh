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
// of x: at 2H = 12 the FMA issue of the CUDA cores and the HBM stream take about the same
// time, so the kernels are written to spend few instructions per FMA.  They use the
// packed fma.rn.f32x2 of sm_100 (two IEEE fp32 FMAs, each rounded to nearest, so the
// result is that of two scalar FMAs in the same order), keep the weight in shared memory
// and move x through shared memory with asynchronous copies.
//
// Outputs are padded to OUT in {8, 12, 16, 24, 32} (>= 2H; padded weight rows and padded
// entries of e are zero).  The weight sits in shared memory as pair-rows: pair-row p holds
// weight[0..OUT-1][2p] then weight[0..OUT-1][2p + 1], padded to kWRow(OUT) floats so that
// the 32 lanes' 16-byte reads of consecutive pair-rows hit distinct banks.
//
// dweight and dbias are reduced deterministically: each block of the partial kernel sums
// a fixed token range into its own record of the workspace; the reduce kernel adds the
// records in a fixed order.  The result depends only on N, never on timing.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace dc {
namespace cg {

constexpr int kThreads = 256;             // forward and dx blocks: 8 warps
constexpr int kDwThreads = 384;           // dweight partial blocks: 12 warps
__host__ __device__ constexpr int dw_units(int OUT) { return OUT <= 12 ? 2 : 1; }   // column pairs per thread, per pass
constexpr size_t kMaxSmem = 227 * 1024;   // dynamic shared memory a block may have
constexpr size_t kDwStageBudget = 100 * 1024;   // one of the dweight kernel's two stages
constexpr int kStages = 6;                // depth of each warp's ring of x stages in the forward
constexpr int kReduceThreads = 512;

struct CgShape {
    int64_t N;
    int D;      // even
    int H;      // 1..16
    int64_t sx;    // elements between tokens of x
    int64_t sdx;   // elements between tokens of dx
};

__host__ __device__ constexpr int out_pad(int H2) { return H2 <= 8 ? 8 : H2 <= 12 ? 12 : H2 <= 16 ? 16 : H2 <= 24 ? 24 : 32; }
__host__ __device__ constexpr int tokens_per_warp(int OUT) { return 64 / OUT; }
__host__ __device__ constexpr int kWRow(int OUT) { return 2 * OUT + 4; }
__host__ __device__ inline size_t weight_smem_bytes(int D, int H) {
    return sizeof(float) * (size_t)(D / 2) * kWRow(out_pad(2 * H));
}

// Shared memory of the forward: the weight, then per warp kStages stages of TPW x 64
// elements of x.
template <typename T>
__host__ __device__ inline size_t fwd_smem_bytes(int D, int H) {
    const int OUT = out_pad(2 * H);
    return weight_smem_bytes(D, H) + sizeof(T) * (size_t)(kThreads / 32) * kStages * tokens_per_warp(OUT) * 64;
}

// Tokens per stage of the dweight kernel, and its shared memory (two stages of x rows
// and of e rows stored as broadcast pairs (e, e)).
inline int dw_chunk(int D, int H, size_t esize) {
    const size_t per_token = esize * (size_t)D + 8 * (size_t)out_pad(2 * H);
    const size_t c = kDwStageBudget / per_token;
    return (int)(c > 64 ? 64 : c < 1 ? 1 : c);
}
__host__ __device__ inline size_t dw_xbytes(int chunk, int D, size_t esize) {
    return (esize * (size_t)chunk * D + 15) / 16 * 16;   // e stages follow on a 16-byte boundary
}
inline size_t dw_smem_bytes(int D, int H, size_t esize) {
    const int chunk = dw_chunk(D, H, esize);
    return 2 * dw_xbytes(chunk, D, esize) + 2 * sizeof(float) * 2 * (size_t)chunk * out_pad(2 * H);
}

// Number of partial records (blocks of the dweight kernel, one wave of one block per SM)
// for N tokens, and the floats in one record: dweight [2H][D] then dbias [2H].
constexpr int kMaxPartials = 148;
inline int partial_blocks(int64_t N) {
    const int64_t want = (N + 63) / 64;
    return (int)(want < 1 ? 1 : want > kMaxPartials ? kMaxPartials : want);
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
// The two elements of a pair, each broadcast to both halves.
__device__ __forceinline__ void split_bcast(f2reg v, f2reg &lo, f2reg &hi) {
    const float2 f = unpack2(v);
    lo = pack2(f.x, f.x);
    hi = pack2(f.y, f.y);
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

// weight [2H][D] into the pair-row layout, as 4-byte asynchronous copies (rows 2H..OUT-1
// zero), committed as one group.  Reads are coalesced along k.
template <int OUT>
__device__ __forceinline__ void stage_weight(const CgShape &s, const float *__restrict__ weight, float *ws) {
    constexpr int WR = kWRow(OUT);
#pragma unroll 1
    for (int o = 0; o < OUT; ++o) {
        const float *src = weight + (int64_t)o * s.D;
        for (int k = threadIdx.x; k < s.D; k += blockDim.x) {
            float *dst = ws + (k >> 1) * WR + (k & 1) * OUT + o;
            if (o < 2 * s.H)
                cp_async4(dst, src + k);
            else
                *dst = 0.f;
        }
    }
    cp_async_commit();
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

// Elements [k0, k0 + 64) of TPW consecutive x rows (rows past N zero-filled) into one ring
// stage [TPW][64].  vec16: every row start is 16-byte aligned and D * sizeof(T) is a
// multiple of 16, so 16-byte copies cover the rows exactly; otherwise 4-byte copies.
template <typename T, int TPW>
__device__ __forceinline__ void copy_stage(const CgShape &s, const T *__restrict__ x, int64_t t0, int k0, T *st,
                                           int lane, bool vec16) {
    const int kn = s.D - k0 < 64 ? s.D - k0 : 64;
    if (vec16) {
        constexpr int E = 16 / (int)sizeof(T);
        constexpr int CPR = 64 / E;   // 16-byte chunks per stage row (a power of two)
#pragma unroll
        for (int c = 0; c < (TPW * CPR + 31) / 32; ++c) {
            const int i = lane + 32 * c;
            const int j = i / CPR, q = i % CPR;
            if (i < TPW * CPR && q * E < kn) {
                T *dst = st + j * 64 + q * E;
                if (t0 + j < s.N)
                    cp_async16(dst, x + (t0 + j) * s.sx + k0 + q * E);
                else
                    *reinterpret_cast<float4 *>(dst) = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
    } else {
        constexpr int E = 4 / (int)sizeof(T);
        constexpr int CPR = 64 / E;   // 4-byte chunks per stage row
#pragma unroll
        for (int c = 0; c < (TPW * CPR + 31) / 32; ++c) {
            const int i = lane + 32 * c;
            const int j = i / CPR, q = i % CPR;
            if (i < TPW * CPR && q * E < kn) {
                T *dst = st + j * 64 + q * E;
                if (t0 + j < s.N)
                    cp_async4(dst, x + (t0 + j) * s.sx + k0 + q * E);
                else
                    *reinterpret_cast<uint32_t *>(dst) = 0u;
            }
        }
    }
}

// c, g.  Work item = (group of TPW tokens, k-step of 64 elements); each warp walks its
// items (its groups grid-strided, each group's k-steps in order) with kStages - 1 items'
// copies in flight.  Lane l of k-step s takes the column pair k = 64 s + 2 l: for each
// token j and output pair (2q, 2q + 1) one packed FMA per column.  Slot j * OUT + o of the
// partial sums is token t0 + j, output o; a reduce-scatter over the warp ends a group.
template <typename T, int OUT>
__global__ void __launch_bounds__(kThreads, 2) cg_fwd_kernel(CgShape s, const T *__restrict__ x,
                                                            const float *__restrict__ weight,
                                                            const float *__restrict__ bias, float *__restrict__ c,
                                                            float *__restrict__ g, int vec16) {
    constexpr int TPW = tokens_per_warp(OUT);
    constexpr int STAGE = TPW * 64;
    constexpr int WR = kWRow(OUT);
    extern __shared__ __align__(16) unsigned char smem[];
    float *ws = reinterpret_cast<float *>(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    T *ring = reinterpret_cast<T *>(smem + weight_smem_bytes(s.D, s.H)) + warp * kStages * STAGE;
    const int ksn = (s.D + 63) / 64;
    const int64_t ngroups = (s.N + TPW - 1) / TPW;
    const int64_t wid = (int64_t)blockIdx.x * (kThreads / 32) + warp, nwarps = (int64_t)gridDim.x * (kThreads / 32);
    const int64_t items = wid < ngroups ? (ngroups - wid + nwarps - 1) / nwarps * ksn : 0;
    const int64_t tstep = nwarps * TPW;
    // issue cursor: item, its group's first token, its k-step, its ring stage
    int64_t iss = 0, iss_t0 = wid * TPW;
    int iss_ks = 0, iss_st = 0;
    auto issue = [&]() {
        if (iss < items) copy_stage<T, TPW>(s, x, iss_t0, iss_ks * 64, ring + iss_st * STAGE, lane, vec16 != 0);
        cp_async_commit();   // one group per item, empty past the end, so the counts stay uniform
        ++iss;
        iss_st = iss_st + 1 == kStages ? 0 : iss_st + 1;
        if (++iss_ks == ksn) {
            iss_ks = 0;
            iss_t0 += tstep;
        }
    };
    stage_weight<OUT>(s, weight, ws);
#pragma unroll 1
    for (int i = 0; i < kStages - 1; ++i) issue();
    cp_async_wait<kStages - 1>();   // the weight group (the oldest) has landed
    __syncthreads();
    const int H2 = 2 * s.H;
    // acc2[j * OUT/2 + q] = partial sums of (output 2q, output 2q + 1) for token j
    f2reg acc2[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) acc2[i] = 0ull;
    int64_t t0 = wid * TPW;
    int ks = 0, st_i = 0;
#pragma unroll 1
    for (int64_t it = 0; it < items; ++it) {
        issue();
        cp_async_wait<kStages - 1>();   // item `it` has landed (this lane's copies) ...
        __syncwarp();                   // ... and every lane's
        const T *st = ring + st_i * STAGE;
        const int p = ks * 32 + lane;   // column pair
        if (2 * p < s.D) {
            // (weight[2q][2p], weight[2q+1][2p]) for q < OUT/2, then the same for column 2p + 1
            const ulonglong2 *w2 = reinterpret_cast<const ulonglong2 *>(ws + p * WR);
            f2reg wv[OUT];
#pragma unroll
            for (int i = 0; i < OUT / 2; ++i) {
                const ulonglong2 t = w2[i];
                wv[2 * i] = t.x;
                wv[2 * i + 1] = t.y;
            }
#pragma unroll
            for (int j = 0; j < TPW; ++j) {
                f2reg xa, xb;
                split_bcast(ldpair<T>(st + j * 64 + 2 * lane), xa, xb);
#pragma unroll
                for (int q = 0; q < OUT / 2; ++q) acc2[j * (OUT / 2) + q] = ffma2(xa, wv[q], acc2[j * (OUT / 2) + q]);
#pragma unroll
                for (int q = 0; q < OUT / 2; ++q)
                    acc2[j * (OUT / 2) + q] = ffma2(xb, wv[OUT / 2 + q], acc2[j * (OUT / 2) + q]);
            }
        }
        __syncwarp();   // the stage is free for the copy issued next iteration
        st_i = st_i + 1 == kStages ? 0 : st_i + 1;
        if (++ks == ksn) {
            float acc[64];
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const float2 v = unpack2(acc2[i]);
                acc[2 * i] = v.x;
                acc[2 * i + 1] = v.y;
                acc2[i] = 0ull;
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
            ks = 0;
            t0 += tstep;
        }
    }
    cp_async_wait<0>();
}

// dx for TPW tokens per warp at a time.  e of the group's tokens is held as output pairs
// (e[2q], e[2q + 1]); lane l of k-step s takes the column pair k = 64 s + 2 l and forms
// for each token one packed FMA per output pair and column, then adds the two halves.
// The TPW * H values of dc (and of dg) a group needs are contiguous; lane l loads entry l
// of each, one group ahead, and the warp reads them by shuffle.
template <typename T, int OUT>
__global__ void __launch_bounds__(kThreads) cg_bwd_dx_kernel(CgShape s, const float *__restrict__ weight,
                                                            const float *__restrict__ dc,
                                                            const float *__restrict__ dg, T *__restrict__ dx) {
    constexpr int TPW = tokens_per_warp(OUT);
    constexpr int WR = kWRow(OUT);
    extern __shared__ __align__(16) unsigned char smem[];
    float *ws = reinterpret_cast<float *>(smem);
    stage_weight<OUT>(s, weight, ws);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t step = (int64_t)gridDim.x * (kThreads / 32) * TPW;
    auto load_e = [&](int64_t t0, float &a, float &b) {
        const int64_t i = t0 * s.H + lane;
        const bool have = t0 < s.N && lane < TPW * s.H && i < s.N * s.H;
        a = have ? __ldg(dc + i) : 0.f;
        b = have ? __ldg(dg + i) : 0.f;
    };
    int64_t t0 = ((int64_t)blockIdx.x * (kThreads / 32) + warp) * TPW;
    float na, nb;
    load_e(t0, na, nb);
    cp_async_wait<0>();
    __syncthreads();
#pragma unroll 1
    for (; t0 < s.N; t0 += step) {
        const float a = na, b = nb;
        load_e(t0 + step, na, nb);
        float e[TPW][OUT];
#pragma unroll
        for (int j = 0; j < TPW; ++j)
#pragma unroll
            for (int o = 0; o < OUT; ++o) {
                // Source lanes are warp-uniform; entries past 2H are zero.
                const int src = j * s.H + (o < s.H ? o : o - s.H);
                const float va = __shfl_sync(0xffffffffu, a, src & 31);
                const float vb = __shfl_sync(0xffffffffu, b, src & 31);
                e[j][o] = o < s.H ? va : (o < 2 * s.H ? vb : 0.f);
            }
        f2reg e2[TPW][OUT / 2];   // (e[2q], e[2q + 1])
#pragma unroll
        for (int j = 0; j < TPW; ++j)
#pragma unroll
            for (int q = 0; q < OUT / 2; ++q) e2[j][q] = pack2(e[j][2 * q], e[j][2 * q + 1]);
        const int nrows = (int)(s.N - t0 < TPW ? s.N - t0 : TPW);
#pragma unroll 1
        for (int p = lane; 2 * p < s.D; p += 32) {
            const ulonglong2 *w2 = reinterpret_cast<const ulonglong2 *>(ws + p * WR);
            f2reg wv[OUT];
#pragma unroll
            for (int i = 0; i < OUT / 2; ++i) {
                const ulonglong2 t = w2[i];
                wv[2 * i] = t.x;
                wv[2 * i + 1] = t.y;
            }
#pragma unroll
            for (int j = 0; j < TPW; ++j) {
                f2reg a0 = 0ull, a1 = 0ull;
#pragma unroll
                for (int q = 0; q < OUT / 2; ++q) {
                    a0 = ffma2(e2[j][q], wv[q], a0);
                    a1 = ffma2(e2[j][q], wv[OUT / 2 + q], a1);
                }
                const float2 r0 = unpack2(a0), r1 = unpack2(a1);
                if (j < nrows) st2<T>(dx + (t0 + j) * s.sdx + 2 * p, make_float2(r0.x + r0.y, r1.x + r1.y));
            }
        }
    }
}

// Partial dweight and dbias of the token range [blockIdx.x * span, +span) into record
// blockIdx.x of `part`.  Thread i takes the column pairs p = i, i + kDwThreads (dw_units
// of them per pass over the columns).  Tokens go through shared memory `chunk` at a time,
// double-buffered with asynchronous copies: the x rows, and e as broadcast pairs (e, e)
// so that one packed FMA per output adds e[o] * (x[2p], x[2p + 1]).  dbias: the threads
// o < 2H add the e column o.
template <typename T, int OUT>
__global__ void __launch_bounds__(kDwThreads) cg_bwd_dw_partial_kernel(CgShape s, int64_t span, int chunk,
                                                                      const T *__restrict__ x,
                                                                      const float *__restrict__ dc,
                                                                      const float *__restrict__ dg,
                                                                      float *__restrict__ part, int vec16) {
    extern __shared__ __align__(16) unsigned char smem[];
    const size_t xbytes = dw_xbytes(chunk, s.D, sizeof(T));
    const size_t ebytes = sizeof(float2) * (size_t)chunk * OUT;
    auto xs = [&](int b) { return reinterpret_cast<T *>(smem + b * xbytes); };
    auto es = [&](int b) { return reinterpret_cast<float2 *>(smem + 2 * xbytes + b * ebytes); };
    const int H2 = 2 * s.H;
    const int tid = threadIdx.x;
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
    auto issue = [&](int ci) {
        if (ci < nchunks) {
            const int64_t tc = ta + (int64_t)ci * chunk;
            const int nt = rows_of(ci);
            T *xd = xs(ci & 1);
            float2 *ed = es(ci & 1);
            if (vec16) {
                constexpr int E = 16 / (int)sizeof(T);
                const int cpr = s.D / E;
                for (int i = tid; i < nt * cpr; i += kDwThreads) {
                    const int r = i / cpr, q = i - r * cpr;
                    cp_async16(xd + r * s.D + q * E, x + (tc + r) * s.sx + q * E);
                }
            } else {
                constexpr int E = 4 / (int)sizeof(T);
                const int cpr = s.D / E;
                for (int i = tid; i < nt * cpr; i += kDwThreads) {
                    const int r = i / cpr, q = i - r * cpr;
                    cp_async4(xd + r * s.D + q * E, x + (tc + r) * s.sx + q * E);
                }
            }
            for (int i = tid; i < chunk * OUT; i += kDwThreads) {
                const int r = i / OUT, o = i - r * OUT;
                float *d2 = reinterpret_cast<float *>(ed + i);
                if (r < nt && o < H2) {
                    const float *src = o < s.H ? dc + (tc + r) * s.H + o : dg + (tc + r) * s.H + o - s.H;
                    cp_async4(d2, src);
                    cp_async4(d2 + 1, src);
                } else {
                    d2[0] = 0.f;
                    d2[1] = 0.f;
                }
            }
        }
        cp_async_commit();
    };
    constexpr int UPT = dw_units(OUT);
    for (int ug = 0; ug < pairs; ug += kDwThreads * UPT) {
        f2reg acc[UPT][OUT];   // (dweight[o][2p], dweight[o][2p + 1])
#pragma unroll
        for (int u = 0; u < UPT; ++u)
#pragma unroll
            for (int o = 0; o < OUT; ++o) acc[u][o] = 0ull;
        float dbacc = 0.f;
        __syncthreads();   // the previous pass's readers are done with both buffers
        issue(0);
#pragma unroll 1
        for (int ci = 0; ci < nchunks; ++ci) {
            issue(ci + 1);
            cp_async_wait<1>();
            __syncthreads();
            const int nt = rows_of(ci);
            const T *xc = xs(ci & 1);
            const float2 *ec = es(ci & 1);
#pragma unroll
            for (int u = 0; u < UPT; ++u) {
                const int p = ug + u * kDwThreads + tid;
                if (ug + u * kDwThreads < pairs) {   // block-uniform test first, then the thread's
#pragma unroll 2
                    for (int r = 0; r < nt; ++r) {
                        const f2reg xv = p < pairs ? ldpair<T>(xc + r * s.D + 2 * p) : 0ull;
                        const ulonglong2 *e2 = reinterpret_cast<const ulonglong2 *>(ec + r * OUT);
#pragma unroll
                        for (int o2 = 0; o2 < OUT / 2; ++o2) {
                            const ulonglong2 ev = e2[o2];   // (e[2 o2], e[2 o2]), (e[2 o2 + 1], e[2 o2 + 1])
                            acc[u][2 * o2] = ffma2(ev.x, xv, acc[u][2 * o2]);
                            acc[u][2 * o2 + 1] = ffma2(ev.y, xv, acc[u][2 * o2 + 1]);
                        }
                    }
                }
            }
            if (ug == 0 && tid < H2)
                for (int r = 0; r < nt; ++r) dbacc += ec[r * OUT + tid].x;
            __syncthreads();   // buffer ci & 1 is free for chunk ci + 2
        }
        cp_async_wait<0>();
#pragma unroll
        for (int u = 0; u < UPT; ++u) {
            const int p = ug + u * kDwThreads + tid;
            if (p < pairs) {
#pragma unroll
                for (int o = 0; o < OUT; ++o)
                    if (o < H2) *reinterpret_cast<f2reg *>(rec + (int64_t)o * s.D + 2 * p) = acc[u][o];
            }
        }
        if (ug == 0 && tid < H2) rec[(int64_t)H2 * s.D + tid] = dbacc;
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
