// common.cuh -- device helpers shared by all libdcattn kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "dcattn.h"

namespace dc {

// Per-device status word (DC_DEVERR_* bits); read and cleared by dc_attn_device_status.
__device__ unsigned int g_status;

__device__ __forceinline__ void raise_status(unsigned int bits) { atomicOr(&g_status, bits); }

// Plain-old-data copy of the public params that kernels take by value.
struct Shape {
    int64_t N;
    int num_docs;
    int H;
    int d;
    int W;
    float scale;
    const int32_t *cu;
    int64_t sq;         // elements between consecutive tokens of q, k, v (>= H * d)
    int64_t sdq;        // ... of dq, dk, dv
    int64_t so;         // ... of o (forward) and dO (backward)
    uint32_t wait_ns;   // limit of every bounded wait in the tcgen05 kernels (nanoseconds)
    int inject;         // test hook: the tcgen05 forward's first CTA leaves out its first Q/K load
};

template <typename T> __device__ __forceinline__ float ldf(const T *p);
template <> __device__ __forceinline__ float ldf<float>(const float *p) { return *p; }
template <> __device__ __forceinline__ float ldf<__nv_bfloat16>(const __nv_bfloat16 *p) {
    return __bfloat162float(*p);
}
template <typename T> __device__ __forceinline__ void stf(T *p, float x);
template <> __device__ __forceinline__ void stf<float>(float *p, float x) { *p = x; }
template <> __device__ __forceinline__ void stf<__nv_bfloat16>(__nv_bfloat16 *p, float x) {
    *p = __float2bfloat16_rn(x);
}

// Document holding token t: the largest i in [0, num_docs) with cu[i] <= t.
// Any cu_seqlens content gives an index in range; callers clamp what they
// derive from it, so malformed input cannot cause out-of-bounds access.
__device__ __forceinline__ int doc_index(const int32_t *cu, int num_docs, int64_t t) {
    int lo = 0, hi = num_docs - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if ((int64_t)__ldg(cu + mid) <= t)
            lo = mid;
        else
            hi = mid - 1;
    }
    return lo;
}

// First key of query t's window: max(t-W+1, document start, 0), never above t.
__device__ __forceinline__ int64_t window_lo(const Shape &s, int64_t t) {
    int64_t a = __ldg(s.cu + doc_index(s.cu, s.num_docs, t));
    int64_t lo = t - s.W + 1;
    if (a > lo) lo = a;
    if (lo < 0) lo = 0;
    if (lo > t) lo = t;
    return lo;
}

// One past the last query that may see key j: min(document end, N), at least j+1.
__device__ __forceinline__ int64_t doc_end(const Shape &s, int64_t j) {
    int64_t b = __ldg(s.cu + doc_index(s.cu, s.num_docs, j) + 1);
    if (b > s.N) b = s.N;
    if (b < j + 1) b = j + 1;
    return b;
}

// Grid-strided check of cu_seqlens: 0-based, non-decreasing, ending at N.
__device__ __forceinline__ void validate_seqlens(const Shape &s) {
    const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t nth = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = tid; i <= s.num_docs; i += nth) {
        int v = __ldg(s.cu + i);
        bool bad = (i == 0 && v != 0) || (i == s.num_docs && (int64_t)v != s.N) ||
                   (i < s.num_docs && __ldg(s.cu + i + 1) < v);
        if (bad) raise_status(DC_DEVERR_SEQLENS);
    }
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}
__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}

}  // namespace dc
