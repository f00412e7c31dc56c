// dcattn.cu -- host side of libdcattn: argument checks, kernel selection,
// launches and the device status word.  One translation unit holds every
// kernel so the status word needs no relocatable device code.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "dcattn.h"
#include "common.cuh"
#include "simt.cuh"
#include "tc_host.cuh"
#include "cg.cuh"
#include "cg_tc.cuh"

namespace {

thread_local int32_t t_launches = 0;

// Test hooks: the limit of every bounded wait in the tcgen05 kernels launched from now
// on, and a one-shot request that the next one-piece tcgen05 forward leaves out a load.
std::atomic<uint32_t> g_wait_ns{dc::tc::kWaitNs};
std::atomic<int> g_inject{0};

struct Checked {
    dc::Shape s;
    int dtype;
    int impl;   // resolved: DC_IMPL_SIMT or DC_IMPL_TCGEN05
};

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

// Host-side argument check; fills `out` and returns DC_OK or an error.
dc_status_t check_params(const dc_attn_params *p, Checked *out) {
    if (!p) return DC_ERR_INVALID_ARG;
    if (p->dtype != DC_F32 && p->dtype != DC_BF16) return DC_ERR_INVALID_ARG;
    if (p->impl != DC_IMPL_AUTO && p->impl != DC_IMPL_SIMT && p->impl != DC_IMPL_TCGEN05)
        return DC_ERR_INVALID_ARG;
    if (p->reserved != 0) return DC_ERR_INVALID_ARG;
    if (p->total_tokens < 0 || p->total_tokens > (int64_t)INT32_MAX) return DC_ERR_INVALID_ARG;
    if (p->num_heads < 1 || p->num_heads > dc::simt::kMaxHeads) return DC_ERR_INVALID_ARG;
    if (p->head_dim < 1 || p->window < 1) return DC_ERR_INVALID_ARG;
    if (p->total_tokens > 0 && (p->num_docs < 1 || p->num_docs > p->total_tokens + 1 || !p->cu_seqlens))
        return DC_ERR_INVALID_ARG;
    if (!(p->softmax_scale == p->softmax_scale)) return DC_ERR_INVALID_ARG;   // NaN
    if (p->head_dim % 32 != 0 || p->head_dim > 128) return DC_ERR_UNSUPPORTED;
    if (p->window > 4096) return DC_ERR_UNSUPPORTED;
    out->s.N = p->total_tokens;
    out->s.num_docs = p->num_docs;
    out->s.H = p->num_heads;
    out->s.d = p->head_dim;
    out->s.W = p->window;
    out->s.scale = p->softmax_scale;
    out->s.cu = p->cu_seqlens;
    // row strides: 0 = contiguous; else at least one token's H * d elements and 16-byte rows
    const int64_t row = (int64_t)p->num_heads * p->head_dim;
    const int64_t esize = p->dtype == DC_F32 ? 4 : 2;
    const int64_t strides[3] = {p->stride_qkv, p->stride_dqkv, p->stride_o};
    int64_t *dst[3] = {&out->s.sq, &out->s.sdq, &out->s.so};
    for (int i = 0; i < 3; ++i) {
        const int64_t st = strides[i] == 0 ? row : strides[i];
        if (st < row || (st * esize) % 16 != 0 || st > ((int64_t)1 << 40) / esize) return DC_ERR_INVALID_ARG;
        *dst[i] = st;
    }
    out->s.wait_ns = g_wait_ns.load(std::memory_order_relaxed);
    out->s.inject = 0;
    out->dtype = p->dtype;
    const bool tc_ok = p->dtype == DC_BF16 && dc::tc::supports(out->s);
    if (p->impl == DC_IMPL_TCGEN05) {
        if (!tc_ok) return DC_ERR_UNSUPPORTED;
        out->impl = DC_IMPL_TCGEN05;
    } else if (p->impl == DC_IMPL_SIMT) {
        out->impl = DC_IMPL_SIMT;
    } else {
        out->impl = tc_ok ? DC_IMPL_TCGEN05 : DC_IMPL_SIMT;
    }
    return DC_OK;
}

dc_status_t ptrs_ok(std::initializer_list<const void *> required, std::initializer_list<const void *> optional) {
    for (const void *x : required)
        if (!x || !aligned16(x)) return DC_ERR_INVALID_ARG;
    for (const void *x : optional)
        if (x && !aligned16(x)) return DC_ERR_INVALID_ARG;
    return DC_OK;
}

dc_status_t cuda_status(cudaError_t e) {
    if (e != cudaSuccess) {
        (void)cudaGetLastError();
        return DC_ERR_CUDA;
    }
    return DC_OK;
}

// --------------------------------------------------------------------------
// SIMT launches
// --------------------------------------------------------------------------

// SIMT kernels: `blocks` CTAs, one warp per work item of a CTA up to 8, fewer when the
// shape's shared memory needs it.
template <typename K>
cudaError_t launch_simt(K kernel, const dc::Shape &s, int64_t blocks, int items, const dc::simt::SimtSmem &m,
                        cudaStream_t st, auto &&...args) {
    const int nw = dc::simt::warps_per_cta(items, m);
    if (nw < 1) return cudaErrorInvalidValue;   // not reached for the shapes check_params admits
    const size_t smem = m.bytes(nw);
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kernel<<<(unsigned)blocks, 32 * nw, smem, st>>>(s, args...);
    ++t_launches;
    return cudaGetLastError();
}

template <typename T, int DPL>
cudaError_t simt_fwd(const dc::Shape &s, const void *q, const void *k, const void *v, const float *c,
                     const float *g, void *o, float *lse, void *pmap, cudaStream_t st) {
    return launch_simt(dc::simt::fwd_kernel<T, DPL>, s, s.N, s.H, dc::simt::fwd_smem(s.H, s.d, s.W), st,
                       (int)dc::simt::fwd_keeps_scores(s.H, s.W), (const T *)q, (const T *)k, (const T *)v, c, g,
                       (T *)o, lse, (T *)pmap, 1);
}

template <typename T, int DPL>
cudaError_t simt_bwd_query(const dc::Shape &s, const void *q, const void *k, const void *v, const float *c,
                           const float *g, const void *dO, const float *lse, const void *pmap, void *dq,
                           float *dc_, float *dg, float *band, cudaStream_t st) {
    return launch_simt(dc::simt::bwd_query_kernel<T, DPL>, s, s.N, s.H, dc::simt::bwdq_smem(s.H, s.d, s.W), st,
                       (const T *)q, (const T *)k, (const T *)v, c, g, (const T *)dO, lse, (const T *)pmap,
                       (T *)dq, dc_, dg, band, 1);
}

template <typename T, int DPL>
cudaError_t simt_bwd_key(const dc::Shape &s, const void *q, const void *k, const float *c, const float *g,
                         const void *dO, const float *lse, const void *pmap, const float *dc_,
                         const float *band, void *dk, void *dv, cudaStream_t st) {
    const int tk = dc::simt::key_tile(s.N);
    return launch_simt(dc::simt::bwd_key_kernel<T, DPL>, s, (s.N + tk - 1) / tk, tk * s.H,
                       dc::simt::bwdk_smem(s.H, s.d, tk), st, tk, (const T *)q, (const T *)k, c, g, (const T *)dO,
                       lse, (const T *)pmap, dc_, band, (T *)dk, (T *)dv);
}

// Calls F<T, DPL>::run(args...) for the runtime dtype and d = 32 * DPL.
#define DC_DISPATCH(FN, dtype, d, ...)                                              \
    [&]() -> cudaError_t {                                                          \
        if ((dtype) == DC_F32) {                                                    \
            switch ((d) / 32) {                                                     \
                case 1: return FN<float, 1>(__VA_ARGS__);                           \
                case 2: return FN<float, 2>(__VA_ARGS__);                           \
                case 3: return FN<float, 3>(__VA_ARGS__);                           \
                default: return FN<float, 4>(__VA_ARGS__);                          \
            }                                                                       \
        }                                                                           \
        switch ((d) / 32) {                                                         \
            case 1: return FN<__nv_bfloat16, 1>(__VA_ARGS__);                       \
            case 2: return FN<__nv_bfloat16, 2>(__VA_ARGS__);                       \
            case 3: return FN<__nv_bfloat16, 3>(__VA_ARGS__);                       \
            default: return FN<__nv_bfloat16, 4>(__VA_ARGS__);                      \
        }                                                                           \
    }()

// The smallest workspace the backward takes: the dP band [N][W] fp32.
// dst[i] += src[i] (fp32 sum, rounded once to T): the dk, dv partials a token-range
// shard returns to the shard that owns the halo keys.
template <typename T>
__global__ void halo_add_kernel(T *dst, const T *src, int64_t n) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        dc::stf<T>(dst + i, dc::ldf<T>(dst + i) + dc::ldf<T>(src + i));
}

size_t band_bytes(const dc::Shape &s) { return sizeof(float) * (size_t)s.N * (size_t)s.W; }

// The workspace the backward asks for: on the tcgen05 path with a one-piece window also
// room for the ds band (used when given; with only band_bytes the key side recomputes ds).
size_t ws_need(const Checked &ck) {
    size_t b = band_bytes(ck.s);
    if (ck.impl == DC_IMPL_TCGEN05 && !dc::tc::segmented(ck.s)) {
        const size_t d = dc::tc::dst_shape(ck.s) ? dc::tc::dst_bytes(ck.s) : dc::tc::dsb_bytes(ck.s);
        if (d > b) b = d;
    }
    return b;
}

}  // namespace

extern "C" {

dc_status_t dc_attn_fwd(const dc_attn_params *params, const void *q, const void *k, const void *v,
                        const float *c, const float *g, void *o, float *lse, void *pmap, void *stream) {
    Checked ck;
    dc_status_t r = check_params(params, &ck);
    if (r != DC_OK) return r;
    t_launches = 0;
    if (ck.s.N == 0) return DC_OK;
    r = ptrs_ok({q, k, v, c, g, o}, {lse, pmap});
    if (r != DC_OK) return r;
    cudaStream_t st = (cudaStream_t)stream;
    // a window cut into segments keeps the per-segment LSE in lse: without it, SIMT
    if (ck.impl == DC_IMPL_TCGEN05 && dc::tc::segmented(ck.s) && !lse) {
        if (params->impl == DC_IMPL_TCGEN05) return DC_ERR_UNSUPPORTED;
        ck.impl = DC_IMPL_SIMT;
    }
    if (ck.impl == DC_IMPL_TCGEN05) {
        if (!dc::tc::segmented(ck.s)) ck.s.inject = g_inject.exchange(0);
        return cuda_status(dc::tc::fwd(ck.s, q, k, v, c, g, o, lse, pmap, st, &t_launches));
    }
    return cuda_status(DC_DISPATCH(simt_fwd, ck.dtype, ck.s.d, ck.s, q, k, v, c, g, o, lse, pmap, st));
}

size_t dc_attn_bwd_workspace_size(const dc_attn_params *params) {
    Checked ck;
    if (check_params(params, &ck) != DC_OK) return 0;
    return ws_need(ck);
}

dc_status_t dc_attn_bwd_query(const dc_attn_params *params, const void *q, const void *k, const void *v,
                              const float *c, const float *g, const void *dO, const float *lse,
                              const void *pmap, void *dq, float *dc_, float *dg, void *workspace,
                              size_t workspace_bytes, void *stream) {
    Checked ck;
    dc_status_t r = check_params(params, &ck);
    if (r != DC_OK) return r;
    t_launches = 0;
    if (ck.s.N == 0) return DC_OK;
    r = ptrs_ok({q, k, v, c, g, dO, lse, pmap, dq, dc_, dg, workspace}, {});
    if (r != DC_OK) return r;
    if (workspace_bytes < band_bytes(ck.s)) return DC_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    float *band = (float *)workspace;
    if (ck.impl == DC_IMPL_TCGEN05)
        return cuda_status(dc::tc::bwd_query(ck.s, q, k, v, c, g, dO, lse, pmap, dq, dc_, dg, workspace,
                                             workspace_bytes, st, &t_launches));
    return cuda_status(DC_DISPATCH(simt_bwd_query, ck.dtype, ck.s.d, ck.s, q, k, v, c, g, dO, lse, pmap, dq,
                                   dc_, dg, band, st));
}

dc_status_t dc_attn_bwd_key(const dc_attn_params *params, const void *q, const void *k, const float *c,
                            const float *g, const void *dO, const float *lse, const void *pmap,
                            const float *dc_, void *dk, void *dv, const void *workspace,
                            size_t workspace_bytes, void *stream) {
    Checked ck;
    dc_status_t r = check_params(params, &ck);
    if (r != DC_OK) return r;
    t_launches = 0;
    if (ck.s.N == 0) return DC_OK;
    r = ptrs_ok({q, k, c, g, dO, lse, pmap, dc_, dk, dv, workspace}, {});
    if (r != DC_OK) return r;
    if (workspace_bytes < band_bytes(ck.s)) return DC_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    const float *band = (const float *)workspace;
    if (ck.impl == DC_IMPL_TCGEN05)
        return cuda_status(dc::tc::bwd_key(ck.s, q, k, c, g, dO, lse, pmap, dc_, workspace, workspace_bytes, dk, dv,
                                           st, &t_launches));
    return cuda_status(DC_DISPATCH(simt_bwd_key, ck.dtype, ck.s.d, ck.s, q, k, c, g, dO, lse, pmap, dc_, band,
                                   dk, dv, st));
}

dc_status_t dc_attn_bwd(const dc_attn_params *params, const void *q, const void *k, const void *v,
                        const float *c, const float *g, const void *dO, const float *lse, const void *pmap,
                        void *dq, void *dk, void *dv, float *dc_, float *dg, void *workspace,
                        size_t workspace_bytes, void *stream) {
    dc_status_t r = dc_attn_bwd_query(params, q, k, v, c, g, dO, lse, pmap, dq, dc_, dg, workspace,
                                      workspace_bytes, stream);
    if (r != DC_OK) return r;
    const int32_t n1 = t_launches;
    r = dc_attn_bwd_key(params, q, k, c, g, dO, lse, pmap, dc_, dk, dv, workspace, workspace_bytes, stream);
    t_launches += n1;
    return r;
}

dc_status_t dc_attn_halo_add(void *dst, const void *src, int64_t n, int32_t dtype, void *stream) {
    if (n < 0 || (dtype != DC_F32 && dtype != DC_BF16)) return DC_ERR_INVALID_ARG;
    t_launches = 0;
    if (n == 0) return DC_OK;
    dc_status_t r = ptrs_ok({dst, src}, {});
    if (r != DC_OK) return r;
    const int threads = 256;
    const int64_t want = (n + threads - 1) / threads;
    const unsigned blocks = (unsigned)(want < 148 * 16 ? want : 148 * 16);
    cudaStream_t st = (cudaStream_t)stream;
    if (dtype == DC_F32)
        halo_add_kernel<float><<<blocks, threads, 0, st>>>((float *)dst, (const float *)src, n);
    else
        halo_add_kernel<__nv_bfloat16><<<blocks, threads, 0, st>>>((__nv_bfloat16 *)dst, (const __nv_bfloat16 *)src, n);
    ++t_launches;
    return cuda_status(cudaGetLastError());
}

int32_t dc_attn_resolve_impl(const dc_attn_params *params) {
    Checked ck;
    if (check_params(params, &ck) != DC_OK) return -1;
    return ck.impl;
}

dc_status_t dc_attn_device_status(void *stream, uint32_t *status_out, int32_t reset) {
    if (!status_out) return DC_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    unsigned int v = 0;
    cudaError_t e = cudaStreamSynchronize(st);
    if (e == cudaSuccess) e = cudaMemcpyFromSymbol(&v, dc::g_status, sizeof(v));
    if (e == cudaSuccess && reset) {
        const unsigned int zero = 0;
        e = cudaMemcpyToSymbol(dc::g_status, &zero, sizeof(zero));
    }
    if (e != cudaSuccess) {
        (void)cudaGetLastError();
        return DC_ERR_CUDA;
    }
    *status_out = v;
    return DC_OK;
}

const char *dc_attn_status_string(dc_status_t status) {
    switch (status) {
        case DC_OK: return "ok";
        case DC_ERR_INVALID_ARG: return "invalid argument";
        case DC_ERR_UNSUPPORTED: return "unsupported shape or type";
        case DC_ERR_CUDA: return "CUDA error";
        case DC_ERR_DEVICE: return "device status word holds an error";
    }
    return "unknown status";
}

int32_t dc_attn_last_launch_count(void) { return t_launches; }

dc_status_t dc_attn_set_wait_limit(uint32_t ns) {
    if (ns == 0) ns = dc::tc::kWaitNs;
    if (ns < 100000u) return DC_ERR_INVALID_ARG;
    g_wait_ns.store(ns, std::memory_order_relaxed);
    return DC_OK;
}

dc_status_t dc_attn_inject_missing_load(void) {
    g_inject.store(1);
    return DC_OK;
}

}  // extern "C"

// --------------------------------------------------------------------------
// Backward without caller-provided scratch.
//
// Some callers cannot hand the backward a workspace: plugin-style interfaces
// that give an op only its input and output tensors, and processes whose device
// memory is reserved up front by their own pool and that must not call
// cudaMalloc later.  For them the dP band lives in the array below, which every
// GPU that loads this library keeps for the life of the process.
// --------------------------------------------------------------------------

#define DC_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)

static __device__ __align__(256) unsigned char g_noalloc_scratch[DC_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mutex;
void *g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  In host code the
// array's name is only a host-side stand-in, never a usable device pointer, so
// the address comes from cudaGetSymbolAddress with that device current.  It is
// looked up again on every call made outside stream capture (a cudaDeviceReset
// in between would leave an older address dangling); a call made while `stream`
// is being captured uses the address an earlier call found on the device, since
// the lookup may load the module, which capture does not allow.
cudaError_t noalloc_scratch(cudaStream_t stream, void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    e = cudaStreamIsCapturing(stream, &cap);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (cap == cudaStreamCaptureStatusNone || !g_noalloc_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" {

dc_status_t dc_attn_bwd_noalloc(const dc_attn_params *params, const void *q, const void *k, const void *v,
                                const float *c, const float *g, const void *dO, const float *lse, const void *pmap,
                                void *dq, void *dk, void *dv, float *dc_, float *dg, void *stream) {
    Checked ck;
    dc_status_t r = check_params(params, &ck);
    if (r != DC_OK) return r;
    const size_t need = band_bytes(ck.s);
    if (need > DC_NOALLOC_SCRATCH_BYTES) return DC_ERR_UNSUPPORTED;   // N * W * 4 above the array size
    if (ck.s.N == 0) {
        t_launches = 0;
        return DC_OK;
    }
    void *scratch = nullptr;
    if (noalloc_scratch((cudaStream_t)stream, &scratch) != cudaSuccess) {
        (void)cudaGetLastError();
        return DC_ERR_CUDA;
    }
    // The query pass writes every band entry [t][w] (t < N, w < W) before the key
    // pass reads it, so nothing left in the array by an earlier call is read.
    return dc_attn_bwd(params, q, k, v, c, g, dO, lse, pmap, dq, dk, dv, dc_, dg, scratch,
                       DC_NOALLOC_SCRATCH_BYTES, stream);
}

}  // extern "C"

// --------------------------------------------------------------------------
// Producer of c and g (assumed per-token affine form; kernels in cg.cuh).
// --------------------------------------------------------------------------

namespace {

dc_status_t check_cg(const dc_cg_params *p, dc::cg::CgShape *s) {
    if (!p) return DC_ERR_INVALID_ARG;
    if (p->dtype != DC_F32 && p->dtype != DC_BF16) return DC_ERR_INVALID_ARG;
    if (p->num_tokens < 0 || p->model_dim < 2 || (p->model_dim & 1) || p->num_heads < 1) return DC_ERR_INVALID_ARG;
    const int64_t D = p->model_dim;
    const int64_t sx = p->stride_x ? p->stride_x : D, sdx = p->stride_dx ? p->stride_dx : D;
    if (sx < D || sdx < D || (sx & 1) || (sdx & 1)) return DC_ERR_INVALID_ARG;
    if (p->weight_splits && !aligned16(p->weight_splits)) return DC_ERR_INVALID_ARG;
    if (p->impl != DC_IMPL_AUTO && p->impl != DC_IMPL_SIMT && p->impl != DC_IMPL_TCGEN05) return DC_ERR_INVALID_ARG;
    if (p->num_heads > 16) return DC_ERR_UNSUPPORTED;
    // the forward keeps the weight and one tile's partial sums in shared memory
    if (dc::cg::fwd_smem_bytes(p->model_dim, p->num_heads) > dc::cg::kMaxSmem) return DC_ERR_UNSUPPORTED;
    s->N = p->num_tokens;
    s->D = p->model_dim;
    s->H = p->num_heads;
    s->sx = sx;
    s->sdx = sdx;
    return DC_OK;
}

// Kernel family of the c/g forward: tcgen05 for bf16 x whose rows TMA can address (row
// stride a multiple of 16 bytes), at least one full 128-token tile and 64 columns, and whose
// weight splits fit shared memory; SIMT otherwise.  -1: TCGEN05 asked for but not possible.
int cg_fwd_impl(const dc_cg_params *p, const dc::cg::CgShape &s) {
    const bool tc_ok = p->dtype == DC_BF16 && (s.sx * 2) % 16 == 0 && s.N >= dc::cg::kTcTile && s.D >= 64 &&
                       dc::cg::tc_stages(s.D, s.H, dc::cg::kMaxSmem) >= 2;
    if (p->impl == DC_IMPL_SIMT) return DC_IMPL_SIMT;
    if (p->impl == DC_IMPL_TCGEN05) return tc_ok ? DC_IMPL_TCGEN05 : -1;
    return tc_ok ? DC_IMPL_TCGEN05 : DC_IMPL_SIMT;
}

// Kernel family of dx: tcgen05 for bf16 with 2H <= 16, dx rows on 16-byte boundaries and the
// weight splits within shared memory; SIMT otherwise.  -1: TCGEN05 asked for but not possible.
int cg_dx_impl(const dc_cg_params *p, const dc::cg::CgShape &s) {
    const bool tc_ok = p->dtype == DC_BF16 && 2 * s.H <= 16 && s.sdx % 8 == 0 &&
                       dc::cg::dx_tc_smem_bytes(s.D) <= dc::cg::kMaxSmem;
    if (p->impl == DC_IMPL_SIMT) return DC_IMPL_SIMT;
    if (p->impl == DC_IMPL_TCGEN05) return tc_ok ? DC_IMPL_TCGEN05 : -1;
    return tc_ok ? DC_IMPL_TCGEN05 : DC_IMPL_SIMT;
}

// Kernel family of the dweight partial sums: tcgen05 on request for bf16 with 2H <= 16 and x
// rows that TMA can address (N >= 64 tokens, D >= 64); AUTO keeps the CUDA-core kernel, which
// measured faster at the GPT-2 width (22.0 against 23.9 us for 16384 x 768 tokens).
int cg_dw_impl(const dc_cg_params *p, const dc::cg::CgShape &s) {
    const bool tc_ok = p->dtype == DC_BF16 && 2 * s.H <= 16 && (s.sx * 2) % 16 == 0 && s.N >= 64 && s.D >= 64;
    if (p->impl == DC_IMPL_TCGEN05) return tc_ok ? DC_IMPL_TCGEN05 : -1;
    return DC_IMPL_SIMT;
}

cudaError_t cg_dw_tc_launch(const dc::cg::CgShape &s, const void *x, const float *dc_, const float *dg, float *part,
                            int blocks, cudaStream_t st) {
    CUtensorMap m;
    cudaError_t e = dc::tc::make_map(&m, x, s.N, 1, s.D, s.sx, dc::cg::kDwTcChunk);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(dc::cg::cg_bwd_dw_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)dc::cg::kDwTcSmem);
    if (e != cudaSuccess) return e;
    const int64_t span = (s.N + blocks - 1) / blocks;
    dc::cg::cg_bwd_dw_tc_kernel<<<blocks, dc::cg::kDwTcThreads, dc::cg::kDwTcSmem, st>>>(
        m, s, span, dc_, dg, part, g_wait_ns.load(std::memory_order_relaxed));
    ++t_launches;
    return cudaGetLastError();
}

cudaError_t cg_dx_tc_launch(const dc::cg::CgShape &s, const float *w, const uint8_t *splits, const float *dc_,
                            const float *dg, void *dx, cudaStream_t st) {
    const size_t smem = dc::cg::dx_tc_smem_bytes(s.D);
    cudaError_t e = cudaFuncSetAttribute(dc::cg::cg_bwd_dx_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)((s.N + dc::cg::kTcTile - 1) / dc::cg::kTcTile);
    dc::cg::cg_bwd_dx_tc_kernel<<<grid, dc::cg::kDxThreads, smem, st>>>(
        s, w, splits, dc_, dg, (__nv_bfloat16 *)dx,
        g_wait_ns.load(std::memory_order_relaxed));
    ++t_launches;
    return cudaGetLastError();
}

template <int R>
cudaError_t cg_fwd_tc_launch(const dc::cg::CgShape &s, const void *x, const float *w, const uint8_t *splits,
                             const float *b, float *c, float *g, cudaStream_t st) {
    CUtensorMap m;
    cudaError_t e = dc::tc::make_map(&m, x, s.N, 1, s.D, s.sx, dc::cg::kTcTile);
    if (e != cudaSuccess) return e;
    auto kern = dc::cg::cg_fwd_tc_kernel<R>;
    const int nst = dc::cg::tc_stages(s.D, s.H, dc::cg::kMaxSmem);
    const size_t smem = dc::cg::tc_smem_bytes(s.D, s.H, nst);
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)((s.N + dc::cg::kTcTile - 1) / dc::cg::kTcTile);
    kern<<<grid, dc::cg::kTcThreads, smem, st>>>(m, s, w, splits, b, c, g, nst,
                                                  g_wait_ns.load(std::memory_order_relaxed));
    ++t_launches;
    return cudaGetLastError();
}

// 16-byte accesses when every row starts on a 16-byte boundary and spans whole 16-byte units.
template <typename T>
int cg_vec16(int64_t stride, int D, const void *base) {
    return (uintptr_t)base % 16 == 0 && (stride * (int64_t)sizeof(T)) % 16 == 0 && (D * sizeof(T)) % 16 == 0;
}

template <typename K>
cudaError_t cg_tile_grid(K kern, size_t smem, int64_t tiles, unsigned *grid) {
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, dc::cg::kThreads, smem);
    if (e != cudaSuccess) return e;
    int sms = 0, dev = 0;
    e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const int64_t resident = (int64_t)sms * (per_sm > 0 ? per_sm : 1);
    *grid = (unsigned)(tiles < resident ? tiles : resident);
    return cudaSuccess;
}

template <int OUT, typename T>
cudaError_t cg_fwd_launch(const dc::cg::CgShape &s, const void *x, const float *w, const float *b, float *c, float *g,
                          cudaStream_t st) {
    auto kern = dc::cg::cg_fwd_kernel<T, OUT>;
    const size_t smem = dc::cg::fwd_smem_bytes(s.D, s.H);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    unsigned grid = 0;
    e = cg_tile_grid(kern, smem, (s.N + dc::cg::tile_tokens(OUT) - 1) / dc::cg::tile_tokens(OUT), &grid);
    if (e != cudaSuccess) return e;
    kern<<<grid, dc::cg::kThreads, smem, st>>>(s, (const T *)x, w, b, c, g, cg_vec16<T>(s.sx, s.D, x));
    ++t_launches;
    return cudaGetLastError();
}

template <int OUT, typename T>
cudaError_t cg_bwd_launch(const dc::cg::CgShape &s, const void *x, const float *w, const float *dc_, const float *dg,
                          void *dx, float *dw, float *db, float *part, int blocks, bool dx_tc, bool dw_tc,
                          const uint8_t *splits, cudaStream_t st) {
    if (s.N > 0 && dx_tc) {
        cudaError_t e = cg_dx_tc_launch(s, w, splits, dc_, dg, dx, st);
        if (e != cudaSuccess) return e;
    } else if (s.N > 0) {
        auto kdx = dc::cg::cg_bwd_dx_kernel<T, OUT>;
        const size_t smem = dc::cg::wp_bytes(s.D, s.H);
        cudaError_t e = cudaFuncSetAttribute(kdx, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        unsigned grid = 0;
        e = cg_tile_grid(kdx, smem, (s.N + dc::cg::tile_tokens(OUT) - 1) / dc::cg::tile_tokens(OUT), &grid);
        if (e != cudaSuccess) return e;
        kdx<<<grid, dc::cg::kThreads, smem, st>>>(s, w, dc_, dg, (T *)dx, cg_vec16<T>(s.sdx, s.D, dx));
        ++t_launches;
    }
    if (s.N > 0 && dw_tc) {
        cudaError_t e = cg_dw_tc_launch(s, x, dc_, dg, part, blocks, st);
        if (e != cudaSuccess) return e;
    } else if (s.N > 0) {
        auto kdw = dc::cg::cg_bwd_dw_partial_kernel<T, OUT>;
        const int chunk = dc::cg::dw_chunk(s.D, s.H, sizeof(T));
        const size_t dsmem = dc::cg::dw_smem_bytes(s.D, s.H, sizeof(T));
        cudaError_t e = cudaFuncSetAttribute(kdw, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dsmem);
        if (e != cudaSuccess) return e;
        const int64_t span = (s.N + blocks - 1) / blocks;
        kdw<<<blocks, dc::cg::kDwThreads, dsmem, st>>>(s, span, chunk, (const T *)x, dc_, dg, part,
                                                     cg_vec16<T>(s.sx, s.D, x));
        ++t_launches;
    }
    const int64_t n = dc::cg::record_floats(s.D, s.H);
    dc::cg::cg_bwd_dw_reduce_kernel<<<(unsigned)((n + 31) / 32), dc::cg::kReduceThreads, 0, st>>>(s, blocks, part, dw,
                                                                                                db);
    ++t_launches;
    return cudaGetLastError();
}

template <typename F>
cudaError_t cg_dispatch(int H, int dtype, F &&f) {
    switch (dc::cg::out_pad(2 * H)) {
        case 8: return dtype == DC_F32 ? f.template operator()<8, float>() : f.template operator()<8, __nv_bfloat16>();
        case 12: return dtype == DC_F32 ? f.template operator()<12, float>() : f.template operator()<12, __nv_bfloat16>();
        case 16: return dtype == DC_F32 ? f.template operator()<16, float>() : f.template operator()<16, __nv_bfloat16>();
        case 24: return dtype == DC_F32 ? f.template operator()<24, float>() : f.template operator()<24, __nv_bfloat16>();
        default: return dtype == DC_F32 ? f.template operator()<32, float>() : f.template operator()<32, __nv_bfloat16>();
    }
}

size_t cg_ws_need(const dc::cg::CgShape &s) {
    if (s.N == 0) return 0;
    return sizeof(float) * (size_t)dc::cg::partial_blocks(s.N) * (size_t)dc::cg::record_floats(s.D, s.H);
}

}  // namespace

extern "C" {

dc_status_t dc_attn_cg_fwd(const dc_cg_params *params, const void *x, const float *weight, const float *bias,
                           float *c, float *g, void *stream) {
    dc::cg::CgShape s;
    dc_status_t r = check_cg(params, &s);
    if (r != DC_OK) return r;
    t_launches = 0;
    if (s.N == 0) return DC_OK;
    r = ptrs_ok({x, weight, bias, c, g}, {});
    if (r != DC_OK) return r;
    const int impl = cg_fwd_impl(params, s);
    if (impl < 0) return DC_ERR_UNSUPPORTED;
    cudaStream_t st = (cudaStream_t)stream;
    if (impl == DC_IMPL_TCGEN05)
    {
        const uint8_t *sp = (const uint8_t *)params->weight_splits;
        return cuda_status(dc::cg::tc_rows_per_split(s.H) == 16 ? cg_fwd_tc_launch<16>(s, x, weight, sp, bias, c, g, st)
                                                                : cg_fwd_tc_launch<32>(s, x, weight, sp, bias, c, g, st));
    }
    return cuda_status(cg_dispatch(s.H, params->dtype, [&]<int OUT, typename T>() {
        return cg_fwd_launch<OUT, T>(s, x, weight, bias, c, g, st);
    }));
}

int32_t dc_attn_cg_resolve_impl(const dc_cg_params *params) {
    dc::cg::CgShape s;
    if (check_cg(params, &s) != DC_OK) return -1;
    return cg_fwd_impl(params, s);
}

size_t dc_attn_cg_bwd_workspace_size(const dc_cg_params *params) {
    dc::cg::CgShape s;
    if (check_cg(params, &s) != DC_OK) return 0;
    return cg_ws_need(s);
}

dc_status_t dc_attn_cg_bwd(const dc_cg_params *params, const void *x, const float *weight, const float *dc_,
                           const float *dg, void *dx, float *dweight, float *dbias, void *workspace,
                           size_t workspace_bytes, void *stream) {
    dc::cg::CgShape s;
    dc_status_t r = check_cg(params, &s);
    if (r != DC_OK) return r;
    t_launches = 0;
    r = ptrs_ok({dweight, dbias}, {});
    if (r != DC_OK) return r;
    if (s.N > 0) {
        r = ptrs_ok({x, weight, dc_, dg, dx, workspace}, {});
        if (r != DC_OK) return r;
        if (workspace_bytes < cg_ws_need(s)) return DC_ERR_INVALID_ARG;
    }
    const int blocks = s.N > 0 ? dc::cg::partial_blocks(s.N) : 0;
    const int dx_impl = cg_dx_impl(params, s), dw_impl = cg_dw_impl(params, s);
    if (dx_impl < 0 || dw_impl < 0) return DC_ERR_UNSUPPORTED;
    cudaStream_t st = (cudaStream_t)stream;
    return cuda_status(cg_dispatch(s.H, params->dtype, [&]<int OUT, typename T>() {
        return cg_bwd_launch<OUT, T>(s, x, weight, dc_, dg, dx, dweight, dbias, (float *)workspace, blocks,
                                     dx_impl == DC_IMPL_TCGEN05, dw_impl == DC_IMPL_TCGEN05,
                                     (const uint8_t *)params->weight_splits, st);
    }));
}

size_t dc_attn_cg_prepare_size(const dc_cg_params *params) {
    dc::cg::CgShape s;
    if (check_cg(params, &s) != DC_OK) return 0;
    return dc::cg::prep_fwd_bytes(s.D, s.H);
}

dc_status_t dc_attn_cg_prepare(const dc_cg_params *params, const float *weight, void *splits, void *stream) {
    dc::cg::CgShape s;
    dc_status_t r = check_cg(params, &s);
    if (r != DC_OK) return r;
    t_launches = 0;
    r = ptrs_ok({weight, splits}, {});
    if (r != DC_OK) return r;
    cudaStream_t st = (cudaStream_t)stream;
    const int R = dc::cg::tc_rows_per_split(s.H);
    const int64_t items = (int64_t)R * ((s.D + 63) / 64) * 8;
    const unsigned blocks = (unsigned)((items + 255) / 256 < 148 ? (items + 255) / 256 : 148);
    if (R == 16)
        dc::cg::cg_prepare_kernel<16><<<blocks, 256, 0, st>>>(s, weight, (uint8_t *)splits);
    else
        dc::cg::cg_prepare_kernel<32><<<blocks, 256, 0, st>>>(s, weight, (uint8_t *)splits);
    ++t_launches;
    return cuda_status(cudaGetLastError());
}

}  // extern "C"
