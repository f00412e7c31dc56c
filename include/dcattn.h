/*
 * dcattn.h -- C ABI of libdcattn, Lightweight DC attention on NVIDIA B200 (sm_100a).
 *
 * The operation (the "Lightweight DC" paragraph of the m.aitntnews.com blog
 * post on the NanoGPT speedrun, section "第二刀-砍层内"): the layer's existing
 * Q and K are reused for an extra causal local window of W keys (112 there);
 * every head takes a softmax over its window scores; the H per-head maps are
 * merged with per-token, input-dependent weights into one shared map; the
 * shared map is applied to each head's V with a per-head scale.  For query
 * token t in document [a, b) and head h:
 *
 *   window(t) = { j : max(a, t-W+1) <= j <= t }
 *   p_h(t,j)  = softmax over window(t) of  sigma * <q_h(t), k_h(j)>
 *   P(t,j)    = sum_h c[t,h] * p_h(t,j)           (c: signed, per token)
 *   o_h(t)    = g[t,h] * sum_j P(t,j) * v_h(j)     (g: per-token head scale)
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Tokens are packed: N = total_tokens rows, documents given by cu_seqlens
 *   (device, int32, num_docs + 1 entries, 0 = cu[0] <= ... <= cu[num_docs] = N;
 *   empty documents are allowed).  No key of another document is ever used.
 * - q, k, v, o, dO, dq, dk, dv: [N][H][d] in `dtype` (fp32 or bf16), each token's
 *   H * d elements contiguous, consecutive tokens `stride` elements apart:
 *   stride_qkv for q, k, v; stride_dqkv for dq, dk, dv; stride_o for o (forward)
 *   and dO (backward).  A stride of 0 means H * d (contiguous tensors).  The
 *   strides let q, k, v be views of one fused projection [N][3][H][d] (stride
 *   3 * H * d) and dq, dk, dv be written straight into its gradient.
 *   c, g, lse, dc, dg: contiguous [N][H] fp32.
 *   pmap: contiguous [N][W] in `dtype`; pmap[t][w] = P(t, t-W+1+w), 0 outside
 *   window(t).  It is the one composed map per token (the H per-head maps are
 *   never written to memory); the forward produces it, the backward reads it.
 * - Every pointer is caller-owned DEVICE memory, 16-byte aligned.  The library
 *   never allocates, frees or synchronizes (except dc_attn_device_status).
 *   Outputs are overwritten, never accumulated into.  Inputs are not modified.
 * - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *   stream).  Argument errors are detected on the host and returned before
 *   anything is launched.  Errors found on the device (malformed cu_seqlens, a
 *   bounded wait that gave up) are recorded in a per-device status word read by
 *   dc_attn_device_status(); kernels never trap.  Malformed cu_seqlens cannot
 *   make a kernel read or write out of bounds; they only make results undefined.
 * - The library is compiled for sm_100a only.
 */
#ifndef DCATTN_H
#define DCATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    DC_OK = 0,
    DC_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size, bad enum   */
    DC_ERR_UNSUPPORTED = 2,   /* valid request outside what this build covers  */
    DC_ERR_CUDA = 3,          /* a CUDA runtime/driver call failed             */
    DC_ERR_DEVICE = 4         /* the device status word holds an error         */
} dc_status_t;

typedef enum { DC_F32 = 0, DC_BF16 = 1 } dc_dtype_t;

/* Kernel family.  AUTO picks the tcgen05/TMA path when the shape allows it
 * (bf16, d in {64,128}, W <= 256) and the SIMT path otherwise.  SIMT is the
 * fp32-accumulating CUDA-core path used for fp32 tensors and any shape.
 * On tcgen05 a window of W > 129 keys runs as two segments (the 128 keys
 * ending at the query, then the rest): the forward first merges the two
 * segments' log-sum-exp values in `lse` and so needs that buffer (AUTO
 * without lse runs such a forward on SIMT; TCGEN05 without lse returns
 * DC_ERR_UNSUPPORTED), and the second segment adds its share to o, dq, dk
 * and dv after the first one has written them, which rounds that partial
 * sum to bf16 once. */
typedef enum { DC_IMPL_AUTO = 0, DC_IMPL_SIMT = 1, DC_IMPL_TCGEN05 = 2 } dc_impl_t;

/* Bits of the device status word. */
#define DC_DEVERR_SEQLENS 0x1u   /* cu_seqlens not 0-based, non-decreasing, ending at N */
#define DC_DEVERR_TIMEOUT 0x2u   /* a bounded wait inside a kernel gave up              */

typedef struct {
    int32_t dtype;              /* dc_dtype_t: type of q,k,v,o,dO,dq,dk,dv,pmap           */
    int32_t impl;               /* dc_impl_t                                              */
    int64_t total_tokens;       /* N >= 0; N == 0 is a no-op                              */
    int32_t num_docs;           /* >= 1 when N > 0                                        */
    int32_t num_heads;          /* H in [1, 16]                                           */
    int32_t head_dim;           /* d in {32, 64, 96, 128} (tcgen05 path: {64, 128})        */
    int32_t window;             /* W in [1, 4096]: keys t-W+1 .. t (query included)       */
    float softmax_scale;        /* sigma, usually 1/sqrt(d); 1 when q is pre-scaled        */
    int32_t reserved;           /* must be 0                                              */
    const int32_t *cu_seqlens;  /* device pointer, num_docs + 1 entries                   */
    int64_t stride_qkv;         /* elements between tokens of q, k, v; 0 = H * d          */
    int64_t stride_dqkv;        /* ... of dq, dk, dv; 0 = H * d                           */
    int64_t stride_o;           /* ... of o and dO; 0 = H * d                             */
    /* A nonzero stride must be >= H * d and a multiple of 16 bytes (8 bf16 or 4 fp32
     * elements), else DC_ERR_INVALID_ARG. */
} dc_attn_params;

/* Forward pass.
 * In : q, k, v [N][H][d]; c, g [N][H] fp32.
 * Out: o [N][H][d]; lse [N][H] fp32, lse_h(t) = log sum_j exp(sigma<q_h(t),k_h(j)>)
 *      (natural log); pmap [N][W].  lse and pmap may be NULL when no backward
 *      pass will follow; the backward needs both. */
dc_status_t dc_attn_fwd(const dc_attn_params *params,
                        const void *q, const void *k, const void *v,
                        const float *c, const float *g,
                        void *o, float *lse, void *pmap, void *stream);

/* Bytes of device scratch the backward entry points ask for; 0 when N == 0.
 * The least they accept is N * W * 4 (the composed-map gradient dP(t, .) handed
 * from the query pass to the key pass, fp32 [N][W]).  On the tcgen05 path with
 * W <= 129 the size returned also holds the ds band, H * N * round8(W) * 2
 * bytes (bf16 ds_h(t, j) of the query pass, which the key pass then reads
 * instead of recomputing it); a workspace smaller than that but at least
 * N * W * 4 runs the recomputing key pass.  Give dc_attn_bwd_query and
 * dc_attn_bwd_key the same workspace and the same size. */
size_t dc_attn_bwd_workspace_size(const dc_attn_params *params);

/* Backward, query side: dq [N][H][d], dc [N][H], dg [N][H] fp32, and dP into
 * the workspace.  Needs lse and pmap from dc_attn_fwd with the same inputs.
 *   dg[t,h]   = sum_j P(t,j) <dO_h(t), v_h(j)>
 *   dP(t,j)   = sum_h g[t,h] <dO_h(t), v_h(j)>
 *   dc[t,h]   = sum_j dP(t,j) p_h(t,j)
 *   ds_h(t,j) = c[t,h] p_h(t,j) (dP(t,j) - dc[t,h])
 *   dq_h(t)   = sigma sum_j ds_h(t,j) k_h(j)
 * (chain rule of the definition above; the page states no backward pass). */
dc_status_t dc_attn_bwd_query(const dc_attn_params *params,
                              const void *q, const void *k, const void *v,
                              const float *c, const float *g, const void *dO,
                              const float *lse, const void *pmap,
                              void *dq, float *dc, float *dg,
                              void *workspace, size_t workspace_bytes, void *stream);

/* Backward, key side: dk, dv [N][H][d].  Must follow dc_attn_bwd_query on the
 * same stream with the same workspace and size (it reads dc and the stored dP,
 * or the stored ds).
 *   dk_h(j) = sigma sum_{t: j in window(t)} ds_h(t,j) q_h(t)
 *   dv_h(j) = sum_{t: j in window(t)} P(t,j) g[t,h] dO_h(t) */
dc_status_t dc_attn_bwd_key(const dc_attn_params *params,
                            const void *q, const void *k,
                            const float *c, const float *g, const void *dO,
                            const float *lse, const void *pmap, const float *dc,
                            void *dk, void *dv,
                            const void *workspace, size_t workspace_bytes, void *stream);

/* Full backward: dc_attn_bwd_query followed by dc_attn_bwd_key. */
dc_status_t dc_attn_bwd(const dc_attn_params *params,
                        const void *q, const void *k, const void *v,
                        const float *c, const float *g, const void *dO,
                        const float *lse, const void *pmap,
                        void *dq, void *dk, void *dv, float *dc, float *dg,
                        void *workspace, size_t workspace_bytes, void *stream);

/* Backward that allocates nothing and takes no workspace (no counterpart on the
 * page; an interface addition).  For callers that cannot provide scratch:
 * plugin-style interfaces that hand an op only its inputs and outputs, and
 * processes whose device memory is reserved by their own pool at start-up and
 * that must not call cudaMalloc afterwards.  Same arguments and results as
 * dc_attn_bwd minus the workspace; the scratch lives instead in a static
 * device array of 32 MiB (33554432 bytes) that every GPU loading this library
 * keeps until the process exits (it is passed on as a workspace of that size,
 * so the ds band is used when it fits).
 * - Returns DC_ERR_UNSUPPORTED, before any launch, when the dP band needs more
 *   than that: N * W * 4 bytes > 32 MiB (e.g. N = 65536 tokens at W = 128).
 * - The array's device address is looked up (with the calling thread's
 *   current device) on every call made outside stream capture, so a
 *   cudaDeviceReset between two calls does no harm.  A call made while its
 *   stream is being captured reuses the address that the last uncaptured call
 *   on that device found: make one uncaptured call on each device before any
 *   capture, and do not replay a captured graph after a cudaDeviceReset.
 * - Every call on a device shares the one array.  Calls whose kernels overlap
 *   on the GPU (different streams, or different host threads, without
 *   ordering between them) race on it and give undefined results; serialise
 *   them.  Nothing needs clearing between calls: the query pass rewrites every
 *   band entry the key pass reads.
 * - Calls no cudaMalloc/cudaFree and no allocating library routine. */
dc_status_t dc_attn_bwd_noalloc(const dc_attn_params *params,
                                const void *q, const void *k, const void *v,
                                const float *c, const float *g, const void *dO,
                                const float *lse, const void *pmap,
                                void *dq, void *dk, void *dv, float *dc, float *dg,
                                void *stream);

/* dst[i] += src[i] for i < n, in `dtype` (dc_dtype_t) with an fp32 sum rounded
 * once (no counterpart on the page; an interface addition for token-range
 * sharding of one long sequence over several GPUs: the dk and dv partials that
 * a shard computes for the W - 1 keys before its range, which belong to its left
 * neighbour, are added there).  dst and src: device, 16-byte aligned, not
 * overlapping.  Asynchronous on `stream`. */
dc_status_t dc_attn_halo_add(void *dst, const void *src, int64_t n, int32_t dtype, void *stream);

/* Which kernel family AUTO resolves to for these params (DC_IMPL_SIMT or
 * DC_IMPL_TCGEN05), or -1 if the params are invalid. */
int32_t dc_attn_resolve_impl(const dc_attn_params *params);

/* Synchronizes `stream`, stores the current device's status word (DC_DEVERR_*
 * bits, 0 = no error) into *status_out and clears it when `reset` != 0.
 * Returns DC_ERR_CUDA if the synchronization itself failed. */
dc_status_t dc_attn_device_status(void *stream, uint32_t *status_out, int32_t reset);

/* Static, human-readable name of a status code. */
const char *dc_attn_status_string(dc_status_t status);

/* Number of kernel launches the last successful call on this host thread made
 * (used to report launches per step). */
int32_t dc_attn_last_launch_count(void);

/* Failure-detection hooks (no counterpart on the page; they exist so that the
 * bounded waits can be tested without a GPU fault).
 *
 * Every wait of a tcgen05 kernel on one of its own pipeline stages (a tile
 * load, a tensor-core product, a hand-over between its warps) gives up after
 * a time limit: the CTA then raises DC_DEVERR_TIMEOUT in the device status
 * word, skips the rest of its work without issuing further loads or products,
 * and exits normally, so the context stays usable and the host learns of it
 * through dc_attn_device_status().
 *
 * dc_attn_set_wait_limit: limit in nanoseconds for kernels launched by later
 * calls from any host thread; 0 restores the default of 2 s.  Values below
 * 100000 (0.1 ms) return DC_ERR_INVALID_ARG.  A legitimate wait lasts
 * microseconds, so a limit of a few milliseconds still never fires in
 * normal operation.
 *
 * dc_attn_inject_missing_load: the next dc_attn_fwd call (from any host
 * thread) that runs the one-piece tcgen05 forward leaves out the first
 * CTA's head-0 Q/K tile loads, so that CTA's wait for them runs out.  The
 * load is never issued, so nothing is in flight when the CTA exits.  That
 * call completes after about one wait limit, its outputs are undefined, and
 * the status word gets DC_DEVERR_TIMEOUT.  One-shot. */
dc_status_t dc_attn_set_wait_limit(uint32_t ns);
dc_status_t dc_attn_inject_missing_load(void);

/* ------------------------------------------------------------------------
 * Producer of c and g.
 *
 * The page's DCMHA paragraph says only that the heads' combination is decided
 * dynamically from the current input; it gives no formula.  These entry
 * points implement the plainest reading, an ASSUMED form: per-token affine maps
 * of the layer's hidden state x [N][D], with no nonlinearity.  For token t,
 * head h < H and weight [2H][D] (row o produces output o, the layout of a
 * linear layer's weight), bias [2H]:
 *
 *   c[t,h] = bias[h]     + sum_k x[t,k] * weight[h][k]
 *   g[t,h] = bias[H + h] + sum_k x[t,k] * weight[H + h][k]
 *
 * The sums are taken in fp32 (x converted from `dtype`); c, g feed
 * dc_attn_fwd directly.  Shapes: x, dx [N][D] in `dtype`, consecutive tokens
 * stride_x / stride_dx elements apart (0 = D); weight, dweight [2H][D] fp32
 * contiguous; bias, dbias [2H] fp32; c, g, dc, dg [N][H] fp32 contiguous.
 * Limits: D even; strides even and >= D; 1 <= H <= 16 (larger H returns
 * DC_ERR_UNSUPPORTED).  The forward keeps in shared memory the weight padded
 * to OUT rows (OUT = 8, 12, 16, 24 or 32, the first >= 2H; 4 * OUT * D bytes)
 * and the 8 column slices' partial sums of 64 tokens (32 when OUT > 12); the
 * two must fit 227 KB, else DC_ERR_UNSUPPORTED (D <= 4330 at H = 6, D <= 1560
 * at H = 16, either dtype).  Pointers: device, 16-byte aligned,
 * caller-owned; asynchronous on `stream`; outputs overwritten.
 * ------------------------------------------------------------------------ */
typedef struct {
    int32_t dtype;        /* dc_dtype_t of x and dx                                   */
    int32_t model_dim;    /* D                                                        */
    int32_t num_heads;    /* H                                                        */
    int32_t impl;         /* dc_impl_t for the forward and for dx                     */
    int64_t num_tokens;   /* N >= 0                                                   */
    int64_t stride_x;     /* elements between tokens of x (0 = D)                     */
    int64_t stride_dx;    /* elements between tokens of dx (0 = D)                    */
    const void *weight_splits;  /* NULL, or the image dc_attn_cg_prepare wrote for this
                                 * weight (device, 16-byte aligned): the tcgen05 kernels
                                 * then copy it instead of converting the weight
                                 * themselves; results are identical either way         */
} dc_cg_params;

/* c, g from x.  N = 0 launches nothing.
 * Two kernel families.  SIMT: CUDA-core fp32 FMAs in a fixed order.  TCGEN05 (bf16 x
 * only, row stride a multiple of 8 elements, N >= 128, D >= 64, and the weight splits
 * below within shared memory: D <= 2048 at H <= 8, D <= 1024 at H <= 16): tensor-core
 * products of x with the three bf16 terms hi + mid + lo of the weight, whose sum is the
 * fp32 weight to within 2^-24 of each element, accumulated in fp32 by the tensor core
 * (its accumulation order and rounding are the hardware's).  AUTO takes TCGEN05 when
 * possible; TCGEN05 where it is not possible returns DC_ERR_UNSUPPORTED. */
dc_status_t dc_attn_cg_fwd(const dc_cg_params *params, const void *x, const float *weight, const float *bias,
                           float *c, float *g, void *stream);

/* Which family the forward resolves to (DC_IMPL_SIMT or DC_IMPL_TCGEN05), or -1 if the
 * params are invalid or ask for TCGEN05 where it is not possible. */
int32_t dc_attn_cg_resolve_impl(const dc_cg_params *params);

/* The weight in the form the tensor-core kernels read (the bf16 splits, laid out as
 * their shared-memory operands), for callers that run the producer many times with one
 * weight (a training step's forward and backward): written once with dc_attn_cg_prepare
 * and passed as params->weight_splits.  Size in bytes for the params' D and H (dtype,
 * N and strides do not matter; 0 if the params are invalid).  The image depends only
 * on the weight's values; after the weight changes it must be prepared again. */
size_t dc_attn_cg_prepare_size(const dc_cg_params *params);
dc_status_t dc_attn_cg_prepare(const dc_cg_params *params, const float *weight, void *splits, void *stream);

/* Bytes of workspace dc_attn_cg_bwd needs (0 when N = 0 or the params are
 * invalid): one fp32 partial record of dweight and dbias per block of tokens. */
size_t dc_attn_cg_bwd_workspace_size(const dc_cg_params *params);

/* Gradients for dL/dc = dc, dL/dg = dg, writing e[t] = (dc[t,:], dg[t,:]).
 * dx runs on tcgen05 for bf16 with 2H <= 16, a dx row stride that is a multiple of 8
 * elements and D <= 2048 (AUTO; TCGEN05 elsewhere returns DC_ERR_UNSUPPORTED): products
 * of the bf16 splits of e and of the weight, six of the nine pairs, whose sum is e * w to
 * within 2^-23 |e w|, accumulated by the tensor core; SIMT otherwise.  The partial sums
 * of dweight run on the CUDA cores under AUTO and SIMT; TCGEN05 moves them to the tensor
 * cores (bf16 with 2H <= 16, x rows that TMA can address (row stride a multiple of 8
 * elements), N >= 64 and D >= 64): products of x with the bf16 splits of e (exact),
 * accumulated by the tensor core over each block's tokens.  dbias and the final sum over
 * blocks are fp32 on the CUDA cores.  TCGEN05 requires both dx and dweight to be possible
 * on the tensor cores:
 *
 *   dx[t,k]       = sum_o e[t,o] * weight[o][k]
 *   dweight[o][k] = sum_t e[t,o] * x[t,k]        dbias[o] = sum_t e[t,o]
 *
 * dweight and dbias are summed over fixed token ranges and then over the
 * ranges in a fixed order: the result is bitwise reproducible for a given N.
 * With N = 0 only dweight and dbias are written (zeros) and the other pointers
 * may be NULL.  workspace_bytes below dc_attn_cg_bwd_workspace_size returns
 * DC_ERR_INVALID_ARG. */
dc_status_t dc_attn_cg_bwd(const dc_cg_params *params, const void *x, const float *weight, const float *dc,
                           const float *dg, void *dx, float *dweight, float *dbias, void *workspace,
                           size_t workspace_bytes, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* DCATTN_H */
