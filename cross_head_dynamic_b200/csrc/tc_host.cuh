// tc_host.cuh -- tcgen05/TMA path (host side).  Placeholder until the kernels land.
#pragma once
#include "common.cuh"

namespace dc {
namespace tc {

inline bool supports(const Shape &) { return false; }

inline cudaError_t fwd(const Shape &, const void *, const void *, const void *, const float *, const float *,
                       void *, float *, void *, cudaStream_t, int32_t *) {
    return cudaErrorNotSupported;
}
inline cudaError_t bwd_query(const Shape &, const void *, const void *, const void *, const float *,
                             const float *, const void *, const float *, const void *, void *, float *,
                             float *, float *, cudaStream_t, int32_t *) {
    return cudaErrorNotSupported;
}
inline cudaError_t bwd_key(const Shape &, const void *, const void *, const float *, const float *,
                           const void *, const float *, const void *, const float *, const float *, void *,
                           void *, cudaStream_t, int32_t *) {
    return cudaErrorNotSupported;
}

}  // namespace tc
}  // namespace dc
