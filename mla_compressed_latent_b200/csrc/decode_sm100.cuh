// Tensor-core (tcgen05 / TMEM / TMA) absorbed decode for sm_100a.
#pragma once
#include "common.cuh"

namespace mla {
namespace sm100 {

inline bool decode_supported(const mla_dims_t*, int32_t, int32_t, int32_t) { return false; }
inline size_t decode_workspace_bytes(const mla_dims_t*, int32_t, int32_t, int32_t, int) { return 0; }
inline int launch_decode(const mla_dims_t*, int32_t, int32_t, const void*, const mla_latent_cache_t*,
                         const int32_t*, int32_t, const int32_t*, void*, float*, void*, size_t, int,
                         cudaStream_t) {
  return MLA_ERR_UNSUPPORTED;
}

}  // namespace sm100
}  // namespace mla
