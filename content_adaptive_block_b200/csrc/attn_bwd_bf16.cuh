// Block-sparse causal attention backward (placeholder until the kernels land).
#pragma once

#include "common.cuh"

namespace gsa {
namespace bwd {

inline gsa_status launch(const void*, const void*, const void*, const void*, const float*, const void*,
                         const gsa_block_csr*, const gsa_attn_desc*, const uint8_t*, float, void*, void*, void*,
                         float*, cudaStream_t) {
    return GSA_ERR_UNSUPPORTED;
}

}  // namespace bwd
}  // namespace gsa
