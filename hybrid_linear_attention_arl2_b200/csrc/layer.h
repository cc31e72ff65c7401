// Host entry points of the hybrid layer shared between translation units of
// the library (the attention block calls the layer through these).
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

#include "arl2.h"

namespace arl2 {

// The hybrid layer's query and commit with Q, K and V read as strided views:
// token rows `ld` elements apart (0: contiguous, H * 128), bf16 only.  The
// C entry points arl2_frame_query / arl2_frame_commit are these with ld = 0.
arl2_status layer_query_ld(::arl2_state* h, const void* q, const void* k, const void* v, int64_t ld, void* o,
                           cudaStream_t st);
arl2_status layer_commit_ld(::arl2_state* h, const void* q, const void* k, const void* v, int64_t ld, const float* alpha,
                            const float* beta, void* o, cudaStream_t st);

}  // namespace arl2
