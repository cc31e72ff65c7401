// Host entry points of the hybrid layer shared between translation units of
// the library (the attention block calls the layer through these).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstddef>
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

// The layer handle's device error word and its wait limit, for kernels the
// attention block launches beside the layer (its GEMMs).
uint32_t* layer_error_word(::arl2_state* h);
uint64_t layer_wait_limit(::arl2_state* h);

// The token-level query (commit = false) and commit of a bf16 hybrid-layer
// handle: arl2_token_query and arl2_token_commit.
arl2_status token_pass(::arl2_state* h, const void* q, const void* k, const void* v, const float* alpha_tok,
                       const float* beta, void* o, cudaStream_t st, bool commit);

// Token-level pass (token_level.cu): operands, scratch and launch.  Q, K, V,
// O bf16 [B, L, H, 128] contiguous (O holds the intra-frame output on entry);
// phi_q [H][i][j] as given, phi_k and phi_v transposed ([H][j][i]); alpha_tok
// and beta f32 [B, H, L]; s_in / s_out f32 [B, H, 128, 128] (s_out null for a
// query pass).  The scratch arrays are f32, bound by token_bind_scratch.
struct TokenParams {
  const __nv_bfloat16 *q, *k, *v;
  const __nv_bfloat16 *phi_q, *phi_k_t, *phi_v_t;
  const float *alpha_tok, *beta;
  float corr;
  int B, L, H, n_chunks;
  float *qp, *kp, *vp, *w, *u, *qt, *ot;  // [B, H, L, 128]
  float *m, *n, *s_chunk;                 // [B, H, n_chunks, 128, 128] (m holds each chunk's M transposed)
  const float* s_in;
  float* s_out;
  __nv_bfloat16* o;
  uint32_t* err;          // the handle's device error word (a wait that ran out)
  uint64_t wait_limit_ns;
};
size_t token_scratch_floats(int B, int H, int L);
void token_bind_scratch(TokenParams& p, float* base);
// with_out = false leaves o as it is (the state steps still run)
cudaError_t launch_token_level(const TokenParams& p, bool with_out, cudaStream_t st);

}  // namespace arl2
