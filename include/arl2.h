/*
 * arl2.h -- C ABI of libarl2.so: the per-frame hot path of the ARL2 hybrid
 * attention module on NVIDIA B200 (sm_100a).
 *
 * Sources.  "ARL2 summary" is the technical summary on the page "Attend
 * Locally, Remember Linearly: Linear Attention as Cross-Frame Memory for
 * Autoregressive Video Diffusion" (gist.science; German, Italian, Japanese and
 * Korean editions carry the same text).  "ARL2 abstract" is the authors'
 * English abstract of arXiv 2605.16579v2 (fugumt.com paper_check page).
 *
 * What one hybrid layer computes, per stream b and head h, for frame N:
 *   intra-frame branch   O_intra = softmax(Q K^T * scale) V over the frame's
 *                        L tokens, bidirectional, no mask
 *                        (ARL2 summary, section 2.1, intra-frame branch);
 *   feature maps         Q' = Q phi_q, K' = rownorm2(K phi_k), V' = V phi_v
 *                        (section 2.1, adaptation by per-head grouped 1x1 maps);
 *   inter-frame read-out O_inter = Q' S_{N-1}   (section 2.1, output);
 *   output               O = O_intra + O_inter;
 *   state write          S_N = alpha S_{N-1} + c K'^T diag(beta)(V' - K' S_{N-1})
 *                        (section 2.1, state update), once per frame on the clean
 *                        pass only, every token reading the same S_{N-1}
 *                        (section 2.2, frame-level access and clean-pass updates;
 *                        ARL2 abstract).
 *
 * Conventions shared by every call:
 *   - Tensor pointers are DEVICE pointers owned by the caller, 16-byte
 *     aligned, contiguous, in the handle's dtype (float32 or bf16).
 *       Q, K, V, O : [B, L, H, d] token-major (row = token, then head, then
 *                    channel); O must not overlap Q, K or V.
 *       phi_*      : [H, d, d] row-major, Q' = Q phi (q'_j = sum_i q_i phi[i][j]).
 *       alpha      : float32 [B, H]      (one decay gate per stream and head).
 *       beta       : float32 [B, H, L]   (one write strength per token).
 *       state      : float32 [B, H, d, d], S[b][h][i][j] with i over K' and
 *                    j over V' channels.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Calls are asynchronous on that stream; their return value covers argument
 *     and launch errors only.  Errors raised inside kernels (a bounded wait that
 *     ran out) are recorded in the handle and returned by arl2_last_error().
 *   - A handle must not be used from two streams at once; calls on one handle
 *     execute in stream order.  The attention and projection-GEMM kernels are
 *     launched with programmatic stream serialisation: their CTAs may start
 *     (barrier and tensor-memory set-up only) while the kernel ahead of them
 *     on the stream finishes, and wait for its completion before any global
 *     memory access, so the stream's ordering of memory effects is unchanged.
 *   - No C++ exception crosses this interface.
 *   - Supported shapes: bf16 needs head_dim = 128; float32 needs head_dim <= 128
 *     and tokens_per_frame <= 4096.  Anything else returns ARL2_ERR_UNSUPPORTED.
 */
#ifndef ARL2_H
#define ARL2_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ARL2_OK = 0,
  ARL2_ERR_INVALID_ARGUMENT = 1, /* null or misaligned pointer, bad handle, bad size */
  ARL2_ERR_UNSUPPORTED = 2,      /* a shape or dtype outside the supported set */
  ARL2_ERR_OUT_OF_MEMORY = 3,    /* a device allocation of the library failed */
  ARL2_ERR_CUDA = 4,             /* a CUDA runtime call or kernel launch failed */
  ARL2_ERR_TIMEOUT = 5,          /* a bounded device-side wait ran out */
  ARL2_ERR_NO_DEVICE = 6,        /* no usable CUDA device / driver */
  ARL2_ERR_SCRATCH_LIMIT = 7,    /* sizes need more than the fixed scratch of
                                    arl2_state_write_noalloc */
  ARL2_ERR_BOUNDS = 8            /* debug builds (libarl2_debug.so) only: a
                                    kernel's index check failed and the access
                                    was skipped; surfaced by arl2_last_error */
} arl2_status;

typedef enum { ARL2_F32 = 0, ARL2_BF16 = 1 } arl2_dtype;

/* Test-only flags of arl2_config.flags: return only one branch of O. */
#define ARL2_INTRA_ONLY 1u
#define ARL2_INTER_ONLY 2u

typedef struct {
  int32_t batch;            /* B independent streams, >= 1 */
  int32_t heads;            /* H, >= 1 */
  int32_t head_dim;         /* d */
  int32_t tokens_per_frame; /* L, >= 1 */
  int32_t dtype;            /* arl2_dtype of Q, K, V, O and phi */
  float softmax_scale;      /* 0 => 1/sqrt(head_dim) */
  float corr_scale;         /* c of the state write; < 0 => 1/L (mean over the frame's tokens) */
  uint32_t flags;           /* 0, or ARL2_INTRA_ONLY / ARL2_INTER_ONLY (tests only) */
} arl2_config;

typedef struct arl2_state* arl2_state_t;
typedef struct arl2_kv* arl2_kv_t;

/* Create a hybrid-layer handle with S_0 = 0 and frame counter 0.
 * phi_q, phi_k, phi_v: device [H, d, d] in cfg->dtype; the library copies them
 * (the caller may free them after the call returns).  The handle owns its
 * state double buffer and work space on the current device.
 * Errors: INVALID_ARGUMENT (null pointers, bad sizes), UNSUPPORTED (shape),
 * OUT_OF_MEMORY (no partial handle is left behind), CUDA. */
arl2_status arl2_state_init(const arl2_config* cfg, const void* phi_q, const void* phi_k,
                            const void* phi_v, void* stream, arl2_state_t* out);

/* One denoising step of a frame (ARL2 summary, section 2.2, clean-pass updates:
 * denoising steps query the state and never write it):
 *   O = softmax(Q K^T * scale) V + (Q phi_q) S_{N-1}.
 * Reads the state, writes only O. */
arl2_status arl2_frame_query(arl2_state_t h, const void* q, const void* k, const void* v, void* o,
                             void* stream);

/* The clean pass of frame N: O as in arl2_frame_query from S_{N-1}, then the
 * frame's single state write
 *   S_N = alpha S_{N-1} + c K'^T diag(beta) (V' - K' S_{N-1}),
 * then the frame counter increments (ARL2 summary, sections 2.1 and 2.2). */
arl2_status arl2_frame_commit(arl2_state_t h, const void* q, const void* k, const void* v,
                              const float* alpha, const float* beta, void* o, void* stream);

/* Query and commit with Q, K and V as strided views of wider token rows, as
 * a fused QKV projection writes them ([B, L, 3 * H * d] with K and V at column
 * offsets H*d and 2*H*d): token rows are `ld` elements apart instead of H*d.
 * bf16 handles only; ld >= H * d and a multiple of 8 (16-byte pitch); ld = 0
 * means contiguous, the same as arl2_frame_query / arl2_frame_commit, which
 * these calls equal bit for bit on the same values.  O stays contiguous and
 * must not overlap the views' spans.  Errors: INVALID_ARGUMENT (also for an
 * f32 handle with ld != 0), CUDA. */
arl2_status arl2_frame_query_strided(arl2_state_t h, const void* q, const void* k, const void* v, int64_t ld,
                                     void* o, void* stream);
arl2_status arl2_frame_commit_strided(arl2_state_t h, const void* q, const void* k, const void* v, int64_t ld,
                                      const float* alpha, const float* beta, void* o, void* stream);

/* Token-level access: the access rule that the ablation of the ARL2 summary
 * (section 4) reports as worse than frame-level access (section 2.2).  Within
 * the pass, token t reads the state left by the tokens before it, and the
 * update of section 2.1 runs one token at a time with a per-token decay:
 *   o_t   = O_intra,t + q'_t S^(t-1),   S^(0) = the handle's current state,
 *   S^(t) = a_t S^(t-1) + c beta_t k'_t^T (v'_t - k'_t S^(t-1)),
 * c being the handle's corr_scale.  The frame-level gate alpha corresponds to
 * a = (alpha, 1, ..., 1).
 * alpha_tok, beta: device float32 [B, H, L], 16-byte aligned.
 * arl2_token_query leaves the state as it is (denoising passes never write
 * it); arl2_token_commit makes S^(L) the current state, advances the frame
 * counter, and refreshes what the frame-level calls read, so the two kinds of
 * call may follow one another on one handle.
 * bf16 handles only.  The first token-level call on a handle allocates its
 * scratch (about 5.2 KB per token and head) with cudaMalloc and adds it to
 * arl2_state_device_bytes, so that first call must not be made while a
 * stream is being captured into a CUDA graph (it fails there with
 * OUT_OF_MEMORY or CUDA); later calls allocate nothing.  The arithmetic past the intra-frame
 * branch is float32.  Errors: INVALID_ARGUMENT, UNSUPPORTED (an f32 handle),
 * OUT_OF_MEMORY, CUDA. */
arl2_status arl2_token_query(arl2_state_t h, const void* q, const void* k, const void* v, const float* alpha_tok,
                             const float* beta, void* o, void* stream);
arl2_status arl2_token_commit(arl2_state_t h, const void* q, const void* k, const void* v, const float* alpha_tok,
                              const float* beta, void* o, void* stream);

/* Copy the current state (float32 [B, H, d, d]) to device memory `dst` and the
 * frame counter to *frame (host pointer, may be null).  Synchronous with
 * respect to `stream` for *frame only; the copy is enqueued on `stream`. */
arl2_status arl2_state_get(arl2_state_t h, float* dst, int64_t* frame, void* stream);

/* Replace the current state with device memory `src` (float32 [B, H, d, d]) and
 * set the frame counter: checkpoint / resume of a stream. */
arl2_status arl2_state_set(arl2_state_t h, const float* src, int64_t frame, void* stream);

/* Synchronise the handle's last stream and return (and clear) the first error
 * recorded by its kernels, ARL2_OK if none. */
arl2_status arl2_last_error(arl2_state_t h);

/* Device bytes held by the handle.  Fixed at init and independent of the
 * frame index, with one exception: the first token-level call
 * (arl2_token_query / arl2_token_commit) allocates that call's scratch and
 * adds it to the count, which then stays constant again. */
int64_t arl2_state_device_bytes(arl2_state_t h);

/* Wall-clock limit of one device-side wait in the handle's kernels (default
 * 1 second).  0 restores the default. */
arl2_status arl2_state_set_wait_limit(arl2_state_t h, uint64_t limit_ns);

arl2_status arl2_state_destroy(arl2_state_t h);

/* ---- Softmax layers kept from the teacher, with a growing KV cache --------
 * (ARL2 summary, section 1: the KV cache grows with every generated block.)
 * The queries of frame n attend, with no mask, to the clean keys and values
 * of frames 0..n-1 followed by the current pass's own K and V.  A query pass
 * leaves the cache's committed frames unchanged; a commit appends its K and V
 * as frame n.  The cache is [B, max_frames * L, H, d] in cfg->dtype. */
arl2_status arl2_kv_init(const arl2_config* cfg, int32_t max_frames, void* stream, arl2_kv_t* out);
arl2_status arl2_kv_query(arl2_kv_t kv, const void* q, const void* k, const void* v, void* o,
                          void* stream);
arl2_status arl2_kv_commit(arl2_kv_t kv, const void* q, const void* k, const void* v, void* o,
                           void* stream);
/* As arl2_kv_query / arl2_kv_commit with Q, K and V read as strided views
 * (token rows `ld` elements apart; bf16 only; ld >= H * d, a multiple of 8;
 * 0 = contiguous), bit-identical to the contiguous calls on the same values.
 * Errors as arl2_frame_query_strided. */
arl2_status arl2_kv_query_strided(arl2_kv_t kv, const void* q, const void* k, const void* v, int64_t ld,
                                  void* o, void* stream);
arl2_status arl2_kv_commit_strided(arl2_kv_t kv, const void* q, const void* k, const void* v, int64_t ld,
                                   void* o, void* stream);
int64_t arl2_kv_frames(arl2_kv_t kv);
int64_t arl2_kv_device_bytes(arl2_kv_t kv);
arl2_status arl2_kv_last_error(arl2_kv_t kv);
arl2_status arl2_kv_destroy(arl2_kv_t kv);

/* ---- Hybrid attention block (the layer around the hot path) ----------------
 * One hybrid layer with the projections a DiT attention block puts around it
 * (ARL2 summary, section 2.1: the frozen pretrained Q/K/V projections feed
 * both branches; alpha and beta are per-token learned projections), bf16 with
 * fp32 accumulation, for a hidden size D = H * 128:
 *   Q = X W_qkv[:, 0:D],  K = X W_qkv[:, D:2D],  V = X W_qkv[:, 2D:3D]
 *   O = the hybrid layer's output on (Q, K, V)  (arl2_frame_query / commit)
 *   Y = O W_o
 * and, on the commit (clean) pass, the gates from the tokens:
 *   alpha[b][h]   = sigmoid( mean over t of (X W_gate)[b][t][h] )
 *   beta[b][h][t] = sigmoid( (X W_gate)[b][t][H + h] )
 * (the pages fix neither the gates' inputs nor their pooling; a head-wise
 * alpha from the frame's mean token and a per-token beta are this build's
 * reading).  No position encoding is applied: Q and K enter the layer as
 * projected.  The projections are plain GEMMs (this library's tcgen05 GEMM,
 * arl2_gemm_bf16: fp32 accumulate, bf16 results): one against
 * [W_qkv | W_gate] (the layer reads Q, K and V as strided views of its rows),
 * one against W_o.
 *   cfg     : bf16 configuration with head_dim 128 (hidden D = heads * 128).
 *   w_qkv   : device bf16 [D, 3D] row-major (X W: y_j = sum_i x_i W[i][j]);
 *   w_o     : device bf16 [D, D];  w_gate : device bf16 [D, 2H] (alpha columns
 *             first, then beta columns);  phi_q, phi_k, phi_v as for
 *             arl2_state_init.  Every weight is copied at init.
 *   x, y    : device bf16 [B, L, D] (token-major; y must not overlap x).
 * The block owns one hybrid-layer handle (its state, KV-free) and its work
 * space (Q, K, V, O, gates: about 5 * B * L * D * 2 bytes, fixed at init).  arl2_block_layer() returns that handle
 * for state get/set, last_error and the device-byte count; it is destroyed
 * with the block.  Errors: INVALID_ARGUMENT, UNSUPPORTED (not bf16 / d != 128),
 * OUT_OF_MEMORY, CUDA. */
typedef struct arl2_block* arl2_block_t;
arl2_status arl2_block_init(const arl2_config* cfg, const void* w_qkv, const void* w_o, const void* w_gate,
                            const void* phi_q, const void* phi_k, const void* phi_v, void* stream,
                            arl2_block_t* out);
arl2_status arl2_block_query(arl2_block_t blk, const void* x, void* y, void* stream);
arl2_status arl2_block_commit(arl2_block_t blk, const void* x, void* y, void* stream);
arl2_state_t arl2_block_layer(arl2_block_t blk);
arl2_status arl2_block_destroy(arl2_block_t blk);

/* The attention block's projection GEMM on its own: C = A B with A [M, K],
 * B [K, N] and C [M, N] row-major bf16 device matrices (leading dimensions
 * lda >= K, ldb >= N, ldc >= N elements, each a multiple of 8; pointers
 * 16-byte aligned), fp32 accumulation, C rounded to bf16.  This is the
 * token-by-weight product that turns the block's input X into Q | K | V | gate
 * logits and the layer's output O into Y (ARL2 summary, section 2.1: the frozen
 * Q/K/V projections feed both branches).  C must not overlap A or B.
 * Errors: INVALID_ARGUMENT (null or misaligned pointers, bad sizes or leading
 * dimensions, overlap), NO_DEVICE, CUDA.  A device-side wait that runs out is
 * not reported here: the call has no handle; the block reports it through its
 * layer (arl2_last_error of arl2_block_layer). */
arl2_status arl2_gemm_bf16(const void* a, int64_t lda, const void* b, int64_t ldb, void* c, int64_t ldc, int64_t m,
                           int64_t n, int64_t k, void* stream);

/* Diagnostic, host only (no device is touched): the work partition the
 * attention kernel uses for `batch` streams of `heads` heads with q_len query
 * rows and kv_len keys on `pairs` CTA pairs.  The (stream, head) slabs are cut
 * into blocks of 256 query rows, each block into key tiles of 128; every pair
 * walks its own list of segments (a run [j0, j1) of key tiles of one block).
 * A block split across pairs is finished by the pair holding key tile 0, which
 * merges the pieces of the n_contrib pairs right after it.  On return
 * *n_pairs is the pairs used (<= pairs), *n_segs the segments, seg_first
 * [*n_pairs + 1] the offsets of each pair's list and segs [*n_segs][5] the
 * segments as (slab = stream * heads + head, block, j0, j1, n_contrib).
 * segs must hold max_segs segments, seg_first 97 entries.
 * Errors: INVALID_ARGUMENT (null pointers, sizes < 1, pairs > 96),
 * UNSUPPORTED (the problem does not fit the partition's encoding or more than
 * max_segs segments). */
arl2_status arl2_attn_partition(int batch, int heads, int q_len, int kv_len, int pairs, int32_t* segs, int max_segs,
                                int32_t* seg_first, int* n_segs, int* n_pairs);

/* ---- State write without allocation ---------------------------------------
 * The paper has no counterpart to this call; it is a deployment aid.  Some
 * callers cannot call cudaMalloc: code that runs while a CUDA graph is being
 * captured, a host that must keep a fixed device-memory budget for the
 * process's whole life, or an embedding runtime whose allocator owns the
 * device and forbids allocations behind its back.  For them this call
 * computes one frame's state write,
 *   S_next = alpha S_prev + c K'^T diag(beta) (V' - K' S_prev),
 * K' = rownorm2(K phi_k), V' = V phi_v, with the same kernels as
 * arl2_frame_commit, but with no handle and without allocating anything: its
 * work space (transposed phi_k and phi_v, a bf16 copy of S_prev, and the
 * per-128-token partial sums) lives in one static device array of
 * ARL2_NOALLOC_SCRATCH_BYTES that every GPU loading the library holds until
 * the process exits.
 *   cfg       : bf16 configuration (head_dim 128); flags and softmax_scale are
 *               ignored; corr_scale < 0 means c = 1/L.
 *   k, v      : device bf16 [B, L, H, 128];  phi_k, phi_v : device bf16 [H, 128, 128]
 *               as given to arl2_state_init;
 *   S_prev    : device float32 [B, H, 128, 128];  alpha : float32 [B, H];
 *   beta      : float32 [B, H, L];  S_next : device float32 [B, H, 128, 128];
 *   dev_error : device uint32, set to 0 by the call and to an arl2_status by a
 *               kernel whose bounded wait ran out (read it after a sync).
 * S_next and dev_error may share no byte with any input or with each other
 * (INVALID_ARGUMENT otherwise).
 * All pointers are caller-owned and 16-byte aligned.  The scratch needed is
 *   2 * H * 32768 + 2 * B * H * 32768 + B * H * ceil(L / 128) * 65536 bytes
 * (each part rounded up to 1 KiB); more than ARL2_NOALLOC_SCRATCH_BYTES returns
 * ARL2_ERR_SCRATCH_LIMIT before any CUDA call.  The first call on a device
 * looks up the array's device address (once per device, with that device
 * current); make that first call before any stream capture begins.  The
 * library keeps that address for the life of the process, so it must not
 * outlive the device context it was looked up in: after cudaDeviceReset (or
 * any other teardown of the device's primary context) do not call this entry
 * point again in the same process.  Every
 * call shares the one array and leaves its contents behind, so calls whose
 * kernels overlap on the GPU (other streams, other host threads) race:
 * serialise them.  Errors: INVALID_ARGUMENT, UNSUPPORTED, SCRATCH_LIMIT, CUDA. */
#define ARL2_NOALLOC_SCRATCH_BYTES (16u << 20)
arl2_status arl2_state_write_noalloc(const arl2_config* cfg, const void* k, const void* v,
                                     const void* phi_k, const void* phi_v, const float* S_prev,
                                     const float* alpha, const float* beta, float* S_next,
                                     uint32_t* dev_error, void* stream);

/* ---- Diagnostics -----------------------------------------------------------
 * Run one kernel whose bounded wait is on a barrier that nothing completes,
 * with the given limit; returns ARL2_ERR_TIMEOUT when the limit worked (the
 * kernel returned and reported it) -- used by the failure-detection tests. */
arl2_status arl2_selftest_wait_timeout(uint64_t limit_ns, void* stream);

/* y[i] = 2^x[i] (device float32 arrays of n values) through the FMA-pipe
 * exponential the attention kernel uses for part of its softmax (a degree-3
 * polynomial after rounding x to an integer; inputs clamped to [-125, 125];
 * relative error <= 1.0e-4).  The attention kernel takes it for 3 of the 16
 * column pairs of every 32-column chunk, in a paired form with the same
 * operations, and the MUFU for the rest.  For accuracy tests of that routine. */
arl2_status arl2_selftest_exp2(const float* x, float* y, int64_t n, void* stream);

const char* arl2_status_string(arl2_status s);
int32_t arl2_abi_version(void);

/* 1 in the debug build (libarl2_debug.so, kernels compiled with
 * -DARL2_DEBUG_BOUNDS: each checks the indices it takes from its parameters and
 * launch shape before it uses them, skips the access when a check fails and
 * records ARL2_ERR_BOUNDS, which arl2_last_error returns), 0 in the release
 * build (libarl2.so), whose kernels carry no such checks.  Needs no device. */
int32_t arl2_debug_bounds_enabled(void);

#ifdef __cplusplus
}
#endif

#endif /* ARL2_H */
