// Launch parameters and launcher declarations shared by the library's
// translation units (kernels and the C ABI).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace arl2 {

constexpr int kAttnMaxGrid = 192;  // persistent CTAs at most (>= the SM count of a B200)

// Fused intra-frame softmax + inter-frame read-out (attn_pair.cu): a
// persistent grid of CTA pairs, each walking its own list of segments (a
// run of key tiles of one 256-row block), see the kernel.
constexpr int kAttnMaxSegs = 1024;  // segments of one launch at most
struct AttnParams {
  int q_len;            // query tokens per stream
  int kv_len;           // valid key/value tokens per stream
  int heads;
  int n_qt;             // query tiles of 128 per (stream, head)
  int n_blk;            // blocks of 256 rows per (stream, head): ceil(n_qt / 2)
  int nkv;              // key tiles of 128
  long long total_units;   // B * H * n_blk * nkv
  int grid;             // persistent CTAs, even (<= kAttnMaxGrid)
  int n_segs;           // entries of seg
  unsigned seg_first[kAttnMaxGrid / 2 + 1];  // pair c walks seg[seg_first[c] .. seg_first[c + 1])
  // one segment: x = bh | (contributors << 28) (the pairs after this one whose
  // pieces a finishing segment merges), y = blk | (j0 << 10) | ((j1 - j0) << 21)
  uint2 seg[kAttnMaxSegs];
  float scale_log2;     // softmax scale * log2(e)
  uint32_t flags;       // 1: intra only, 2: inter only
  int has_inter;        // 1: add Q MqT^T
  float* scratch;       // [grid][kAttnPairSlotFloats] normalised partial O and (m, l) per CTA
  unsigned* ready;      // [grid][kAttnPairFlags] partial-ready flags, zero between launches
  uint32_t* err;        // device error word
  uint64_t wait_limit_ns;
};

// floats of one CTA's partial slot of the CTA-pair kernel (attn_pair.cu): its
// 128 x 128 piece of O normalised by its own l, in bf16 (the first 32 KB, laid
// out as the kernel describes), then from float 16384 m[128] and l[128] in fp32
constexpr int kAttnPairSlotFloats = 128 * 128 + 256;
// ready flags per CTA of the pair kernel (one per epilogue warp)
constexpr int kAttnPairFlags = 4;
// device words of the attention scratch and flags a handle allocates for `sms` SMs
constexpr size_t attn_scratch_floats(int sms) { return size_t(sms) * size_t(kAttnPairSlotFloats); }
constexpr size_t attn_ready_words(int sms) { return size_t(sms) * kAttnPairFlags; }

// State write and read-out preparation (state_bf16.cu).
struct StateParams {
  const float* S_prev;      // [B, H, 128, 128]
  const float* alpha;       // [B, H]
  const float* beta;        // [B, H, L]
  float* partial;           // [B, H, n_chunks, 128, 128]
  float* S_next;            // [B, H, 128, 128]
  __nv_bfloat16* S_next_bf; // [B, H, 128, 128]
  __nv_bfloat16* mqt;       // [B, H, 128, 128]
  int L;
  int heads;
  int n_chunks;
  float corr;
  uint32_t* err;
  uint64_t wait_limit_ns;
  int batch;                // B (the debug build checks the launch shape against it)
};

// float32 path (f32_path.cu).
struct F32AttnParams {
  const float* q;      // [B, q_len, H, d]
  const float* k;      // [B, kv_stride, H, d]
  const float* v;
  float* o;            // [B, q_len, H, d]
  const float* phi_q;  // [H, d, d] (null: no read-out)
  const float* S;      // [B, H, d, d]
  int q_len, kv_len, kv_stride, heads, d;
  float scale;
  uint32_t flags;
};

struct F32CommitParams {
  const float* k;      // [B, L, H, d]
  const float* v;
  const float* phi_k;  // [H, d, d]
  const float* phi_v;
  const float* S_prev; // [B, H, d, d]
  float* S_next;
  const float* alpha;  // [B, H]
  const float* beta;   // [B, H, L]
  int L, heads, d;
  float corr;
};

// tq: Q in 128-row boxes; tk: K in 64-row boxes (a CTA's half of a key tile);
// tv: V in 128-row boxes; tmq: 64-row boxes of the [B*H, 128, 128] MqT slabs
// (read only when has_inter); tmo: the output O [B, q_len, H, 128] in boxes
// of 64 columns x 32 rows, written with tile stores.  p.grid is the CTA count
// (even), p.range is per pair.
cudaError_t launch_attn_pair(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             const CUtensorMap& tmq, const CUtensorMap& tmo, const AttnParams& p,
                             cudaStream_t stream);
// Fills the partition fields of `p` for B streams; max_pairs: the clusters of
// two the device holds at once (attn_pair_capacity).  False if the problem is
// too large for 32-bit unit indices.
bool attn_pair_partition(AttnParams& p, int batch, int max_pairs);
// Clusters of the pair kernel resident at once on the current device (0 on error).
int attn_pair_capacity();
cudaError_t launch_state_partial(const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tpk,
                                 const CUtensorMap& tpv, const CUtensorMap& ts, const StateParams& p, int batch,
                                 cudaStream_t stream);
cudaError_t launch_state_finalize(const StateParams& p, int batch, cudaStream_t stream);
// The whole state write in one launch (state_bf16.cu): one cluster of
// n_chunks CTAs per (stream, head), reducing the chunks' partials on chip in
// chunk order (bit-identical to partial + finalize) and forming MqT into p.mqt.
// Needs n_chunks <= 16 and a device that schedules such clusters.
bool state_fused_supported(int n_chunks, int heads, int batch);
cudaError_t launch_state_fused(const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tpk,
                               const CUtensorMap& tpv, const CUtensorMap& ts, const CUtensorMap& tphiq,
                               const StateParams& p, int batch, cudaStream_t stream);
cudaError_t launch_readout_prep(const CUtensorMap& ts, const CUtensorMap& tphiq, const StateParams& p, int batch,
                                cudaStream_t stream);
cudaError_t launch_f32_attn(const F32AttnParams& p, int batch, cudaStream_t stream);
cudaError_t launch_f32_commit(const F32CommitParams& p, int batch, cudaStream_t stream);
cudaError_t launch_transpose_bf16(const __nv_bfloat16* src, __nv_bfloat16* dst, int slabs, cudaStream_t stream);
cudaError_t launch_to_bf16(const float* src, __nv_bfloat16* dst, size_t n, cudaStream_t stream);
cudaError_t launch_wait_selftest(uint32_t* err, uint64_t limit_ns, cudaStream_t stream);
cudaError_t launch_exp2_poly(const float* x, float* y, long long n, cudaStream_t stream);

// Projection GEMM of the attention block (gemm_bf16.cu): C[M][N] = A[M][K] B[K][N],
// bf16 row-major operands with leading dimensions lda, ldb, ldc (elements,
// multiples of 8), fp32 accumulation, bf16 C.
struct GemmParams {
  int M, N, K;
  uint32_t* err;
  uint64_t wait_limit_ns;
};
cudaError_t gemm_bf16(const void* A, int64_t lda, const void* B, int64_t ldb, void* C, int64_t ldc, const GemmParams& p,
                      int sms, cudaStream_t stream);

// Sets the dynamic shared-memory limit of `func` once per device.
cudaError_t ensure_smem_attr(const void* func, int bytes, unsigned* done_mask);

}  // namespace arl2
