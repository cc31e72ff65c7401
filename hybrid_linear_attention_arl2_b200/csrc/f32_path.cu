// float32 path of the hybrid layer: plain FMA (SIMT) kernels for head_dim <= 128
// and up to 4096 tokens per frame.  tcgen05 has no full-fp32 MMA kind and tf32
// cannot hold the float32 tolerance, so this path stays on the CUDA cores; it
// serves the small float32 streams.
//
//  f32_attn_kernel    one warp per query token: online softmax over the keys
//                     (ARL2 summary, section 2.1, intra-frame branch) plus the
//                     read-out (q phi_q) S_{N-1} (section 2.1, output);
//  f32_commit_kernel  one CTA per (stream, head): the frame's state write
//                     S_N = alpha S + c K'^T diag(beta)(V' - K'S) (section 2.1,
//                     state update), tokens in chunks of 16, every token
//                     reading the same S_{N-1} (section 2.2).

#include <math.h>

#include "params.h"

namespace arl2 {

constexpr int kF32Warps = 4;

__global__ void __launch_bounds__(kF32Warps * 32) f32_attn_kernel(const F32AttnParams p) {
  __shared__ float sq[kF32Warps][128];
  __shared__ float sqp[kF32Warps][128];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kF32Warps + warp;
  const int h = blockIdx.y, b = blockIdx.z;
  if (t >= p.q_len) return;
  const int d = p.d;
  const float* qrow = p.q + ((size_t(b) * p.q_len + t) * p.heads + h) * d;
  float qv[4], acc[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int c = lane + 32 * u;
    qv[u] = c < d ? qrow[c] : 0.f;
    acc[u] = 0.f;
    sq[warp][c] = qv[u];
  }
  float m = -INFINITY, l = 0.f;
  for (int j = 0; j < p.kv_len; ++j) {
    const size_t off = ((size_t(b) * p.kv_stride + j) * p.heads + h) * d;
    float s = 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int c = lane + 32 * u;
      if (c < d) s = fmaf(qv[u], p.k[off + c], s);
    }
#pragma unroll
    for (int sh = 16; sh > 0; sh >>= 1) s += __shfl_xor_sync(0xffffffffu, s, sh);
    s *= p.scale;
    const float m_new = fmaxf(m, s);
    const float f = expf(m - m_new);  // 0 on the first key (m = -inf)
    const float e = expf(s - m_new);
    l = l * f + e;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int c = lane + 32 * u;
      acc[u] = acc[u] * f + (c < d ? e * p.v[off + c] : 0.f);
    }
    m = m_new;
  }
  float out[4];
  const bool intra = !(p.flags & 2u), inter = p.phi_q && !(p.flags & 1u);
#pragma unroll
  for (int u = 0; u < 4; ++u) out[u] = intra ? acc[u] / l : 0.f;
  if (inter) {
    __syncwarp();
    const float* ph = p.phi_q + size_t(h) * d * d;
#pragma unroll
    for (int u = 0; u < 4; ++u) {  // q' = q phi_q
      const int c = lane + 32 * u;
      float s = 0.f;
      if (c < d)
        for (int i = 0; i < d; ++i) s = fmaf(sq[warp][i], ph[size_t(i) * d + c], s);
      sqp[warp][c] = s;
    }
    __syncwarp();
    const float* S = p.S + (size_t(b) * p.heads + h) * d * d;
#pragma unroll
    for (int u = 0; u < 4; ++u) {  // o_inter = q' S
      const int c = lane + 32 * u;
      float s = 0.f;
      if (c < d)
        for (int i = 0; i < d; ++i) s = fmaf(sqp[warp][i], S[size_t(i) * d + c], s);
      out[u] += s;
    }
  }
  float* orow = p.o + ((size_t(b) * p.q_len + t) * p.heads + h) * d;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int c = lane + 32 * u;
    if (c < d) orow[c] = out[u];
  }
}

constexpr int kChunk = 16;
constexpr int kCommitThreads = 256;

// Shared memory: delta accumulator d*d, K' chunk, V' chunk (then R), K~ norms.
__global__ void __launch_bounds__(kCommitThreads) f32_commit_kernel(const F32CommitParams p) {
  extern __shared__ float sm[];
  const int d = p.d;
  float* acc = sm;                    // d*d
  float* kp = acc + d * d;            // kChunk*d
  float* vp = kp + kChunk * d;        // kChunk*d
  float* inv = vp + kChunk * d;       // kChunk
  const int slab = blockIdx.x;
  const int b = slab / p.heads, h = slab % p.heads;
  const float* Sp = p.S_prev + size_t(slab) * d * d;
  const float* phk = p.phi_k + size_t(h) * d * d;
  const float* phv = p.phi_v + size_t(h) * d * d;
  for (int e = threadIdx.x; e < d * d; e += kCommitThreads) acc[e] = 0.f;
  __syncthreads();
  for (int t0 = 0; t0 < p.L; t0 += kChunk) {
    const int nt = min(kChunk, p.L - t0);
    // K~ = K phi_k and V' = V phi_v for the chunk.
    for (int e = threadIdx.x; e < nt * d; e += kCommitThreads) {
      const int t = e / d, j = e % d;
      const size_t row = ((size_t(b) * p.L + t0 + t) * p.heads + h) * d;
      float sk = 0.f, sv = 0.f;
      for (int i = 0; i < d; ++i) {
        sk = fmaf(p.k[row + i], phk[size_t(i) * d + j], sk);
        sv = fmaf(p.v[row + i], phv[size_t(i) * d + j], sv);
      }
      kp[e] = sk;
      vp[e] = sv;
    }
    __syncthreads();
    for (int t = threadIdx.x; t < nt; t += kCommitThreads) {
      float ss = 0.f;
      for (int j = 0; j < d; ++j) ss = fmaf(kp[t * d + j], kp[t * d + j], ss);
      inv[t] = 1.f / fmaxf(sqrtf(ss), 1e-12f);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < nt * d; e += kCommitThreads) kp[e] *= inv[e / d];
    __syncthreads();
    // R = beta (V' - K' S_{N-1}), in place of V'.
    float r_local[(kChunk * 128 + kCommitThreads - 1) / kCommitThreads];
    int n_local = 0;
    for (int e = threadIdx.x; e < nt * d; e += kCommitThreads) {
      const int t = e / d, j = e % d;
      float pred = 0.f;
      for (int i = 0; i < d; ++i) pred = fmaf(kp[t * d + i], Sp[size_t(i) * d + j], pred);
      const float bt = p.beta[size_t(slab) * p.L + t0 + t];
      r_local[n_local++] = bt * (vp[e] - pred);
    }
    __syncthreads();
    n_local = 0;
    for (int e = threadIdx.x; e < nt * d; e += kCommitThreads) vp[e] = r_local[n_local++];
    __syncthreads();
    // delta += K'^T R
    for (int e = threadIdx.x; e < d * d; e += kCommitThreads) {
      const int i = e / d, j = e % d;
      float s = acc[e];
      for (int t = 0; t < nt; ++t) s = fmaf(kp[t * d + i], vp[t * d + j], s);
      acc[e] = s;
    }
    __syncthreads();
  }
  const float a = p.alpha[slab];
  for (int e = threadIdx.x; e < d * d; e += kCommitThreads)
    p.S_next[size_t(slab) * d * d + e] = fmaf(a, Sp[e], p.corr * acc[e]);
}

cudaError_t launch_f32_attn(const F32AttnParams& p, int batch, cudaStream_t stream) {
  dim3 grid((p.q_len + kF32Warps - 1) / kF32Warps, p.heads, batch);
  f32_attn_kernel<<<grid, kF32Warps * 32, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_f32_commit(const F32CommitParams& p, int batch, cudaStream_t stream) {
  const size_t smem = (size_t(p.d) * p.d + 2 * kChunk * p.d + kChunk) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(f32_commit_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  f32_commit_kernel<<<batch * p.heads, kCommitThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace arl2
