// Token-level access: the access rule that the ablation of the ARL2 summary
// (section 4) reports as worse than the frame-level rule of section 2.2.
// Within one pass, token t of the frame reads the state left by the tokens
// before it, and the update of section 2.1 runs one token at a time:
//
//   o_t   = O_intra,t + q'_t S^(t-1),           S^(0) = S_{N-1},
//   S^(t) = a_t S^(t-1) + c beta_t k'_t^T (v'_t - k'_t S^(t-1)),
//
// with a per-token decay a_t (the frame-level gate alpha is a = (alpha, 1,
// ..., 1); a general a is the per-token gate the section 2.1 wording allows).
//
// The scan is cut into 128-token chunks.  For a chunk with entering state S,
// decay products g (g_prev[t] = a_0..a_{t-1}, g_tail[s] = a_{s+1}..a_{n-1},
// g_C = all of them, G[t][s] = a_{s+1}..a_{t-1} for s < t) and w = c beta,
// the rows u_t = w_t (v_t - k_t S^(t-1)) solve a unit-lower-triangular
// system A u = w (v - g_prev k S), A = I + diag(w) (G * K K^T).  With
// T = A^-1, W = T diag(w g_prev) K and U' = T diag(w) V the chunk is the
// affine map
//
//   S_next = M S + N,        M = g_C I - Kt^T W,  N = Kt^T U',  Kt = diag(g_tail) K,
//   O      = Qt S + Ot,      Qt = diag(g_prev) Q - P W,  Ot = P U',  P = G * (Q K^T),
//
// whose operands need no state.  So: (1) the maps per token; (2) one block
// per (stream, head, chunk) builds M, N, Qt, Ot; (3) one block per (stream,
// head, 16-column slab of S) runs S_next = M S + N over the chunks in order;
// (4) one block per (stream, head, chunk) adds Qt S + Ot to the intra-frame
// output.  This first version computes in fp32 on the CUDA cores.

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "layer.h"
#include "params.h"

namespace arl2 {
namespace {

constexpr int kD = 128;         // head dim
constexpr int kChunk = 128;     // tokens per chunk
constexpr int kLd = kChunk + 1;  // padded row pitch of the chunk matrices in shared memory
constexpr int kSlab = 16;       // state columns per block of the sequential kernel
constexpr size_t kChunkSmem = (3 * size_t(kChunk) * kLd + 3 * kChunk) * sizeof(float);

__device__ __forceinline__ float bf(const __nv_bfloat16 x) { return __bfloat162float(x); }

// (1) One block per (stream, token, head), one thread per channel j:
// q'_j = sum_i q_i phi_q[i][j], k' likewise then divided by max(|k'|, 1e-12),
// v' likewise.  Rows go to [B, H, L, 128] f32.
__global__ void __launch_bounds__(kD) tok_maps_kernel(TokenParams p) {
  const int r = blockIdx.x;  // (b * L + t) * H + h
  const int h = r % p.H, bt = r / p.H, t = bt % p.L, b = bt / p.L;
  const int j = threadIdx.x;
  __shared__ float xq[kD], xk[kD], xv[kD], red[kD / 32];
  const size_t row = (size_t(bt) * p.H + h) * kD;
  xq[j] = bf(p.q[row + j]);
  xk[j] = bf(p.k[row + j]);
  xv[j] = bf(p.v[row + j]);
  __syncthreads();
  const __nv_bfloat16* pq = p.phi_q + size_t(h) * kD * kD + j;        // pq[i * kD] = phi_q[h][i][j]
  const __nv_bfloat16* pk = p.phi_k_t + (size_t(h) * kD + j) * kD;    // pk[i] = phi_k[h][i][j]
  const __nv_bfloat16* pv = p.phi_v_t + (size_t(h) * kD + j) * kD;    // pv[i] = phi_v[h][i][j]
  float aq = 0.f, ak = 0.f, av = 0.f;
  for (int i = 0; i < kD; ++i) {
    aq = fmaf(xq[i], bf(pq[size_t(i) * kD]), aq);
    ak = fmaf(xk[i], bf(pk[i]), ak);
    av = fmaf(xv[i], bf(pv[i]), av);
  }
  float sq = ak * ak;
  for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
  if ((j & 31) == 0) red[j >> 5] = sq;
  __syncthreads();
  const float inv = 1.f / fmaxf(sqrtf(red[0] + red[1] + red[2] + red[3]), 1e-12f);
  const size_t out = ((size_t(b) * p.H + h) * p.L + t) * kD + j;
  p.qp[out] = aq;
  p.kp[out] = ak * inv;
  p.vp[out] = av;
}

// (2) One block per (stream, head, chunk), 128 threads.
__global__ void __launch_bounds__(kChunk) tok_chunk_kernel(TokenParams p) {
  extern __shared__ float sm[];
  float* X0 = sm;                    // A, then W
  float* X1 = X0 + kChunk * kLd;     // T = A^-1, then U'
  float* X2 = X1 + kChunk * kLd;     // P
  float* w = X2 + kChunk * kLd;      // c beta
  float* g_prev = w + kChunk;
  float* g_tail = g_prev + kChunk;
  __shared__ float g_all;
  const int c = blockIdx.x % p.n_chunks, bh = blockIdx.x / p.n_chunks;
  const int t0 = c * kChunk, n = min(kChunk, p.L - t0);
  const int tid = threadIdx.x;
  const size_t tok0 = size_t(bh) * p.L + t0;  // row of the chunk's first token in the [B, H, L] arrays
  const float* Kc = p.kp + tok0 * kD;
  const float* Qc = p.qp + tok0 * kD;
  const float* Vc = p.vp + tok0 * kD;
  const float* a = p.alpha_tok + tok0;
  if (tid < n) w[tid] = p.corr * p.beta[tok0 + tid];
  if (tid == 0) {
    float g = 1.f;
    for (int t = 0; t < n; ++t) {
      g_prev[t] = g;
      g *= a[t];
    }
    g_all = g;
    g = 1.f;
    for (int s = n - 1; s >= 0; --s) {
      g_tail[s] = g;
      g *= a[s];
    }
  }
  __syncthreads();
  // A (strictly lower part; the unit diagonal is implicit) and P, row t per thread
  if (tid < n) {
    const float* kt = Kc + size_t(tid) * kD;
    const float* qt = Qc + size_t(tid) * kD;
    float g = 1.f;  // G[t][s], s going down from t - 1
    for (int s = tid - 1; s >= 0; --s) {
      const float* ks = Kc + size_t(s) * kD;
      float dk = 0.f, dq = 0.f;
      for (int i = 0; i < kD; ++i) {
        dk = fmaf(kt[i], ks[i], dk);
        dq = fmaf(qt[i], ks[i], dq);
      }
      X0[tid * kLd + s] = w[tid] * g * dk;
      X2[tid * kLd + s] = g * dq;
      g *= a[s];
    }
  }
  __syncthreads();
  // T = A^-1 by forward substitution, column j per thread (each thread reads
  // and writes only its own column of T)
  if (tid < n) {
    const int j = tid;
    for (int i = 0; i < n; ++i) {
      float x = i == j ? 1.f : 0.f;
      if (i > j)
        for (int k = j; k < i; ++k) x = fmaf(-X0[i * kLd + k], X1[k * kLd + j], x);
      X1[i * kLd + j] = x;
    }
  }
  __syncthreads();
  // W = T diag(w g_prev) K and U' = T diag(w) V, column j per thread (128 columns)
  const int j = tid;
  for (int t = 0; t < n; ++t) {
    float aw = 0.f, au = 0.f;
    for (int s = 0; s <= t; ++s) {
      const float tv = X1[t * kLd + s];
      aw = fmaf(tv * w[s] * g_prev[s], Kc[size_t(s) * kD + j], aw);
      au = fmaf(tv * w[s], Vc[size_t(s) * kD + j], au);
    }
    p.w[(tok0 + t) * kD + j] = aw;
    p.u[(tok0 + t) * kD + j] = au;
  }
  __syncthreads();  // every thread is done with T and A: W into X0, U' into X1
  for (int t = 0; t < n; ++t) {
    X0[t * kLd + j] = p.w[(tok0 + t) * kD + j];
    X1[t * kLd + j] = p.u[(tok0 + t) * kD + j];
  }
  __syncthreads();
  // M = g_C I - Kt^T W and N = Kt^T U', column j per thread, rows i over the state
  const size_t mn0 = (size_t(bh) * p.n_chunks + c) * kD * kD;
  for (int i = 0; i < kD; ++i) {
    float am = i == j ? g_all : 0.f, an = 0.f;
    for (int s = 0; s < n; ++s) {
      const float kt = g_tail[s] * Kc[size_t(s) * kD + i];
      am = fmaf(-kt, X0[s * kLd + j], am);
      an = fmaf(kt, X1[s * kLd + j], an);
    }
    p.m[mn0 + size_t(i) * kD + j] = am;
    p.n[mn0 + size_t(i) * kD + j] = an;
  }
  // Qt = diag(g_prev) Q - P W and Ot = P U', column j per thread
  for (int t = 0; t < n; ++t) {
    float aq = g_prev[t] * Qc[size_t(t) * kD + j], ao = 0.f;
    for (int s = 0; s < t; ++s) {
      const float pv = X2[t * kLd + s];
      aq = fmaf(-pv, X0[s * kLd + j], aq);
      ao = fmaf(pv, X1[s * kLd + j], ao);
    }
    p.qt[(tok0 + t) * kD + j] = aq;
    p.ot[(tok0 + t) * kD + j] = ao;
  }
}

// (3) One block per (stream, head, 16-column slab of S), thread i = row i:
// S_next = M S + N over the chunks in order; the state entering each chunk is
// kept for (4), and the final one goes to s_out (a commit) or nowhere (a query).
__global__ void __launch_bounds__(kD) tok_state_kernel(TokenParams p) {
  __shared__ float Ss[kD][kSlab];
  const int slab = blockIdx.x % (kD / kSlab), bh = blockIdx.x / (kD / kSlab);
  const int i = threadIdx.x, j0 = slab * kSlab;
  for (int jj = 0; jj < kSlab; ++jj) Ss[i][jj] = p.s_in[(size_t(bh) * kD + i) * kD + j0 + jj];
  __syncthreads();
  for (int c = 0; c < p.n_chunks; ++c) {
    const size_t mn0 = (size_t(bh) * p.n_chunks + c) * kD * kD;
    float acc[kSlab];
    for (int jj = 0; jj < kSlab; ++jj) {
      p.s_chunk[mn0 + size_t(i) * kD + j0 + jj] = Ss[i][jj];
      acc[jj] = p.n[mn0 + size_t(i) * kD + j0 + jj];
    }
    const float* mrow = p.m + mn0 + size_t(i) * kD;
    for (int k = 0; k < kD; ++k) {
      const float mv = mrow[k];
#pragma unroll
      for (int jj = 0; jj < kSlab; ++jj) acc[jj] = fmaf(mv, Ss[k][jj], acc[jj]);
    }
    __syncthreads();
#pragma unroll
    for (int jj = 0; jj < kSlab; ++jj) Ss[i][jj] = acc[jj];
    __syncthreads();
  }
  if (p.s_out)
    for (int jj = 0; jj < kSlab; ++jj) p.s_out[(size_t(bh) * kD + i) * kD + j0 + jj] = Ss[i][jj];
}

// (4) One block per (stream, head, chunk), thread j = channel j:
// o_t += Qt_t S_c + Ot_t on top of the intra-frame output already in o.
__global__ void __launch_bounds__(kD) tok_out_kernel(TokenParams p) {
  extern __shared__ float Sc[];  // [kD][kD], the state entering the chunk
  const int c = blockIdx.x % p.n_chunks, bh = blockIdx.x / p.n_chunks;
  const int b = bh / p.H, h = bh % p.H;
  const int t0 = c * kChunk, n = min(kChunk, p.L - t0);
  const int j = threadIdx.x;
  const size_t mn0 = (size_t(bh) * p.n_chunks + c) * kD * kD;
  for (int i = 0; i < kD; ++i) Sc[i * kD + j] = p.s_chunk[mn0 + size_t(i) * kD + j];
  __syncthreads();
  const size_t tok0 = size_t(bh) * p.L + t0;
  for (int t = 0; t < n; ++t) {
    const float* qrow = p.qt + (tok0 + t) * kD;
    float acc = p.ot[(tok0 + t) * kD + j];
    for (int i = 0; i < kD; ++i) acc = fmaf(qrow[i], Sc[i * kD + j], acc);
    const size_t o = ((size_t(b) * p.L + t0 + t) * p.H + h) * kD + j;
    p.o[o] = __float2bfloat16_rn(bf(p.o[o]) + acc);
  }
}

}  // namespace

size_t token_scratch_floats(int B, int H, int L) {
  const size_t rows = size_t(B) * H * L * kD;
  const size_t mats = size_t(B) * H * ((L + kChunk - 1) / kChunk) * kD * kD;
  return 7 * rows + 3 * mats;
}

void token_bind_scratch(TokenParams& p, float* base) {
  const size_t rows = size_t(p.B) * p.H * p.L * kD;
  const size_t mats = size_t(p.B) * p.H * p.n_chunks * kD * kD;
  p.qp = base;
  p.kp = p.qp + rows;
  p.vp = p.kp + rows;
  p.w = p.vp + rows;
  p.u = p.w + rows;
  p.qt = p.u + rows;
  p.ot = p.qt + rows;
  p.m = p.ot + rows;
  p.n = p.m + mats;
  p.s_chunk = p.n + mats;
}

cudaError_t launch_token_level(const TokenParams& p, bool with_out, cudaStream_t st) {
  static unsigned done_chunk = 0, done_out = 0;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(tok_chunk_kernel), int(kChunkSmem), &done_chunk);
  if (e != cudaSuccess) return e;
  e = ensure_smem_attr(reinterpret_cast<const void*>(tok_out_kernel), int(kD * kD * sizeof(float)), &done_out);
  if (e != cudaSuccess) return e;
  const unsigned bh = unsigned(p.B) * unsigned(p.H);
  tok_maps_kernel<<<unsigned(p.B) * unsigned(p.L) * unsigned(p.H), kD, 0, st>>>(p);
  tok_chunk_kernel<<<bh * unsigned(p.n_chunks), kChunk, kChunkSmem, st>>>(p);
  tok_state_kernel<<<bh * unsigned(kD / kSlab), kD, 0, st>>>(p);
  if (with_out) tok_out_kernel<<<bh * unsigned(p.n_chunks), kD, kD * kD * sizeof(float), st>>>(p);
  return cudaGetLastError();
}

}  // namespace arl2
