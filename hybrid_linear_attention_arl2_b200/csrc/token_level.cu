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
#include "sm100.cuh"

namespace arl2 {
namespace {

constexpr int kD = 128;         // head dim
constexpr int kChunk = 128;     // tokens per chunk
constexpr int kLd = kChunk + 1;  // padded row pitch of the chunk matrices in shared memory
constexpr int kSlab = 16;       // state columns per block of the sequential kernel
constexpr size_t kChunkSmem = (3 * size_t(kChunk) * kLd + 3 * kChunk) * sizeof(float);

__device__ __forceinline__ float bf(const __nv_bfloat16 x) { return __bfloat162float(x); }

// (1) One CTA per (stream, head, 128-token chunk), 128 threads (thread t =
// token t of the chunk).  The chunk's Q, K and V rows and the head's phi_q,
// phi_k^T and phi_v^T go to shared memory in the 128-byte-swizzle layout of
// two 64-column boxes; three tcgen05 MMAs (M = tokens, N = K = 128, fp32
// accumulation in tensor memory) give Q phi_q, K phi_k and V phi_v; thread t
// reads its rows and writes q'_t, k'_t / max(|k'_t|, 1e-12) and v'_t in f32 to
// [B, H, L, 128].
constexpr uint32_t kMapTile = 32768;   // 128 rows x 128 bf16
constexpr uint32_t kMapHalf = 16384;   // one 64-column box
constexpr int kMapsSmem = int(6 * kMapTile) + 64 + 1024;

// Byte offset of bf16 element (row, col) of a 128-row tile stored as two
// 64-column boxes with the 128-byte swizzle (16-byte chunks of a row XORed
// with row % 8): the layout the tensor cores read through smem_desc_sw128.
__device__ __forceinline__ uint32_t tok_sw128(int row, int col) {
  const int box = col >> 6, cc = col & 63;
  return uint32_t(box) * kMapHalf + uint32_t(row) * 128 + uint32_t(((cc >> 3) ^ (row & 7)) * 16 + (cc & 7) * 2);
}

__global__ void __launch_bounds__(kD, 1) tok_maps_kernel(TokenParams p) {
  extern __shared__ uint8_t tok_smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(tok_smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sX = sm;                   // Q, K, V rows of the chunk (A operands, K-major)
  uint8_t* sF = sm + 3 * kMapTile;    // phi_q (B, MN-major: rows i), phi_k^T, phi_v^T (B, K-major: rows j)
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + 6 * kMapTile);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  const int c = blockIdx.x % p.n_chunks, bh = blockIdx.x / p.n_chunks;
  const int b = bh / p.H, h = bh % p.H;
  const int t0 = c * kChunk, n = min(kChunk, p.L - t0);
  const int tid = threadIdx.x, warp = tid >> 5;
  if (tid == 0) {
    mbar_init(bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc(tmem_holder, 512);
  const __nv_bfloat16* xs[3] = {p.q, p.k, p.v};
  const __nv_bfloat16* fs[3] = {p.phi_q, p.phi_k_t, p.phi_v_t};
  for (int x = tid; x < 3 * 2048; x += kD) {  // 16-byte chunks: tile x >> 11, row (x >> 4) & 127, chunk x & 15
    const int m = x >> 11, r = (x >> 4) & 127, cc = x & 15;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (r < n) v = *reinterpret_cast<const uint4*>(xs[m] + ((size_t(b) * p.L + t0 + r) * p.H + h) * kD + cc * 8);
    *reinterpret_cast<uint4*>(sX + m * kMapTile + tok_sw128(r, cc * 8)) = v;
    const uint4 f = *reinterpret_cast<const uint4*>(fs[m] + (size_t(h) * kD + r) * kD + cc * 8);
    *reinterpret_cast<uint4*>(sF + m * kMapTile + tok_sw128(r, cc * 8)) = f;
  }
  fence_async_smem();  // the tiles were written through the generic proxy
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const WaitCtl w{abort_flag, p.err, p.wait_limit_ns};
  if (tid == 0) {
    const uint32_t xa = smem_u32(sX), fa = smem_u32(sF);
    const uint32_t id_mn = idesc_bf16(128, 128, 0, 1), id_k = idesc_bf16(128, 128, 0, 0);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {  // Q phi_q: phi_q stored [i][j], N = j contiguous (MN-major)
      const uint32_t aoff = (kk >> 2) * kMapHalf + (kk & 3) * 32;
      mma_ss(tmem, smem_desc_sw128(xa + aoff, 16, 1024), smem_desc_sw128(fa + kk * 2048, kMapHalf, 1024), id_mn,
             kk > 0);
    }
#pragma unroll
    for (int m = 1; m < 3; ++m) {  // K phi_k, V phi_v: phi^T stored [j][i], K = i contiguous (K-major)
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t off = (kk >> 2) * kMapHalf + (kk & 3) * 32;
        mma_ss(tmem + m * 128, smem_desc_sw128(xa + m * kMapTile + off, 16, 1024),
               smem_desc_sw128(fa + m * kMapTile + off, 16, 1024), id_k, kk > 0);
      }
    }
    mma_commit(bar);
  }
  bool ok = mbar_wait(bar, 0, w);
  ok = __all_sync(0xffffffffu, ok);
  if (ok) {
    tc_fence_after();
    const uint32_t lane_off = uint32_t(warp * 32) << 16;
    const size_t out = ((size_t(b) * p.H + h) * p.L + t0 + tid) * kD;
    float ss = 0.f;  // |k~_t|^2
#pragma unroll 1
    for (int q = 0; q < 4; ++q) {
      uint32_t r[32];
      tmem_ld32(tmem + 128 + lane_off + q * 32, r);
      tmem_wait_ld();
#pragma unroll
      for (int x = 0; x < 32; ++x) ss = fmaf(__uint_as_float(r[x]), __uint_as_float(r[x]), ss);
    }
    const float inv = 1.f / fmaxf(sqrtf(ss), 1e-12f);
    float* dsts[3] = {p.qp, p.kp, p.vp};
#pragma unroll 1
    for (int m = 0; m < 3; ++m) {
#pragma unroll 1
      for (int q = 0; q < 4; ++q) {
        uint32_t r[32];
        tmem_ld32(tmem + m * 128 + lane_off + q * 32, r);
        tmem_wait_ld();
        if (tid < n) {
          const float sc = m == 1 ? inv : 1.f;
          float4* d4 = reinterpret_cast<float4*>(dsts[m] + out + q * 32);
#pragma unroll
          for (int x = 0; x < 8; ++x)
            d4[x] = make_float4(__uint_as_float(r[4 * x]) * sc, __uint_as_float(r[4 * x + 1]) * sc,
                                __uint_as_float(r[4 * x + 2]) * sc, __uint_as_float(r[4 * x + 3]) * sc);
        }
      }
    }
  } else if (tid == 0) {  // the MMAs land before tensor memory is released
    const uint64_t t_0 = global_timer_ns();
    while (!mbar_try_wait(bar, 0) && global_timer_ns() - t_0 < 10000000ull) {
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
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
  // K K^T and Q K^T of the chunk: K and Q staged in X1 and X2 (rows past n
  // zero), then register-tiled products, thread (ty, tx) = (tid / 8, tid % 8)
  // owning rows 8 ty .. 8 ty + 7 and columns tx + 8 c (c < 16)
  for (int x = tid; x < kChunk * kD; x += kChunk) {
    const int t = x / kD, i = x % kD;
    X1[t * kLd + i] = t < n ? Kc[size_t(t) * kD + i] : 0.f;
    X2[t * kLd + i] = t < n ? Qc[size_t(t) * kD + i] : 0.f;
  }
  __syncthreads();
  {
    const int ty = tid >> 3, tx = tid & 7;
    float acc[8][16];
#pragma unroll 1
    for (int pass = 0; pass < 2; ++pass) {  // pass 0: K K^T into X0; pass 1: Q K^T into X2
      const float* Arows = pass == 0 ? X1 : X2;
#pragma unroll
      for (int r = 0; r < 8; ++r)
#pragma unroll
        for (int c2 = 0; c2 < 16; ++c2) acc[r][c2] = 0.f;
#pragma unroll 4
      for (int i = 0; i < kD; ++i) {
        float av[8], bv[16];
#pragma unroll
        for (int r = 0; r < 8; ++r) av[r] = Arows[(8 * ty + r) * kLd + i];
#pragma unroll
        for (int c2 = 0; c2 < 16; ++c2) bv[c2] = X1[(tx + 8 * c2) * kLd + i];
#pragma unroll
        for (int r = 0; r < 8; ++r)
#pragma unroll
          for (int c2 = 0; c2 < 16; ++c2) acc[r][c2] = fmaf(av[r], bv[c2], acc[r][c2]);
      }
      float* dst = pass == 0 ? X0 : X2;
      if (pass == 1) __syncthreads();  // every thread is done reading Q out of X2
#pragma unroll
      for (int r = 0; r < 8; ++r)
#pragma unroll
        for (int c2 = 0; c2 < 16; ++c2) dst[(8 * ty + r) * kLd + tx + 8 * c2] = acc[r][c2];
    }
  }
  __syncthreads();
  // A (strictly lower part; the unit diagonal is implicit) and P, row t per
  // thread: A[t][s] = w_t G[t][s] (K K^T)[t][s], P[t][s] = G[t][s] (Q K^T)[t][s]
  if (tid < n) {
    float g = 1.f;  // G[t][s], s going down from t - 1
    for (int s2 = tid - 1; s2 >= 0; --s2) {
      X0[tid * kLd + s2] *= w[tid] * g;
      X2[tid * kLd + s2] *= g;
      g *= a[s2];
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
// Each chunk's M is first copied into shared memory with coalesced loads.
constexpr int kStateSmem = (kD * kLd + kD * kSlab) * int(sizeof(float));
__global__ void __launch_bounds__(kD) tok_state_kernel(TokenParams p) {
  extern __shared__ float st_sm[];
  float* Ms = st_sm;                                            // [kD][kLd]
  float(*Ss)[kSlab] = reinterpret_cast<float(*)[kSlab]>(st_sm + kD * kLd);  // [kD][kSlab]
  const int slab = blockIdx.x % (kD / kSlab), bh = blockIdx.x / (kD / kSlab);
  const int i = threadIdx.x, j0 = slab * kSlab;
  for (int jj = 0; jj < kSlab; ++jj) Ss[i][jj] = p.s_in[(size_t(bh) * kD + i) * kD + j0 + jj];
  for (int c = 0; c < p.n_chunks; ++c) {
    const size_t mn0 = (size_t(bh) * p.n_chunks + c) * kD * kD;
    for (int x = i; x < kD * kD; x += kD) Ms[(x / kD) * kLd + x % kD] = p.m[mn0 + x];
    __syncthreads();  // M in; the previous step's state rows are all written
    float acc[kSlab];
    for (int jj = 0; jj < kSlab; ++jj) {
      p.s_chunk[mn0 + size_t(i) * kD + j0 + jj] = Ss[i][jj];
      acc[jj] = p.n[mn0 + size_t(i) * kD + j0 + jj];
    }
    const float* mrow = Ms + i * kLd;
    for (int k = 0; k < kD; ++k) {
      const float mv = mrow[k];
#pragma unroll
      for (int jj = 0; jj < kSlab; ++jj) acc[jj] = fmaf(mv, Ss[k][jj], acc[jj]);
    }
    __syncthreads();  // every row of the entering state is read
#pragma unroll
    for (int jj = 0; jj < kSlab; ++jj) Ss[i][jj] = acc[jj];
  }
  __syncthreads();
  if (p.s_out)
    for (int jj = 0; jj < kSlab; ++jj) p.s_out[(size_t(bh) * kD + i) * kD + j0 + jj] = Ss[i][jj];
}

// (4) One block per (stream, head, chunk), thread j = channel j:
// o_t += Qt_t S_c + Ot_t on top of the intra-frame output already in o.  The
// chunk's entering state and its Qt rows are first copied into shared memory.
constexpr int kOutSmem = (kD * kD + kChunk * kLd) * int(sizeof(float));
__global__ void __launch_bounds__(kD) tok_out_kernel(TokenParams p) {
  extern __shared__ float Sc[];  // [kD][kD], the state entering the chunk; then Qt [kChunk][kLd]
  float* Qs = Sc + kD * kD;
  const int c = blockIdx.x % p.n_chunks, bh = blockIdx.x / p.n_chunks;
  const int b = bh / p.H, h = bh % p.H;
  const int t0 = c * kChunk, n = min(kChunk, p.L - t0);
  const int j = threadIdx.x;
  const size_t mn0 = (size_t(bh) * p.n_chunks + c) * kD * kD;
  const size_t tok0 = size_t(bh) * p.L + t0;
  for (int i = 0; i < kD; ++i) Sc[i * kD + j] = p.s_chunk[mn0 + size_t(i) * kD + j];
  for (int x = j; x < n * kD; x += kD) Qs[(x / kD) * kLd + x % kD] = p.qt[tok0 * kD + x];
  __syncthreads();
  for (int t = 0; t < n; ++t) {
    const float* qrow = Qs + t * kLd;
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
  static unsigned done_chunk = 0, done_out = 0, done_maps = 0;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(tok_maps_kernel), kMapsSmem, &done_maps);
  if (e != cudaSuccess) return e;
  e = ensure_smem_attr(reinterpret_cast<const void*>(tok_chunk_kernel), int(kChunkSmem), &done_chunk);
  if (e != cudaSuccess) return e;
  e = ensure_smem_attr(reinterpret_cast<const void*>(tok_out_kernel), kOutSmem, &done_out);
  if (e != cudaSuccess) return e;
  static unsigned done_state = 0;
  e = ensure_smem_attr(reinterpret_cast<const void*>(tok_state_kernel), kStateSmem, &done_state);
  if (e != cudaSuccess) return e;
  const unsigned bh = unsigned(p.B) * unsigned(p.H);
  tok_maps_kernel<<<bh * unsigned(p.n_chunks), kD, kMapsSmem, st>>>(p);
  tok_chunk_kernel<<<bh * unsigned(p.n_chunks), kChunk, kChunkSmem, st>>>(p);
  tok_state_kernel<<<bh * unsigned(kD / kSlab), kD, kStateSmem, st>>>(p);
  if (with_out) tok_out_kernel<<<bh * unsigned(p.n_chunks), kD, kOutSmem, st>>>(p);
  return cudaGetLastError();
}

}  // namespace arl2
