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
// whose operands need no state.  So: (1) the maps per token (tcgen05); (2)
// one CTA per (stream, head, chunk) builds M, N, Qt, Ot (tcgen05 products,
// A^-1 in f32 on the CUDA cores); (3) one block per (stream, head, 16-column
// slab of S) runs S_next = M S + N over the chunks in order (f32); (4) one
// block per (stream, head, chunk) adds Qt S + Ot to the intra-frame output
// (f32, register-tiled).

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

__device__ __forceinline__ float bf(const __nv_bfloat16 x) { return __bfloat162float(x); }

// acc[r][c] = sum over s < ns of A(8 ty + r, s) B(s, tx + 8 c) for thread
// (ty, tx) = (tid / 8, tid % 8) of 128: a 128 x 128 product tiled 8 x 16 per
// thread (operands read through the accessors, from shared memory).
template <class FA, class FB>
__device__ __forceinline__ void tile_product(float (&acc)[8][16], int ns, FA fa, FB fb) {
  const int ty = threadIdx.x >> 3, tx = threadIdx.x & 7;
#pragma unroll
  for (int r = 0; r < 8; ++r)
#pragma unroll
    for (int c = 0; c < 16; ++c) acc[r][c] = 0.f;
#pragma unroll 2
  for (int s = 0; s < ns; ++s) {
    float av[8], bv[16];
#pragma unroll
    for (int r = 0; r < 8; ++r) av[r] = fa(8 * ty + r, s);
#pragma unroll
    for (int c = 0; c < 16; ++c) bv[c] = fb(s, tx + 8 * c);
#pragma unroll
    for (int r = 0; r < 8; ++r)
#pragma unroll
      for (int c = 0; c < 16; ++c) acc[r][c] = fmaf(av[r], bv[c], acc[r][c]);
  }
}

// Copy rows [0, n) of a row-major [rows][128] f32 matrix into shared memory
// with row pitch `ld` floats (rows n .. 127 zero when zero_tail), NT threads
// (128 or 256), eight 16-byte loads in flight per thread.
template <int NT = 128>
__device__ __forceinline__ void stage_rows(float* dst, int ld, const float* src, int n, bool zero_tail) {
  const int tid = threadIdx.x;
#pragma unroll 1
  for (int base = 0; base < 4096; base += 8 * NT) {  // 128 rows x 32 float4
    float4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int x = base + u * NT + tid, r = x >> 5;
      v[u] = r < n ? reinterpret_cast<const float4*>(src)[x] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int x = base + u * NT + tid, r = x >> 5, c4 = x & 31;
      if (r < n || zero_tail) {
        float* d = dst + r * ld + c4 * 4;
        d[0] = v[u].x;
        d[1] = v[u].y;
        d[2] = v[u].z;
        d[3] = v[u].w;
      }
    }
  }
}

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
  if (!ARL2_IN_BOUNDS(p.err, bh < p.B * p.H && t0 < p.L)) return;  // (debug build) before any barrier
  if (tid == 0) {
    mbar_init(bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc(tmem_holder, 512);
#pragma unroll 1
  for (int base = 0; base < 3 * 2048; base += 8 * kD) {  // 16-byte chunks: tile x >> 11, row (x >> 4) & 127, chunk x & 15
    uint4 v[8], f[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int x = base + u * kD + tid, m = x >> 11, r = (x >> 4) & 127, cc = x & 15;
      const __nv_bfloat16* xsrc = m == 0 ? p.q : (m == 1 ? p.k : p.v);
      const __nv_bfloat16* fsrc = m == 0 ? p.phi_q : (m == 1 ? p.phi_k_t : p.phi_v_t);
      v[u] = r < n ? *reinterpret_cast<const uint4*>(xsrc + ((size_t(b) * p.L + t0 + r) * p.H + h) * kD + cc * 8)
                   : make_uint4(0u, 0u, 0u, 0u);
      f[u] = *reinterpret_cast<const uint4*>(fsrc + (size_t(h) * kD + r) * kD + cc * 8);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int x = base + u * kD + tid, m = x >> 11, r = (x >> 4) & 127, cc = x & 15;
      *reinterpret_cast<uint4*>(sX + m * kMapTile + tok_sw128(r, cc * 8)) = v[u];
      *reinterpret_cast<uint4*>(sF + m * kMapTile + tok_sw128(r, cc * 8)) = f[u];
    }
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
#pragma unroll 1
    for (int m = 0; m < 3; ++m) {
      float* dst_m = m == 0 ? p.qp : (m == 1 ? p.kp : p.vp);
#pragma unroll 1
      for (int q = 0; q < 4; ++q) {
        uint32_t r[32];
        tmem_ld32(tmem + m * 128 + lane_off + q * 32, r);
        tmem_wait_ld();
        if (tid < n) {
          const float sc = m == 1 ? inv : 1.f;
          float4* d4 = reinterpret_cast<float4*>(dst_m + out + q * 32);
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

// (2) The chunk's maps on tcgen05: one CTA per (stream, head, chunk), 128 threads
// (thread t = token t, or state row t).  bf16 operands in shared memory (the
// 128-byte-swizzle tiles the tensor cores read), f32 accumulation in tensor
// memory; A^-1 by forward substitution in f32 on the CUDA cores.  Products:
//   K K^T, Q K^T                  -> A (f32), P = G * (Q K^T) (bf16)
//   W = T1 K,  U' = T2 V          T1 = T diag(w g_prev), T2 = T diag(w)
//   M' = K^T Wt, N = K^T Ut       Wt = diag(g_tail) W, Ut = diag(g_tail) U'
//   Qt' = P W, Ot = P U'          M = g_C I - M', Qt = diag(g_prev) Q - Qt'
// (bf16 operands keep the outputs within 6e-3 and the state within 4e-3 of
// the f64 recurrence on the 1560-token frame, CPU emulation.)
constexpr uint32_t kTcTile = 32768, kTcHalf = 16384;
constexpr uint32_t kTcF32 = 66560;  // one f32 128 x 129 matrix, rounded up to 1 KB
constexpr int kTcSmem = int(2 * kTcTile + 2 * kTcF32) + 3 * kChunk * 4 + 64 + 1024;

// Row `row` of a bf16 tile from 128 f32 values (16-byte chunks, swizzled).
__device__ __forceinline__ void tile_row_bf16(uint8_t* tile, int row, const float (&v)[128]) {
#pragma unroll
  for (int c = 0; c < 16; ++c)
    *reinterpret_cast<uint4*>(tile + tok_sw128(row, 8 * c)) =
        make_uint4(pack_bf16x2(v[8 * c], v[8 * c + 1]), pack_bf16x2(v[8 * c + 2], v[8 * c + 3]),
                   pack_bf16x2(v[8 * c + 4], v[8 * c + 5]), pack_bf16x2(v[8 * c + 6], v[8 * c + 7]));
}

// Rows [0, n) of a row-major [rows][128] f32 matrix into a bf16 tile (rows
// past n zero), 128 threads.
__device__ __forceinline__ void tile_from_f32(uint8_t* tile, const float* src, int n) {
#pragma unroll 4
  for (int x = threadIdx.x; x < 2048; x += kD) {
    const int r = x >> 4, cc = x & 15;
    float4 a4 = make_float4(0.f, 0.f, 0.f, 0.f), b4 = a4;
    if (r < n) {
      a4 = reinterpret_cast<const float4*>(src + r * kD + cc * 8)[0];
      b4 = reinterpret_cast<const float4*>(src + r * kD + cc * 8)[1];
    }
    *reinterpret_cast<uint4*>(tile + tok_sw128(r, cc * 8)) =
        make_uint4(pack_bf16x2(a4.x, a4.y), pack_bf16x2(a4.z, a4.w), pack_bf16x2(b4.x, b4.y), pack_bf16x2(b4.z, b4.w));
  }
}

// 128 x 128 x 128 product into tensor memory: A and B by their descriptors'
// layouts (K-major: 64-column boxes, K steps of 32 bytes; MN-major: K steps of
// 2048 bytes, boxes kTcHalf apart).
__device__ __forceinline__ void mma_tile(uint32_t d, uint32_t a, bool a_mn, uint32_t b, bool b_mn) {
  const uint32_t id = idesc_bf16(128, 128, a_mn ? 1 : 0, b_mn ? 1 : 0);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const uint32_t koff = (kk >> 2) * kTcHalf + (kk & 3) * 32, moff = kk * 2048;
    mma_ss(d, a_mn ? smem_desc_sw128(a + moff, kTcHalf, 1024) : smem_desc_sw128(a + koff, 16, 1024),
           b_mn ? smem_desc_sw128(b + moff, kTcHalf, 1024) : smem_desc_sw128(b + koff, 16, 1024), id, kk > 0);
  }
}

__device__ __forceinline__ void tmem_row128(uint32_t taddr, float (&v)[128]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) tmem_ld32(taddr + q * 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32 * q]));
  tmem_wait_ld();
}

__global__ void __launch_bounds__(kD, 1) tok_chunk_tc_kernel(TokenParams p) {
  extern __shared__ uint8_t tc_smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(tc_smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* tK = sm;                       // K' [t][d] (bf16)
  uint8_t* tP = sm + kTcTile;             // Q' [t][d], then P [t][s]
  uint8_t* R0 = sm + 2 * kTcTile;         // A (f32), then T1, T2; then Wt, W (bf16 tiles)
  uint8_t* R1 = R0 + kTcF32;              // G, then T (f32); then V'; then Ut, U' (bf16 tiles)
  float* F0 = reinterpret_cast<float*>(R0);
  float* F1 = reinterpret_cast<float*>(R1);
  float* w = reinterpret_cast<float*>(R1 + kTcF32);  // c beta
  float* g_prev = w + kChunk;
  float* g_tail = g_prev + kChunk;
  uint64_t* bars = reinterpret_cast<uint64_t*>(g_tail + kChunk);  // [3] MMA phases
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 3);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  __shared__ float g_all;
  const int c = blockIdx.x % p.n_chunks, bh = blockIdx.x / p.n_chunks;
  const int t0 = c * kChunk, n = min(kChunk, p.L - t0);
  if (!ARL2_IN_BOUNDS(p.err, bh < p.B * p.H && t0 < p.L)) return;  // (debug build) before any barrier
  const int tid = threadIdx.x, warp = tid >> 5;
  const uint32_t lane_off = uint32_t(warp * 32) << 16;
  const size_t tok0 = size_t(bh) * p.L + t0;
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
    for (int s2 = n - 1; s2 >= 0; --s2) {
      g_tail[s2] = g;
      g *= a[s2];
    }
    for (int i = 0; i < 3; ++i) mbar_init(&bars[i], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc(tmem_holder, 512);
  tile_from_f32(tK, p.kp + tok0 * kD, n);
  tile_from_f32(tP, p.qp + tok0 * kD, n);
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const WaitCtl wc{abort_flag, p.err, p.wait_limit_ns};
  const uint32_t aK = smem_u32(tK), aP = smem_u32(tP), a0 = smem_u32(R0), a1 = smem_u32(R1);
  if (tid == 0) {  // K K^T and Q K^T
    mma_tile(tmem, aK, false, aK, false);
    mma_tile(tmem + 128, aP, false, aK, false);
    mma_commit(&bars[0]);
  }
  bool ok = __all_sync(0xffffffffu, mbar_wait(&bars[0], 0, wc));
  const int t = tid;
  if (ok) {
    tc_fence_after();
    // A[t][s] = w_t G[t][s] (K K^T)[t][s] (s < t) into F0, G[t][s] into F1
    float v[128];
    tmem_row128(tmem + lane_off, v);
    float g = 1.f;
    const float wt = t < n ? w[t] : 0.f;
#pragma unroll
    for (int s2 = kChunk - 1; s2 >= 0; --s2) {
      if (s2 < t && t < n) {
        F0[t * kLd + s2] = wt * g * v[s2];
        F1[t * kLd + s2] = g;
        g *= a[s2];
      }
    }
    // P[t][s] = G[t][s] (Q K^T)[t][s] (s < t), bf16 over Q' (read by the MMA)
    tmem_row128(tmem + 128 + lane_off, v);
#pragma unroll
    for (int s2 = 0; s2 < kChunk; ++s2) v[s2] = (s2 < t && t < n) ? v[s2] * F1[t * kLd + s2] : 0.f;
    tile_row_bf16(tP, t, v);
  }
  __syncthreads();
  // T = A^-1 (unit lower triangular) by forward substitution, column j per
  // thread, into F1; each dot product runs as four interleaved partial sums
  if (ok && tid < n) {
    const int j = tid;
    for (int i = 0; i < n; ++i) {
      float x0 = i == j ? 1.f : 0.f, x1 = 0.f, x2 = 0.f, x3 = 0.f;
      if (i > j) {
        const float* ai = F0 + i * kLd;
        int k = j;
        for (; k + 3 < i; k += 4) {
          x0 = fmaf(-ai[k], F1[k * kLd + j], x0);
          x1 = fmaf(-ai[k + 1], F1[(k + 1) * kLd + j], x1);
          x2 = fmaf(-ai[k + 2], F1[(k + 2) * kLd + j], x2);
          x3 = fmaf(-ai[k + 3], F1[(k + 3) * kLd + j], x3);
        }
        for (; k < i; ++k) x0 = fmaf(-ai[k], F1[k * kLd + j], x0);
      }
      F1[i * kLd + j] = (x0 + x1) + (x2 + x3);
    }
  }
  __syncthreads();
  // T1 = T diag(w g_prev), T2 = T diag(w) (rows t, columns s <= t < n) as bf16 tiles over A
  if (ok) {
    float v[128];
#pragma unroll
    for (int s2 = 0; s2 < kChunk; ++s2) v[s2] = (s2 <= t && t < n) ? F1[t * kLd + s2] * w[s2] * g_prev[s2] : 0.f;
    tile_row_bf16(R0, t, v);
#pragma unroll
    for (int s2 = 0; s2 < kChunk; ++s2) v[s2] = (s2 <= t && t < n) ? F1[t * kLd + s2] * w[s2] : 0.f;
    tile_row_bf16(R0 + kTcTile, t, v);
  }
  __syncthreads();  // T is read: V' into its place
  tile_from_f32(R1, p.vp + tok0 * kD, n);
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  if (ok && tid == 0) {  // W = T1 K', U' = T2 V' (K' and V' as MN-major B: rows s, columns d)
    tc_fence_after();
    mma_tile(tmem + 256, a0, false, aK, true);
    mma_tile(tmem + 384, a0 + kTcTile, false, a1, true);
    mma_commit(&bars[1]);
  }
  ok = ok && __all_sync(0xffffffffu, mbar_wait(&bars[1], 0, wc));
  if (ok) {  // row s of W and U': Wt, W over T1, T2; Ut, U' over V'
    tc_fence_after();
    const int s2 = tid;
    const float gt = s2 < n ? g_tail[s2] : 0.f;
    float v[128];
    tmem_row128(tmem + 256 + lane_off, v);
    tile_row_bf16(R0 + kTcTile, s2, v);
#pragma unroll
    for (int j = 0; j < kD; ++j) v[j] *= gt;
    tile_row_bf16(R0, s2, v);
    tmem_row128(tmem + 384 + lane_off, v);
    tile_row_bf16(R1 + kTcTile, s2, v);
#pragma unroll
    for (int j = 0; j < kD; ++j) v[j] *= gt;
    tile_row_bf16(R1, s2, v);
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  if (ok && tid == 0) {  // M' = K'^T Wt, N = K'^T Ut (K' as MN-major A), Qt' = P W, Ot = P U'
    tc_fence_after();
    mma_tile(tmem, aK, true, a0, true);
    mma_tile(tmem + 128, aK, true, a1, true);
    mma_tile(tmem + 256, aP, false, a0 + kTcTile, true);
    mma_tile(tmem + 384, aP, false, a1 + kTcTile, true);
    mma_commit(&bars[2]);
  }
  ok = ok && __all_sync(0xffffffffu, mbar_wait(&bars[2], 0, wc));
  if (ok) {
    tc_fence_after();
    const size_t mn0 = (size_t(bh) * p.n_chunks + c) * kD * kD;
    const int i = tid;
#pragma unroll 1
    for (int part = 0; part < 4; ++part) {
      float v[128];
      tmem_row128(tmem + part * 128 + lane_off, v);
      if (part == 0) {  // M, stored transposed (column i of M^T per thread: coalesced)
        float* dst = p.m + mn0 + i;
#pragma unroll
        for (int k = 0; k < kD; ++k) dst[size_t(k) * kD] = (i == k ? g_all : 0.f) - v[k];
      } else if (part == 1) {  // N (row i)
        float* dst = p.n + mn0 + size_t(i) * kD;
#pragma unroll
        for (int j4 = 0; j4 < 32; ++j4)
          reinterpret_cast<float4*>(dst)[j4] = make_float4(v[4 * j4], v[4 * j4 + 1], v[4 * j4 + 2], v[4 * j4 + 3]);
      } else if (t < n) {  // Qt (row t), Ot (row t)
        float* dst = (part == 2 ? p.qt : p.ot) + (tok0 + t) * kD;
        const float* q = p.qp + (tok0 + t) * kD;
        const float gp = g_prev[t];
#pragma unroll
        for (int j4 = 0; j4 < 32; ++j4) {
          float4 o = make_float4(v[4 * j4], v[4 * j4 + 1], v[4 * j4 + 2], v[4 * j4 + 3]);
          if (part == 2) {
            const float4 q4 = reinterpret_cast<const float4*>(q)[j4];
            o = make_float4(gp * q4.x - o.x, gp * q4.y - o.y, gp * q4.z - o.z, gp * q4.w - o.w);
          }
          reinterpret_cast<float4*>(dst)[j4] = o;
        }
      }
    }
  } else if (tid == 0) {  // MMAs in flight land before tensor memory is released
    mma_commit(&bars[2]);
    const uint64_t t_0 = global_timer_ns();
    while (!mbar_try_wait(&bars[2], 0) && !mbar_try_wait(&bars[2], 1) && global_timer_ns() - t_0 < 10000000ull) {
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// (3) One block per (stream, head, 16-column slab of S), thread i = row i:
// S_next = M S + N over the chunks in order; the state entering each chunk is
// kept for (4), and the final one goes to s_out (a commit) or nowhere (a query).
// Each chunk's M is copied into one of two shared-memory buffers with
// asynchronous copies issued a chunk ahead, so the copy of chunk c + 1 runs
// while chunk c computes.
constexpr int kStateSmem = (2 * kD * kD + kD * kSlab) * int(sizeof(float));

// M^T of a chunk ([128][128] f32, row k = column k of M) into shared memory
// with 16-byte asynchronous copies.
__device__ __forceinline__ void copy_async_m(float* dst, const float* src) {
  const int tid = threadIdx.x;
#pragma unroll 8
  for (int x = tid; x < kD * kD / 4; x += kD) {
    const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst + 4 * x));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src + 4 * x) : "memory");
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
}

__global__ void __launch_bounds__(kD) tok_state_kernel(TokenParams p) {
  extern __shared__ float st_sm[];
  float* Mbuf = st_sm;                                                             // [2][kD][kD]: M^T
  float(*Ss)[kSlab] = reinterpret_cast<float(*)[kSlab]>(st_sm + 2 * kD * kD);  // [kD][kSlab]
  const int slab = blockIdx.x % (kD / kSlab), bh = blockIdx.x / (kD / kSlab);
  const int i = threadIdx.x, j0 = slab * kSlab;
  if (!ARL2_IN_BOUNDS(p.err, bh < p.B * p.H)) return;  // (debug build)
  for (int jj = 0; jj < kSlab; ++jj) Ss[i][jj] = p.s_in[(size_t(bh) * kD + i) * kD + j0 + jj];
  copy_async_m(Mbuf, p.m + size_t(bh) * p.n_chunks * kD * kD);
  for (int c = 0; c < p.n_chunks; ++c) {
    const size_t mn0 = (size_t(bh) * p.n_chunks + c) * kD * kD;
    float acc[kSlab];
#pragma unroll
    for (int jj = 0; jj < kSlab; ++jj) acc[jj] = p.n[mn0 + size_t(i) * kD + j0 + jj];
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncthreads();  // M(c) in; the previous step's state rows are all written
    if (c + 1 < p.n_chunks) copy_async_m(Mbuf + ((c + 1) & 1) * kD * kD, p.m + mn0 + kD * kD);
#pragma unroll
    for (int jj = 0; jj < kSlab; ++jj) p.s_chunk[mn0 + size_t(i) * kD + j0 + jj] = Ss[i][jj];
    const float* mcol = Mbuf + (c & 1) * kD * kD + i;  // M[i][k] = M^T[k][i]: conflict-free across threads
#pragma unroll 4
    for (int k = 0; k < kD; ++k) {
      const float mv = mcol[k * kD];
      const float4* sk = reinterpret_cast<const float4*>(Ss[k]);  // row k of the slab: 4 broadcast loads
#pragma unroll
      for (int q = 0; q < kSlab / 4; ++q) {
        const float4 s4 = sk[q];
        acc[4 * q] = fmaf(mv, s4.x, acc[4 * q]);
        acc[4 * q + 1] = fmaf(mv, s4.y, acc[4 * q + 1]);
        acc[4 * q + 2] = fmaf(mv, s4.z, acc[4 * q + 2]);
        acc[4 * q + 3] = fmaf(mv, s4.w, acc[4 * q + 3]);
      }
    }
    __syncthreads();  // every row of the entering state and of M(c) is read
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
  if (!ARL2_IN_BOUNDS(p.err, bh < p.B * p.H && t0 < p.L)) return;  // (debug build)
  const size_t mn0 = (size_t(bh) * p.n_chunks + c) * kD * kD;
  const size_t tok0 = size_t(bh) * p.L + t0;
  stage_rows(Sc, kD, p.s_chunk + mn0, kD, true);
  stage_rows(Qs, kLd, p.qt + tok0 * kD, n, true);
  __syncthreads();
  // Qt S_c as a register-tiled product (thread (ty, tx): tokens 8 ty + r,
  // channels tx + 8 c), then o += it + Ot with every load of the tile in flight
  float acc[8][16];
  tile_product(acc, kD, [&](int t, int i) { return Qs[t * kLd + i]; }, [&](int i, int jj) { return Sc[i * kD + jj]; });
  const int ty = j >> 3, tx = j & 7;
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    const int t = 8 * ty + r;
    if (t < n) {
      float ot[16];
      __nv_bfloat16 ov[16];
      const size_t o0 = ((size_t(b) * p.L + t0 + t) * p.H + h) * kD;
#pragma unroll
      for (int c2 = 0; c2 < 16; ++c2) {
        ot[c2] = p.ot[(tok0 + t) * kD + tx + 8 * c2];
        ov[c2] = p.o[o0 + tx + 8 * c2];
      }
#pragma unroll
      for (int c2 = 0; c2 < 16; ++c2) p.o[o0 + tx + 8 * c2] = __float2bfloat16_rn(bf(ov[c2]) + acc[r][c2] + ot[c2]);
    }
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
  e = ensure_smem_attr(reinterpret_cast<const void*>(tok_chunk_tc_kernel), kTcSmem, &done_chunk);
  if (e != cudaSuccess) return e;
  e = ensure_smem_attr(reinterpret_cast<const void*>(tok_out_kernel), kOutSmem, &done_out);
  if (e != cudaSuccess) return e;
  static unsigned done_state = 0;
  e = ensure_smem_attr(reinterpret_cast<const void*>(tok_state_kernel), kStateSmem, &done_state);
  if (e != cudaSuccess) return e;
  const unsigned bh = unsigned(p.B) * unsigned(p.H);
  tok_maps_kernel<<<bh * unsigned(p.n_chunks), kD, kMapsSmem, st>>>(p);
  tok_chunk_tc_kernel<<<bh * unsigned(p.n_chunks), kD, kTcSmem, st>>>(p);
  tok_state_kernel<<<bh * unsigned(kD / kSlab), kD, kStateSmem, st>>>(p);
  if (with_out) tok_out_kernel<<<bh * unsigned(p.n_chunks), kD, kOutSmem, st>>>(p);
  return cudaGetLastError();
}

}  // namespace arl2
