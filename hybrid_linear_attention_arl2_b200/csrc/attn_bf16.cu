// Intra-frame softmax attention with the inter-frame read-out fused into its
// epilogue, bf16 operands, fp32 accumulation in tensor memory (sm_100a).
//
//   O = softmax(Q K^T * scale) V  +  Q MqT^T        (MqT = (phi_q S_{N-1})^T)
//
// The first term is the intra-frame branch (ARL2 summary, section 2.1: the
// original bidirectional softmax attention within each frame).  The second is
// the inter-frame read-out O_inter = Q' S_{N-1} = (Q phi_q) S_{N-1}, computed
// as Q (phi_q S_{N-1}): the product phi_q S is formed once per state write, so
// a pass costs one extra 128 x 128 x 128 MMA per query tile.
//
// One CTA = 128 query rows of one (stream, head).  Warp roles:
//   warp 0      TMA producer: Q once, then K_j and V_j per key tile, then MqT;
//   warp 1      tcgen05 issuer: S = Q K_j^T, O += P V_j, X = Q MqT^T;
//   warps 2..5  softmax + epilogue, one query row per thread (TMEM lane).
// Tensor memory (256 columns): [0,128) S_j fp32, overwritten in place by
// P_j (bf16 pairs, columns [0,64)) and finally by X; [128,256) the O
// accumulator.  Two CTAs fit on an SM (99.5 KB shared memory, 256 TMEM
// columns each), so one CTA's softmax overlaps the other's MMAs.
//
// The same kernel without the read-out serves the softmax layers that keep a
// growing KV cache (the K/V tensor maps then cover the cache).

#include "params.h"
#include "sm100.cuh"

namespace arl2 {

constexpr int kAttnThreads = 192;
constexpr uint32_t kTile = 32768;  // 128 rows x 128 bf16
constexpr uint32_t kHalf = 16384;  // one 64-column box
constexpr int kAttnSmem = 3 * kTile + 256 + 1024;

enum { B_Q, B_KF, B_KE, B_VF, B_VE, B_SF, B_PF, B_OF, B_MQ, B_XF, B_DRAIN, B_COUNT };

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const WaitCtl& w) {
  bool ok = mbar_wait(bar, parity, w);
  return __all_sync(0xffffffffu, ok);
}

__global__ void __launch_bounds__(kAttnThreads, 2)
attn_bf16_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_mq,
                 const AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = smem + kTile;  // also MqT after the last S MMA
  uint8_t* sV = smem + 2 * kTile;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 3 * kTile);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + B_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int nkv = (p.kv_len + 127) >> 7;

  if (threadIdx.x == 0) {
    for (int i = 0; i < B_COUNT; ++i) mbar_init(&bars[i], i == B_PF ? 4u : 1u);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_holder, 256);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t tS = tmem, tO = tmem + 128;
  const WaitCtl w{abort_flag, p.err, p.wait_limit_ns};

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------------- producer
      tma_prefetch(&tm_q);
      tma_prefetch(&tm_k);
      tma_prefetch(&tm_v);
      const int x0 = h * 128;
      mbar_expect_tx(&bars[B_Q], kTile);
      tma_load_3d(sQ, &tm_q, &bars[B_Q], x0, qt * 128, b);
      tma_load_3d(sQ + kHalf, &tm_q, &bars[B_Q], x0 + 64, qt * 128, b);
      bool ok = true;
      for (int j = 0; j < nkv; ++j) {
        if (j > 0 && !(ok = mbar_wait(&bars[B_KE], (j - 1) & 1, w))) break;
        mbar_expect_tx(&bars[B_KF], kTile);
        tma_load_3d(sK, &tm_k, &bars[B_KF], x0, j * 128, b);
        tma_load_3d(sK + kHalf, &tm_k, &bars[B_KF], x0 + 64, j * 128, b);
        if (j > 0 && !(ok = mbar_wait(&bars[B_VE], (j - 1) & 1, w))) break;
        mbar_expect_tx(&bars[B_VF], kTile);
        tma_load_3d(sV, &tm_v, &bars[B_VF], x0, j * 128, b);
        tma_load_3d(sV + kHalf, &tm_v, &bars[B_VF], x0 + 64, j * 128, b);
      }
      if (ok && p.has_inter && mbar_wait(&bars[B_KE], (nkv - 1) & 1, w)) {
        mbar_expect_tx(&bars[B_MQ], kTile);
        const int slab = b * p.heads + h;
        tma_load_3d(sK, &tm_mq, &bars[B_MQ], 0, 0, slab);
        tma_load_3d(sK + kHalf, &tm_mq, &bars[B_MQ], 64, 0, slab);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------------------- MMA issuer
      const uint32_t qa = smem_u32(sQ), ka = smem_u32(sK), va = smem_u32(sV);
      const uint32_t id_o = idesc_bf16(128, 128, 0, 1);  // P (TMEM) x V (MN-major)
      bool ok = mbar_wait(&bars[B_Q], 0, w);
      for (int j = 0; ok && j < nkv; ++j) {
        const int valid = min(128, p.kv_len - j * 128);
        const int ns = min(128, (valid + 15) & ~15);
        if (!(ok = mbar_wait(&bars[B_KF], j & 1, w))) break;
        if (j > 0 && !(ok = mbar_wait(&bars[B_OF], (j - 1) & 1, w))) break;
        tc_fence_after();
        const uint32_t id_s = idesc_bf16(128, ns, 0, 0);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
          mma_ss(tS, smem_desc_sw128(qa + off, 16, 1024), smem_desc_sw128(ka + off, 16, 1024), id_s, kk > 0);
        }
        mma_commit(&bars[B_SF]);
        mma_commit(&bars[B_KE]);
        if (!(ok = mbar_wait(&bars[B_PF], j & 1, w))) break;
        if (!(ok = mbar_wait(&bars[B_VF], j & 1, w))) break;
        tc_fence_after();
        const int nk = (valid + 15) >> 4;
        for (int kk = 0; kk < nk; ++kk)
          mma_ts(tO, tS + kk * 8, smem_desc_sw128(va + kk * 2048, kHalf, 1024), id_o, (j > 0 || kk > 0));
        mma_commit(&bars[B_OF]);
        mma_commit(&bars[B_VE]);
      }
      if (ok && p.has_inter && mbar_wait(&bars[B_OF], (nkv - 1) & 1, w) && mbar_wait(&bars[B_MQ], 0, w)) {
        tc_fence_after();
        const uint32_t id_x = idesc_bf16(128, 128, 0, 0);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
          mma_ss(tS, smem_desc_sw128(qa + off, 16, 1024), smem_desc_sw128(ka + off, 16, 1024), id_x, kk > 0);
        }
        mma_commit(&bars[B_XF]);
      }
    }
  } else {
    // ------------------------------------------------------------------ softmax + epilogue
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = uint32_t(quarter * 32) << 16;
    const float sl2 = p.scale_log2;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      if (!(ok = warp_wait(&bars[B_SF], j & 1, w))) break;
      tc_fence_after();
      const int valid = min(128, p.kv_len - j * 128);
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(tS + lane_off + c * 32, r);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (c * 32 + i < valid) mx = fmaxf(mx, __uint_as_float(r[i]));
      }
      mx *= sl2;
      // Lazy rescaling: the running max moves only when it grows by more than
      // 2^8, so P stays <= 256 and the O accumulator is touched rarely.
      if (j == 0) {
        m = mx;
      } else {
        const bool need = mx > m + 8.f;
        if (__any_sync(0xffffffffu, need)) {
          const float f = need ? fast_exp2(m - mx) : 1.f;
          if (need) m = mx;
          l *= f;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t r[32];
            tmem_ld32(tO + lane_off + c * 32, r);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * f);
            tmem_st32(tO + lane_off + c * 32, r);
          }
          tmem_wait_st();
        }
      }
      const float nm = -m;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(tS + lane_off + c * 32, r);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int col = c * 32 + 2 * i;
          const float p0 = col < valid ? fast_exp2(fmaf(__uint_as_float(r[2 * i]), sl2, nm)) : 0.f;
          const float p1 = col + 1 < valid ? fast_exp2(fmaf(__uint_as_float(r[2 * i + 1]), sl2, nm)) : 0.f;
          l += p0 + p1;
          pk[i] = pack_bf16x2(p0, p1);
        }
        tmem_st16(tS + lane_off + c * 16, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[B_PF]);
    }
    if (ok) ok = warp_wait(&bars[B_OF], (nkv - 1) & 1, w);
    if (ok && p.has_inter) ok = warp_wait(&bars[B_XF], 0, w);
    if (ok) {
      tc_fence_after();
      const float inv_l = 1.f / l;
      const bool use_intra = !(p.flags & 2u);
      const bool use_inter = p.has_inter && !(p.flags & 1u);
      const int q_row = qt * 128 + row;
      __nv_bfloat16* dst = p.o + ((size_t(b) * p.q_len + q_row) * p.heads + h) * 128;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t ro[32], rx[32];
        tmem_ld32(tO + lane_off + c * 32, ro);
        if (p.has_inter) tmem_ld32(tS + lane_off + c * 32, rx);
        tmem_wait_ld();
        uint32_t packed[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float v0 = use_intra ? __uint_as_float(ro[2 * i]) * inv_l : 0.f;
          float v1 = use_intra ? __uint_as_float(ro[2 * i + 1]) * inv_l : 0.f;
          if (use_inter) {
            v0 += __uint_as_float(rx[2 * i]);
            v1 += __uint_as_float(rx[2 * i + 1]);
          }
          packed[i] = pack_bf16x2(v0, v1);
        }
        if (q_row < p.q_len) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            d4[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
        }
      }
    }
  }

  // ------------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    // A wait ran out: let this CTA's own asynchronous work land before the
    // shared and tensor memory are released.
    if (warp == 1 && lane == 0) {
      mma_commit(&bars[B_DRAIN]);
      WaitCtl drain{abort_flag, nullptr, 10000000ull};
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(&bars[B_DRAIN], 0) && global_timer_ns() - t0 < drain.limit_ns) {
      }
    }
    if (warp == 0 && lane == 0) {
      const uint64_t t0 = global_timer_ns();
      while (global_timer_ns() - t0 < 2000000ull) {
      }
    }
    __syncthreads();
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

cudaError_t launch_attn_bf16(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             const CUtensorMap& tmq, const AttnParams& p, int batch, cudaStream_t stream) {
  static unsigned done = 0;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(attn_bf16_kernel), kAttnSmem, &done);
  if (e != cudaSuccess) return e;
  dim3 grid((p.q_len + 127) / 128, p.heads, batch);
  attn_bf16_kernel<<<grid, kAttnThreads, kAttnSmem, stream>>>(tq, tk, tv, tmq, p);
  return cudaGetLastError();
}

}  // namespace arl2
