// The frame's state write on the clean pass, bf16 operands, fp32 state (sm_100a):
//
//   S_N = alpha S_{N-1} + c K'^T diag(beta) (V' - K' S_{N-1})
//
// with K' = rownorm2(K phi_k) and V' = V phi_v (ARL2 summary, section 2.1,
// feature maps and state update; section 2.2, one write per frame from the
// pre-update state).  Three kernels:
//
//  state_partial_kernel   one CTA per 128-token chunk of one (stream, head):
//                         K~ = K phi_k and V~ = V phi_v (tcgen05), K' by row
//                         normalisation, R = diag(beta)(V~ - K' S_{N-1}),
//                         partial delta = K'^T R (tcgen05), stored fp32;
//  state_finalize_kernel  sums the chunks' partials in fixed chunk order
//                         (deterministic, no float atomics), applies the decay,
//                         writes S_N (fp32) and its bf16 copy;
//  readout_prep_kernel    MqT = (phi_q S_N)^T in bf16, the operand the next
//                         frame's passes use for O_inter = Q' S_N (tcgen05).
//
// Shared-memory tiles use the 128-byte-swizzle layout of a TMA box with 64
// bf16 columns; tiles written by threads (K', R) are stored in that same
// layout so that the tensor cores can read them with the same descriptors.

#include "params.h"
#include "sm100.cuh"

namespace arl2 {

constexpr uint32_t kTileB = 32768;
constexpr uint32_t kHalfB = 16384;
constexpr int kStateThreads = 192;
// Three 32 KB tiles (K then K'; V then S_{N-1}; phi_k^T then phi_v^T then R):
// two CTAs fit on an SM, so the 13 chunks x 12 heads of a 1560-token frame run
// in one wave on 148 SMs.
constexpr int kPartialSmem = 3 * kTileB + 256 + 1024;
constexpr int kPrepSmem = 2 * kTileB + 256 + 1024;

// Byte offset of bf16 element (row, col) of a 128-row tile stored as two
// 64-column boxes in the 128-byte-swizzle layout (16-byte chunks of a row
// XORed with row % 8).
__device__ __forceinline__ uint32_t sw128_offset(int row, int col) {
  const int box = col >> 6, cc = col & 63;
  const int chunk = (cc >> 3) ^ (row & 7);
  return uint32_t(box) * kHalfB + uint32_t(row) * 128 + uint32_t(chunk) * 16 + uint32_t(cc & 7) * 2;
}

__device__ __forceinline__ bool warp_wait_s(uint64_t* bar, uint32_t parity, const WaitCtl& w) {
  bool ok = mbar_wait(bar, parity, w);
  return __all_sync(0xffffffffu, ok);
}

enum { P_IN, P_MK, P_PV, P_MV, P_KP, P_S, P_KS, P_R, P_DS, P_PQ, P_MQ, P_DRAIN, P_COUNT };

__device__ __forceinline__ uint32_t cluster_rank_s() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_nrank_s() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ float4 ld_dsmem_f4(uint32_t cluster_addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(cluster_addr)
               : "memory");
  return v;
}
__device__ __forceinline__ void st_dsmem_v2(uint32_t cluster_addr, uint2 v) {
  asm volatile("st.shared::cluster.v2.b32 [%0], {%1, %2};" ::"r"(cluster_addr), "r"(v.x), "r"(v.y) : "memory");
}

// Float offset of 16-byte chunk c (columns 4c..4c+3) of row i of a chunk's
// fp32 partial held in shared memory for the cluster's reduction: chunks are
// XOR-swizzled by row so that a warp writing one chunk of 32 rows spreads over
// every bank.
__device__ __forceinline__ uint32_t part_off(int i, int c) { return uint32_t(i) * 128 + uint32_t((c ^ (i & 31)) << 2); }

// kFused = false: one CTA per 128-token chunk writes its partial delta to
// global memory (state_finalize_kernel then reduces).  kFused = true: the
// CTAs of one (stream, head) form a cluster, one per chunk; they reduce their
// partials through distributed shared memory in chunk order (the same sums,
// in the same order, as state_finalize_kernel), apply the decay, write S_N and
// its bf16 copy, and the cluster's rank 0 forms MqT = (phi_q S_N)^T: the whole
// state write in one launch, with no partial leaving the chip.
template <bool kFused>
__global__ void __launch_bounds__(kStateThreads, 2)
state_partial_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                     const __grid_constant__ CUtensorMap tm_phik_t, const __grid_constant__ CUtensorMap tm_phiv_t,
                     const __grid_constant__ CUtensorMap tm_s_bf, const __grid_constant__ CUtensorMap tm_phiq,
                     const StateParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = smem;               // K tile, then K' (bf16)
  uint8_t* sV = smem + kTileB;      // V tile, then S_{N-1} (bf16)
  uint8_t* sP = smem + 2 * kTileB;  // phi_k^T, then phi_v^T, then R (bf16)
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 3 * kTileB);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + P_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int chunk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int slab = b * p.heads + h;
  const int rank = kFused ? int(cluster_rank_s()) : 0;
  // (debug build) the launch is n_chunks x H x B; the test is the same for
  // every CTA of a cluster, so a whole cluster leaves before any barrier
  if (!ARL2_IN_BOUNDS(p.err, int(gridDim.x) == p.n_chunks && h < p.heads && b < p.batch)) return;

  if (threadIdx.x == 0) {
    for (int i = 0; i < P_COUNT; ++i) mbar_init(&bars[i], (i == P_KP || i == P_R) ? 4u : 1u);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_holder, 256);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t tA = tmem, tB = tmem + 128;  // [0,128): K~ then K'S ; [128,256): V~ then delta
  const WaitCtl w{abort_flag, p.err, p.wait_limit_ns};

  if (warp == 0) {
    if (lane == 0) {
      const int x0 = h * 128, t0 = chunk * 128;
      mbar_expect_tx(&bars[P_IN], 3 * kTileB);
      tma_load_3d(sK, &tm_k, &bars[P_IN], x0, t0, b);
      tma_load_3d(sK + kHalfB, &tm_k, &bars[P_IN], x0 + 64, t0, b);
      tma_load_3d(sV, &tm_v, &bars[P_IN], x0, t0, b);
      tma_load_3d(sV + kHalfB, &tm_v, &bars[P_IN], x0 + 64, t0, b);
      tma_load_3d(sP, &tm_phik_t, &bars[P_IN], 0, 0, h);
      tma_load_3d(sP + kHalfB, &tm_phik_t, &bars[P_IN], 64, 0, h);
      if (mbar_wait(&bars[P_MK], 0, w)) {  // phi_k^T read: phi_v^T in its place
        mbar_expect_tx(&bars[P_PV], kTileB);
        tma_load_3d(sP, &tm_phiv_t, &bars[P_PV], 0, 0, h);
        tma_load_3d(sP + kHalfB, &tm_phiv_t, &bars[P_PV], 64, 0, h);
        if (mbar_wait(&bars[P_MV], 0, w)) {  // V read: S_{N-1} in its place
          mbar_expect_tx(&bars[P_S], kTileB);
          tma_load_3d(sV, &tm_s_bf, &bars[P_S], 0, 0, slab);
          tma_load_3d(sV + kHalfB, &tm_s_bf, &bars[P_S], 64, 0, slab);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t ka = smem_u32(sK), va = smem_u32(sV), pa = smem_u32(sP);
      const uint32_t id_kk = idesc_bf16(128, 128, 0, 0);
      bool ok = mbar_wait(&bars[P_IN], 0, w);
      if (ok) {  // K~ = K phi_k
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * kHalfB + (kk & 3) * 32;
          mma_ss(tA, smem_desc_sw128(ka + off, 16, 1024), smem_desc_sw128(pa + off, 16, 1024), id_kk, kk > 0);
        }
        mma_commit(&bars[P_MK]);
      }
      if (ok && (ok = mbar_wait(&bars[P_PV], 0, w))) {  // V~ = V phi_v
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * kHalfB + (kk & 3) * 32;
          mma_ss(tB, smem_desc_sw128(va + off, 16, 1024), smem_desc_sw128(pa + off, 16, 1024), id_kk, kk > 0);
        }
        mma_commit(&bars[P_MV]);
      }
      // K'S: A = K' (K-major), B = S_{N-1} stored [i][j]: N = j contiguous -> MN-major.
      if (ok && (ok = mbar_wait(&bars[P_KP], 0, w)) && (ok = mbar_wait(&bars[P_S], 0, w))) {
        tc_fence_after();
        const uint32_t id_ks = idesc_bf16(128, 128, 0, 1);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t aoff = (kk >> 2) * kHalfB + (kk & 3) * 32;
          mma_ss(tA, smem_desc_sw128(ka + aoff, 16, 1024), smem_desc_sw128(va + kk * 2048, kHalfB, 1024), id_ks,
                 kk > 0);
        }
        mma_commit(&bars[P_KS]);
      }
      // delta = K'^T R: M = i, N = j, K = tokens; both operands MN-major.
      if (ok && (ok = mbar_wait(&bars[P_R], 0, w))) {
        tc_fence_after();
        const uint32_t id_d = idesc_bf16(128, 128, 1, 1);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(tB, smem_desc_sw128(ka + kk * 2048, kHalfB, 1024), smem_desc_sw128(pa + kk * 2048, kHalfB, 1024),
                 id_d, kk > 0);
        mma_commit(&bars[P_DS]);
      }
    }
  } else {
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;  // token within the chunk, then state row i
    const uint32_t lane_off = uint32_t(quarter * 32) << 16;
    const int token = chunk * 128 + row;
    const bool valid = token < p.L;
    bool ok = warp_wait_s(&bars[P_MK], 0, w);
    if (ok) {
      tc_fence_after();
      // K' = K~ / max(|K~|, 1e-12), written over the K tile (the K~ MMA has read it).
      float ss = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(tA + lane_off + c * 32, r);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float x = __uint_as_float(r[i]);
          ss = fmaf(x, x, ss);
        }
      }
      const float inv = 1.f / fmaxf(sqrtf(ss), 1e-12f);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(tA + lane_off + c * 32, r);
        tmem_wait_ld();
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          uint4 v;
          v.x = pack_bf16x2(__uint_as_float(r[8 * g + 0]) * inv, __uint_as_float(r[8 * g + 1]) * inv);
          v.y = pack_bf16x2(__uint_as_float(r[8 * g + 2]) * inv, __uint_as_float(r[8 * g + 3]) * inv);
          v.z = pack_bf16x2(__uint_as_float(r[8 * g + 4]) * inv, __uint_as_float(r[8 * g + 5]) * inv);
          v.w = pack_bf16x2(__uint_as_float(r[8 * g + 6]) * inv, __uint_as_float(r[8 * g + 7]) * inv);
          *reinterpret_cast<uint4*>(sK + sw128_offset(row, c * 32 + 8 * g)) = v;
        }
      }
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[P_KP]);
    }
    // R = beta (V~ - K'S), written over phi_v^T (the V~ MMA, complete with
    // the K'S one, has read it); zero for tokens past L.
    if (ok) ok = warp_wait_s(&bars[P_KS], 0, w);
    if (ok) {
      tc_fence_after();
      const float bt = valid ? p.beta[size_t(slab) * p.L + token] : 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t ks[32], vt[32];
        tmem_ld32(tA + lane_off + c * 32, ks);
        tmem_ld32(tB + lane_off + c * 32, vt);
        tmem_wait_ld();
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          float rr[8];
#pragma unroll
          for (int e = 0; e < 8; ++e)
            rr[e] = bt * (__uint_as_float(vt[8 * g + e]) - __uint_as_float(ks[8 * g + e]));
          uint4 v = make_uint4(pack_bf16x2(rr[0], rr[1]), pack_bf16x2(rr[2], rr[3]), pack_bf16x2(rr[4], rr[5]),
                               pack_bf16x2(rr[6], rr[7]));
          *reinterpret_cast<uint4*>(sP + sw128_offset(row, c * 32 + 8 * g)) = v;
        }
      }
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[P_R]);
    }
    // This chunk's delta rows (row = state row i): to global memory, or (fused)
    // to this CTA's shared memory for the cluster's reduction (the K and V
    // tiles are free once the last MMA has completed).
    if (ok) ok = warp_wait_s(&bars[P_DS], 0, w);
    if (ok) {
      tc_fence_after();
      float* dst = kFused ? reinterpret_cast<float*>(sK) : p.partial + ((size_t(slab) * p.n_chunks + chunk) * 128 + row) * 128;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(tB + lane_off + c * 32, r);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float4 v4 = make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                                        __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3]));
          if (kFused)
            *reinterpret_cast<float4*>(dst + part_off(row, c * 8 + i)) = v4;
          else
            reinterpret_cast<float4*>(dst + c * 32)[i] = v4;
        }
      }
    }
  }
  if (kFused) {
    // Every CTA of the cluster reaches these barriers, also after a timeout
    // (ok = false): the cluster's reduction is skipped then, not its barriers.
    __syncthreads();
    const int nrank = int(cluster_nrank_s());
    const bool ok_all = !*abort_flag;
    // rank 0: phi_q into the tile R occupied (the last MMA has read it)
    if (rank == 0 && warp == 0 && lane == 0 && ok_all) {
      mbar_expect_tx(&bars[P_PQ], kTileB);
      tma_load_3d(sP, &tm_phiq, &bars[P_PQ], 0, 0, h);
      tma_load_3d(sP + kHalfB, &tm_phiq, &bars[P_PQ], 64, 0, h);
    }
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
    // This rank's rows of S_N: sum the chunks' partials in chunk order (rank
    // q holds chunk q), then S_N = alpha S_{N-1} + c * sum.
    const int rpc = (128 + nrank - 1) / nrank;
    const int i0 = rank * rpc, i1 = min(128, i0 + rpc);
    const int nchunks16 = max(0, i1 - i0) * 32;  // 16-byte chunks of this rank's rows
    const uint32_t part_base = smem_u32(sK);
    const float a = p.alpha[slab];
    // Every rank's value of a chunk is loaded before any is added, so the
    // remote loads overlap, and the sum still runs in chunk order.  A thread's
    // first kMaxPer chunks (all of them from 9 ranks up) have their S_{N-1}
    // loaded while the other ranks finish their partials, and keep their bf16
    // values for the copy to rank 0; further ones are read from global memory.
    constexpr int kMaxPer = 3;
    uint2 keep[kMaxPer];
    float4 prev[kMaxPer];
#pragma unroll
    for (int t = 0; t < kMaxPer; ++t) {
      const int q16 = threadIdx.x + t * kStateThreads;
      prev[t] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (ok_all && q16 < nchunks16)
        prev[t] = *reinterpret_cast<const float4*>(p.S_prev + size_t(slab) * 16384 + size_t(i0 + q16 / 32) * 128 +
                                                   (q16 % 32) * 4);
    }
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
    for (int q16 = threadIdx.x, t = 0; ok_all && q16 < nchunks16; q16 += kStateThreads, ++t) {
      const int i = i0 + q16 / 32, c = q16 % 32;
      const uint32_t off = part_base + part_off(i, c) * 4;
      float4 v[16];
#pragma unroll
      for (int q = 0; q < 16; ++q)
        if (q < nrank) v[q] = ld_dsmem_f4(cluster_map(off, uint32_t(q)));
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        if (q < nrank) {
          acc.x += v[q].x;
          acc.y += v[q].y;
          acc.z += v[q].z;
          acc.w += v[q].w;
        }
      }
      const size_t e = size_t(slab) * 16384 + size_t(i) * 128 + c * 4;
      float4 sp4;
      if (t < kMaxPer) {
#pragma unroll
        for (int x = 0; x < kMaxPer; ++x)
          if (x == t) sp4 = prev[x];
      } else {
        sp4 = *reinterpret_cast<const float4*>(p.S_prev + e);
      }
      float4 r;
      r.x = fmaf(a, sp4.x, p.corr * acc.x);
      r.y = fmaf(a, sp4.y, p.corr * acc.y);
      r.z = fmaf(a, sp4.z, p.corr * acc.z);
      r.w = fmaf(a, sp4.w, p.corr * acc.w);
      *reinterpret_cast<float4*>(p.S_next + e) = r;
      const uint2 bf = make_uint2(pack_bf16x2(r.x, r.y), pack_bf16x2(r.z, r.w));
      *reinterpret_cast<uint2*>(p.S_next_bf + e) = bf;
#pragma unroll
      for (int x = 0; x < kMaxPer; ++x)
        if (x == t) keep[x] = bf;
    }
    // every partial is read: rank 0's K/V tiles take the bf16 S_N for the
    // read-out MMA (row k = state row, 64-column boxes, 128-byte swizzle: the
    // layout the tensor cores read as an MN-major operand); columns 4c..4c+3
    // of a row are 8 contiguous bytes of that layout
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
    for (int q16 = threadIdx.x, t = 0; ok_all && q16 < nchunks16; q16 += kStateThreads, ++t) {
      const int i = i0 + q16 / 32, c = q16 % 32;
      uint2 bf = make_uint2(0u, 0u);
      if (t < kMaxPer) {
#pragma unroll
        for (int x = 0; x < kMaxPer; ++x)
          if (x == t) bf = keep[x];
      } else {
        bf = *reinterpret_cast<const uint2*>(p.S_next_bf + size_t(slab) * 16384 + size_t(i) * 128 + c * 4);
      }
      st_dsmem_v2(cluster_map(smem_u32(sK) + sw128_offset(i, 4 * c), 0u), bf);
    }
    asm volatile("fence.proxy.async.shared::cluster;" ::: "memory");
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
    if (rank == 0 && ok_all) {
      // MqT[j][i] = sum_k S_N[k][j] phi_q[i][k]: M = j, N = i, K = k (as in readout_prep_kernel)
      if (warp == 1) {
        if (lane == 0 && mbar_wait(&bars[P_PQ], 0, w)) {
          tc_fence_after();
          const uint32_t sa = smem_u32(sK), pa = smem_u32(sP);
          const uint32_t id = idesc_bf16(128, 128, 1, 0);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t boff = (kk >> 2) * kHalfB + (kk & 3) * 32;
            mma_ss(tA, smem_desc_sw128(sa + kk * 2048, kHalfB, 1024), smem_desc_sw128(pa + boff, 16, 1024), id,
                   kk > 0);
          }
          mma_commit(&bars[P_MQ]);
        }
        __syncwarp();
      } else if (warp >= 2) {
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;  // j
        const uint32_t lane_off = uint32_t(quarter * 32) << 16;
        if (warp_wait_s(&bars[P_MQ], 0, w)) {
          tc_fence_after();
          __nv_bfloat16* dst = p.mqt + (size_t(slab) * 128 + row) * 128;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t r[32];
            tmem_ld32(tA + lane_off + c * 32, r);
            tmem_wait_ld();
            uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              d4[i] = make_uint4(pack_bf16x2(__uint_as_float(r[8 * i]), __uint_as_float(r[8 * i + 1])),
                                 pack_bf16x2(__uint_as_float(r[8 * i + 2]), __uint_as_float(r[8 * i + 3])),
                                 pack_bf16x2(__uint_as_float(r[8 * i + 4]), __uint_as_float(r[8 * i + 5])),
                                 pack_bf16x2(__uint_as_float(r[8 * i + 6]), __uint_as_float(r[8 * i + 7])));
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    if (warp == 1 && lane == 0) {
      mma_commit(&bars[P_DRAIN]);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(&bars[P_DRAIN], 0) && global_timer_ns() - t0 < 10000000ull) {
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

// S_N = alpha S_{N-1} + c * sum_chunks partial, in fixed chunk order.
// Grid: (B*H, 16); each CTA covers 8 rows (1024 values, 4 per thread).
__global__ void __launch_bounds__(256) state_finalize_kernel(const StateParams p) {
  const int slab = blockIdx.x;
  const int e = (blockIdx.y * 256 + threadIdx.x) * 4;  // element index within the 128x128 state
  if (!ARL2_IN_BOUNDS(p.err, slab < p.batch * p.heads && e + 4 <= 16384)) return;  // (debug build)
  const size_t base = size_t(slab) * 16384 + e;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  const float* part = p.partial + size_t(slab) * p.n_chunks * 16384 + e;
  for (int c = 0; c < p.n_chunks; ++c) {
    const float4 v = *reinterpret_cast<const float4*>(part + size_t(c) * 16384);
    acc.x += v.x;
    acc.y += v.y;
    acc.z += v.z;
    acc.w += v.w;
  }
  const float a = p.alpha[slab];
  const float4 s = *reinterpret_cast<const float4*>(p.S_prev + base);
  float4 r;
  r.x = fmaf(a, s.x, p.corr * acc.x);
  r.y = fmaf(a, s.y, p.corr * acc.y);
  r.z = fmaf(a, s.z, p.corr * acc.z);
  r.w = fmaf(a, s.w, p.corr * acc.w);
  *reinterpret_cast<float4*>(p.S_next + base) = r;
  uint2 bf = make_uint2(pack_bf16x2(r.x, r.y), pack_bf16x2(r.z, r.w));
  *reinterpret_cast<uint2*>(p.S_next_bf + base) = bf;
}

// MqT[j][i] = sum_k S[k][j] phi_q[i][k]: M = j, N = i, K = k.
// A = S^T read from S stored [k][j] (MN-major); B = phi_q stored [i][k] (K-major).
enum { R_IN, R_D, R_COUNT };

__global__ void __launch_bounds__(kStateThreads, 1)
readout_prep_kernel(const __grid_constant__ CUtensorMap tm_s_bf, const __grid_constant__ CUtensorMap tm_phiq,
                    const StateParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sS = smem;
  uint8_t* sP = smem + kTileB;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 2 * kTileB);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + R_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int slab = blockIdx.x;
  const int h = slab % p.heads;
  if (!ARL2_IN_BOUNDS(p.err, slab < p.batch * p.heads)) return;  // (debug build) before any barrier

  if (threadIdx.x == 0) {
    for (int i = 0; i < R_COUNT; ++i) mbar_init(&bars[i], 1u);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_holder, 128);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const WaitCtl w{abort_flag, p.err, p.wait_limit_ns};

  if (warp == 0) {
    if (lane == 0) {
      mbar_expect_tx(&bars[R_IN], 2 * kTileB);
      tma_load_3d(sS, &tm_s_bf, &bars[R_IN], 0, 0, slab);
      tma_load_3d(sS + kHalfB, &tm_s_bf, &bars[R_IN], 64, 0, slab);
      tma_load_3d(sP, &tm_phiq, &bars[R_IN], 0, 0, h);
      tma_load_3d(sP + kHalfB, &tm_phiq, &bars[R_IN], 64, 0, h);
    }
  } else if (warp == 1) {
    if (lane == 0 && mbar_wait(&bars[R_IN], 0, w)) {
      tc_fence_after();
      const uint32_t sa = smem_u32(sS), pa = smem_u32(sP);
      const uint32_t id = idesc_bf16(128, 128, 1, 0);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t boff = (kk >> 2) * kHalfB + (kk & 3) * 32;
        mma_ss(tmem, smem_desc_sw128(sa + kk * 2048, kHalfB, 1024), smem_desc_sw128(pa + boff, 16, 1024), id, kk > 0);
      }
      mma_commit(&bars[R_D]);
    }
  } else {
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;  // j
    const uint32_t lane_off = uint32_t(quarter * 32) << 16;
    if (warp_wait_s(&bars[R_D], 0, w)) {
      tc_fence_after();
      __nv_bfloat16* dst = p.mqt + (size_t(slab) * 128 + row) * 128;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_off + c * 32, r);
        tmem_wait_ld();
        uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
        for (int i = 0; i < 4; ++i)
          d4[i] = make_uint4(pack_bf16x2(__uint_as_float(r[8 * i]), __uint_as_float(r[8 * i + 1])),
                             pack_bf16x2(__uint_as_float(r[8 * i + 2]), __uint_as_float(r[8 * i + 3])),
                             pack_bf16x2(__uint_as_float(r[8 * i + 4]), __uint_as_float(r[8 * i + 5])),
                             pack_bf16x2(__uint_as_float(r[8 * i + 6]), __uint_as_float(r[8 * i + 7])));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    if (warp == 1 && lane == 0) {
      const uint64_t t0 = global_timer_ns();
      while (global_timer_ns() - t0 < 2000000ull) {
      }
    }
    __syncthreads();
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

cudaError_t launch_state_partial(const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tpk,
                                 const CUtensorMap& tpv, const CUtensorMap& ts, const StateParams& p, int batch,
                                 cudaStream_t stream) {
  static unsigned done = 0;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(state_partial_kernel<false>), kPartialSmem, &done);
  if (e != cudaSuccess) return e;
  dim3 grid(p.n_chunks, p.heads, batch);
  state_partial_kernel<false><<<grid, kStateThreads, kPartialSmem, stream>>>(tk, tv, tpk, tpv, ts, ts, p);
  return cudaGetLastError();
}

namespace {
cudaLaunchConfig_t fused_config(int n_chunks, int heads, int batch, cudaLaunchAttribute* attr) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_chunks, heads, batch);
  cfg.blockDim = dim3(kStateThreads);
  cfg.dynamicSmemBytes = kPartialSmem;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = n_chunks;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cfg;
}
cudaError_t fused_attrs() {
  static unsigned done = 0;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(state_partial_kernel<true>), kPartialSmem, &done);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(state_partial_kernel<true>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
}
}  // namespace

bool state_fused_supported(int n_chunks, int heads, int batch) {
  if (n_chunks < 1 || n_chunks > 16) return false;
  if (fused_attrs() != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = fused_config(n_chunks, heads, batch, attr);
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, state_partial_kernel<true>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return n >= 1;
}

cudaError_t launch_state_fused(const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tpk,
                               const CUtensorMap& tpv, const CUtensorMap& ts, const CUtensorMap& tphiq,
                               const StateParams& p, int batch, cudaStream_t stream) {
  cudaError_t e = fused_attrs();
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = fused_config(p.n_chunks, p.heads, batch, attr);
  cfg.stream = stream;
  return cudaLaunchKernelEx(&cfg, state_partial_kernel<true>, tk, tv, tpk, tpv, ts, tphiq, p);
}

cudaError_t launch_state_finalize(const StateParams& p, int batch, cudaStream_t stream) {
  dim3 grid(batch * p.heads, 16);
  state_finalize_kernel<<<grid, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_readout_prep(const CUtensorMap& ts, const CUtensorMap& tphiq, const StateParams& p, int batch,
                                cudaStream_t stream) {
  static unsigned done = 0;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(readout_prep_kernel), kPrepSmem, &done);
  if (e != cudaSuccess) return e;
  readout_prep_kernel<<<batch * p.heads, kStateThreads, kPrepSmem, stream>>>(ts, tphiq, p);
  return cudaGetLastError();
}

}  // namespace arl2
