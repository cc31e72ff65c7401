// Dense projection GEMM of the attention block, bf16 operands, fp32
// accumulation in tensor memory, bf16 output (sm_100a):
//
//   C[M][N] = A[M][K] B[K][N]      (all row-major; A = token rows, B = weights)
//
// Persistent clusters of two CTAs (one per SM of a pair) walk 256 x 256
// output tiles with tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 16: the
// shape that keeps the tensor cores at their full rate).  Per tile each CTA
// streams K-slices of 64 through a 6-stage TMA ring: its own 128 rows of A
// (K-major) and its own 128 of the 256 columns of B (read as an MN-major
// operand), so that a CTA reads a third less from L2 per output than a
// single-SM 128 x 256 tile.  Rank 0's thread issues the MMAs into one of two
// tensor-memory accumulators (256 columns each; every CTA holds its 128 rows);
// each CTA's epilogue warpgroup drains the other accumulator -- bf16
// conversion, 64-column chunks staged in shared memory, TMA tile stores (rows
// and columns past M and N are clipped by the tensor map) -- while the next
// tile accumulates.  No load uses cluster multicast.

#include <cudaTypedefs.h>

#include "params.h"
#include "sm100.cuh"

namespace arl2 {

namespace {

constexpr int kThreads = 256;
constexpr int kStages = 6;
constexpr int kBM = 128, kBN = 128, kBK = 64;  // per CTA: its rows of A, its half of the pair's 256 columns
constexpr uint32_t kABytes = kBM * kBK * 2;   // 16 KB
constexpr uint32_t kBBytes = kBK * kBN * 2;   // 16 KB: two 64-column boxes of 64 rows
constexpr uint32_t kStageBytes = kABytes + kBBytes;
constexpr uint32_t kStageOut = 2 * 4096;      // per epilogue warp: two 32-row x 64-column boxes
constexpr uint32_t kTiles = kStages * kStageBytes + 4 * kStageOut;
constexpr int kSmem = int(kTiles) + 256 + 1024;
static_assert(kSmem <= 232448, "shared memory layout too large");

enum { G_FULL = 0, G_EMPTY = kStages, G_AF = 2 * kStages, G_AE = G_AF + 2, G_DRAIN = G_AE + 2, G_COUNT };

__device__ __forceinline__ bool warp_wait_g(uint64_t* bar, uint32_t parity, const WaitCtl& w) {
  const bool ok = mbar_wait(bar, parity, w);
  return __all_sync(0xffffffffu, ok);
}

// 2-D tile load into this CTA's shared memory whose bytes count on the pair
// leader's mbarrier at the same offset.
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1) {
  const uint32_t leader_bar = cluster_map(smem_u32(bar), 0);
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(leader_bar), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int c0, int c1) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(c0), "r"(c1)
               : "memory");
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
gemm_bf16_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                 const __grid_constant__ CUtensorMap tm_c, const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sOut = smem + kStages * kStageBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kTiles);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + G_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rank = int(cluster_ctarank());
  const int pair = blockIdx.x >> 1, pairs = gridDim.x >> 1;
  // the same offset in both CTAs (both launch with the same dynamic shared memory)
  const bool fits = size_t(smem - smem_raw) + kTiles + 256 <= size_t(kSmem);
  if (threadIdx.x == 0) {
    for (int i = 0; i < G_COUNT; ++i) mbar_init(&bars[i], (i == G_AE || i == G_AE + 1) ? 8u : 1u);
    *abort_flag = fits ? 0 : 1;
    fence_barrier_init();
  }
  if (warp == 2) tmem_alloc_pair(tmem_holder, 512);
  tc_fence_before();
  __syncthreads();
  cluster_barrier();  // both CTAs' barriers initialised before any remote arrive or load
  tc_fence_after();
  // The set-up above may overlap the kernel before this one on the stream;
  // every global access below follows its completion.
  grid_dependency_wait();
  allow_dependent_launch();
  if (threadIdx.x == 0 && !fits) record_error(p.err, kDevBadShape);
  const uint32_t tmem = *tmem_holder;
  const WaitCtl w{abort_flag, p.err, p.wait_limit_ns};
  const int tiles_m = (p.M + 2 * kBM - 1) / (2 * kBM), tiles_n = (p.N + 2 * kBN - 1) / (2 * kBN);
  const int n_tiles = tiles_m * tiles_n;
  const int nk = (p.K + kBK - 1) / kBK;

  if (!*abort_flag) {
    if (warp == 0 && lane == 0) {  // ---------------------------------------- producer (both CTAs)
      tma_prefetch(&tm_a);
      tma_prefetch(&tm_b);
      uint32_t it = 0;
      for (int t = pair; t < n_tiles; t += pairs) {
        const int m0 = (t % tiles_m) * 2 * kBM + rank * kBM, n0 = (t / tiles_m) * 2 * kBN + rank * kBN;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const uint32_t s = it % kStages;
          if (it >= kStages && !mbar_wait(&bars[G_EMPTY + s], ((it / kStages) - 1) & 1, w)) break;
          uint8_t* dst = smem + s * kStageBytes;
          if (rank == 0) mbar_expect_tx(&bars[G_FULL + s], 2 * kStageBytes);
          tma_load_2d_pair(dst, &tm_a, &bars[G_FULL + s], kb * kBK, m0);
          tma_load_2d_pair(dst + kABytes, &tm_b, &bars[G_FULL + s], n0, kb * kBK);
          tma_load_2d_pair(dst + kABytes + kBBytes / 2, &tm_b, &bars[G_FULL + s], n0 + 64, kb * kBK);
        }
        if (*abort_flag) break;
      }
    } else if (warp == 1 && lane == 0 && rank == 0) {  // -------------------- MMA issuer (rank 0)
      const uint32_t id = idesc_bf16(2 * kBM, 2 * kBN, 0, 1);
      const uint32_t base = smem_u32(smem);
      const uint64_t da64 = smem_desc_sw128(base, 16, 1024);                     // A: K-major, 128-byte rows
      const uint64_t db64 = smem_desc_sw128(base + kABytes, kBBytes / 2, 1024);  // B: MN-major, 64-column boxes 8 KB apart
      const uint32_t hi = uint32_t(da64 >> 32);
      const uint32_t da0 = uint32_t(da64), db0 = uint32_t(db64);
      uint32_t it = 0, tc = 0;
      for (int t = pair; t < n_tiles; t += pairs, ++tc) {
        const uint32_t acc = tc & 1;
        // both CTAs' epilogues have drained this accumulator (two tiles ago)
        if (tc >= 2 && !mbar_wait(&bars[G_AE + acc], ((tc >> 1) - 1) & 1, w)) break;
        tc_fence_after();
        const uint32_t d = tmem + acc * 256;
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const uint32_t s = it % kStages;
          if (!mbar_wait(&bars[G_FULL + s], (it / kStages) & 1, w)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t so = (s * kStageBytes) >> 4;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_pair_ss(d, da0 + so + kk * 2, db0 + so + kk * 128, hi, id, uint32_t(kb > 0 || kk > 0));
          mma_commit_pair(&bars[G_EMPTY + s]);
        }
        if (!ok) break;
        mma_commit_pair(&bars[G_AF + acc]);
      }
    } else if (warp >= 4) {  // ------------------------------------------------ epilogue (both CTAs)
      const int quarter = warp & 3;
      const uint32_t lane_off = uint32_t(quarter * 32) << 16;
      const uint32_t ae_leader = cluster_map(smem_u32(&bars[G_AE]), 0);
      uint8_t* wst = sOut + quarter * kStageOut;
      uint32_t tc = 0, stores = 0;
      for (int t = pair; t < n_tiles; t += pairs, ++tc) {
        const int m0 = (t % tiles_m) * 2 * kBM + rank * kBM, n0 = (t / tiles_m) * 2 * kBN;
        const uint32_t acc = tc & 1;
        if (!warp_wait_g(&bars[G_AF + acc], (tc >> 1) & 1, w)) break;
        tc_fence_after();
        const uint32_t src = tmem + acc * 256 + lane_off;
        const bool warp_on = m0 + quarter * 32 < p.M;
#pragma unroll 1
        for (int q = 0; q < 4; ++q) {  // 64 output columns at a time
          uint32_t r0[32], r1[32];
          tmem_ld32(src + q * 64, r0);
          tmem_ld32(src + q * 64 + 32, r1);
          tmem_wait_ld();
          if (q == 3) {  // the accumulator is read: the MMA may reuse it
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster_relaxed(ae_leader + acc * 8);
          }
          uint8_t* box = wst + (stores & 1) * 4096;
          if (lane == 0 && stores >= 2) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
          __syncwarp();
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint32_t* r = c < 4 ? r0 + 8 * c : r1 + 8 * (c - 4);
            *reinterpret_cast<uint4*>(box + lane * 128 + ((c ^ (lane & 7)) << 4)) =
                make_uint4(pack_bf16x2(__uint_as_float(r[0]), __uint_as_float(r[1])),
                           pack_bf16x2(__uint_as_float(r[2]), __uint_as_float(r[3])),
                           pack_bf16x2(__uint_as_float(r[4]), __uint_as_float(r[5])),
                           pack_bf16x2(__uint_as_float(r[6]), __uint_as_float(r[7])));
          }
          fence_async_smem();
          __syncwarp();
          if (lane == 0 && warp_on && n0 + 64 * q < p.N) tma_store_2d(&tm_c, box, n0 + 64 * q, m0 + quarter * 32);
          if (lane == 0) bulk_commit();
          ++stores;
        }
      }
      if (lane == 0) bulk_wait0();
    }
  }

  // ------------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1 && lane == 0 && rank == 0) {  // every MMA completed before tensor memory is released
    mma_commit_pair(&bars[G_DRAIN]);
  }
  if (warp == 1 && lane == 0) {  // both CTAs see the drain commit (multicast)
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(&bars[G_DRAIN], 0) && global_timer_ns() - t0 < 10000000ull) {
    }
  }
  if (*abort_flag && warp == 0 && lane == 0) {  // copies in flight land before shared memory goes away
    const uint64_t t0 = global_timer_ns();
    while (global_timer_ns() - t0 < 2000000ull) {
    }
  }
  __syncthreads();
  cluster_barrier();  // neither CTA leaves while the other may still signal it
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

}  // namespace

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_tiled() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }
  return fn;
}

// 2-D bf16 matrix of `rows` x `cols` (row pitch `ld` elements), 128-byte
// swizzle, boxes of 64 columns x `box_rows` rows; out-of-range elements read
// as zero and are not written.
bool make_2d(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint64_t ld, uint32_t box_rows) {
  auto fn = encode_tiled();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {ld * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t gemm_bf16(const void* A, int64_t lda, const void* B, int64_t ldb, void* C, int64_t ldc, const GemmParams& p,
                      int sms, cudaStream_t stream) {
  if (p.M < 1 || p.N < 1 || p.K < 1) return cudaSuccess;
  if ((lda | ldb | ldc) % 8 != 0 || lda < p.K || ldb < p.N || ldc < p.N) return cudaErrorInvalidValue;
  CUtensorMap ta, tb, tc;
  if (!make_2d(&ta, A, uint64_t(p.M), uint64_t(p.K), uint64_t(lda), kBM) ||
      !make_2d(&tb, B, uint64_t(p.K), uint64_t(p.N), uint64_t(ldb), kBK) ||
      !make_2d(&tc, C, uint64_t(p.M), uint64_t(p.N), uint64_t(ldc), 32))
    return cudaErrorInvalidValue;
  static unsigned done = 0;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(gemm_bf16_kernel), kSmem, &done);
  if (e != cudaSuccess) return e;
  const int tiles = ((p.M + 2 * kBM - 1) / (2 * kBM)) * ((p.N + 2 * kBN - 1) / (2 * kBN));
  cudaLaunchConfig_t cfg{};
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = size_t(kSmem);
  cfg.stream = stream;
  // clusters of two resident at once
  int cap = 0;
  cfg.gridDim = dim3(2);
  e = cudaOccupancyMaxActiveClusters(&cap, gemm_bf16_kernel, &cfg);
  if (e != cudaSuccess) return e;
  if (cap < 1) return cudaErrorInvalidConfiguration;
  (void)sms;
  const int pairs = tiles < cap ? tiles : cap;
  cfg.gridDim = dim3(2 * pairs);
  // programmatic stream serialisation: the grid's set-up may overlap the
  // previous kernel's tail (the kernel waits for it before any global access)
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, gemm_bf16_kernel, ta, tb, tc, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace arl2
