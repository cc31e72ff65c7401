// Small helper kernels of the library: parameter transposes and conversions
// done once per handle or per state restore, the bounded-wait self-test, and
// the per-device shared-memory attribute cache.

#include "params.h"
#include "sm100.cuh"

namespace arl2 {

// dst[s][j][i] = src[s][i][j] for stacked 128 x 128 bf16 matrices.
__global__ void transpose128_kernel(const __nv_bfloat16* __restrict__ src, __nv_bfloat16* __restrict__ dst) {
  __shared__ __nv_bfloat16 tile[32][33];
  const size_t base = size_t(blockIdx.z) * 128 * 128;
  const int i0 = blockIdx.y * 32, j0 = blockIdx.x * 32;
  for (int r = threadIdx.y; r < 32; r += 8) tile[r][threadIdx.x] = src[base + size_t(i0 + r) * 128 + j0 + threadIdx.x];
  __syncthreads();
  for (int r = threadIdx.y; r < 32; r += 8) dst[base + size_t(j0 + r) * 128 + i0 + threadIdx.x] = tile[threadIdx.x][r];
}

cudaError_t launch_transpose_bf16(const __nv_bfloat16* src, __nv_bfloat16* dst, int slabs, cudaStream_t stream) {
  dim3 grid(4, 4, slabs), block(32, 8);
  transpose128_kernel<<<grid, block, 0, stream>>>(src, dst);
  return cudaGetLastError();
}

__global__ void to_bf16_kernel(const float* __restrict__ src, __nv_bfloat16* __restrict__ dst, size_t n) {
  for (size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += size_t(gridDim.x) * blockDim.x)
    dst[i] = __float2bfloat16_rn(src[i]);
}

cudaError_t launch_to_bf16(const float* src, __nv_bfloat16* dst, size_t n, cudaStream_t stream) {
  const int blocks = int((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
  to_bf16_kernel<<<blocks, 256, 0, stream>>>(src, dst, n);
  return cudaGetLastError();
}

// One thread waits, with the library's bounded wait, on an mbarrier that
// nothing completes; the wait must give up, record the timeout and return.
__global__ void wait_selftest_kernel(uint32_t* err, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1u);
    abort_flag = 0;
    fence_barrier_init();
    const WaitCtl w{&abort_flag, err, limit_ns};
    if (mbar_wait(&bar, 0, w)) record_error(err, 1u);  // completing would be a bug
  }
}

cudaError_t launch_wait_selftest(uint32_t* err, uint64_t limit_ns, cudaStream_t stream) {
  wait_selftest_kernel<<<1, 32, 0, stream>>>(err, limit_ns);
  return cudaGetLastError();
}

// y = 2^x through the attention kernel's FMA-pipe exp2 (for its accuracy test).
__global__ void exp2_poly_kernel(const float* __restrict__ x, float* __restrict__ y, long long n) {
  const long long i = 2 * ((long long)blockIdx.x * blockDim.x + threadIdx.x);
  if (i + 1 < n) {
    exp2_poly2(y[i], y[i + 1], x[i], x[i + 1]);
  } else if (i < n) {
    float d;
    exp2_poly2(y[i], d, x[i], 0.f);
  }
}

cudaError_t launch_exp2_poly(const float* x, float* y, long long n, cudaStream_t stream) {
  const long long pairs = (n + 1) / 2;
  exp2_poly_kernel<<<unsigned((pairs + 255) / 256), 256, 0, stream>>>(x, y, n);
  return cudaGetLastError();
}

cudaError_t ensure_smem_attr(const void* func, int bytes, unsigned* done_mask) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned bit = 1u << (dev & 31);
  if (*done_mask & bit) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) __atomic_fetch_or(done_mask, bit, __ATOMIC_RELAXED);
  return e;
}

}  // namespace arl2
