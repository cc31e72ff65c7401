// The hybrid attention block: the hybrid layer with the projections a DiT
// attention block puts around it, and the commit's gates from the tokens.
//
//   Q, K, V = X W_qkv (three column blocks of D),  O = hybrid layer (Q, K, V),
//   Y = O W_o;  on the commit pass  alpha = sigmoid(mean_t X W_gate[:, :H]),
//   beta = sigmoid(X W_gate[:, H:])
//
// (ARL2 summary, section 2.1: the frozen pretrained Q/K/V projections feed
// both branches; alpha and beta are per-token learned projections; the
// pooling of alpha over the frame is this build's reading.)  The projections
// run on this library's tcgen05 GEMM (gemm_bf16.cu; bf16 in, fp32
// accumulate): one GEMM against the column-concatenated [W_qkv | W_gate]
// gives Q, K, V and the gates' logits side by side in each token's row, which
// the layer reads as strided views; the hybrid layer is this library's own
// handle; the gates are one small kernel here.

#include <cstdint>
#include <mutex>
#include <new>
#include <set>

#include "arl2.h"
#include "layer.h"
#include "params.h"

namespace arl2 {

// alpha[b][h] = sigmoid(mean_t g[b][t][h]); beta[b][h][t] = sigmoid(g[b][t][H + h]),
// g bf16 with token rows `ld` elements apart.  One CTA per (stream, head); the
// mean is a fixed-order reduction.
__global__ void __launch_bounds__(256) block_gates_kernel(const __nv_bfloat16* __restrict__ g, int64_t ld,
                                                          float* __restrict__ alpha, float* __restrict__ beta, int L,
                                                          int H) {
  const int bh = blockIdx.x, b = bh / H, h = bh % H;
  float sum = 0.f;
  for (int t = threadIdx.x; t < L; t += blockDim.x) {
    const __nv_bfloat16* row = g + (size_t(b) * L + t) * ld;
    sum += __bfloat162float(row[h]);
    beta[size_t(bh) * L + t] = 1.f / (1.f + expf(-__bfloat162float(row[H + h])));
  }
  __shared__ float part[8];
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = sum;
  __syncthreads();
  if (threadIdx.x == 0) {
    float tot = 0.f;
    for (int w = 0; w < int(blockDim.x >> 5); ++w) tot += part[w];
    alpha[bh] = 1.f / (1.f + expf(-tot / float(L)));
  }
}

}  // namespace arl2

namespace {

constexpr uint64_t kBlockMagic = 0x41524c32424c4b31ull;  // "ARL2BLK1"

std::mutex g_block_mu;
std::set<const void*> g_blocks;

bool live_block(const arl2_block_t b);

}  // namespace

struct arl2_block {
  uint64_t magic;
  arl2_config cfg;
  arl2_state_t layer;
  int sms;       // persistent GEMM grid
  int64_t ldw;   // columns of w_all and qkvg: 3D, then 2H gate columns, padded to a multiple of 8
  void* w_all;   // [D, ldw] bf16: W_qkv | W_gate | 0
  void* w_o;
  void* qkvg;    // [B * L, ldw] bf16: Q | K | V | gate logits per token
  void* o;
  float* alpha;
  float* beta;
};

namespace {

bool live_block(const arl2_block_t b) {
  std::lock_guard<std::mutex> lk(g_block_mu);
  return b && g_blocks.count(b) && b->magic == kBlockMagic;
}

arl2_status from_cuda_e(cudaError_t e) {
  return e == cudaErrorMemoryAllocation ? ARL2_ERR_OUT_OF_MEMORY : ARL2_ERR_CUDA;
}

bool aligned(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

void free_block(arl2_block* b) {
  if (b->layer) arl2_state_destroy(b->layer);
  for (void* p : {b->w_all, b->w_o, b->qkvg, b->o, (void*)b->alpha, (void*)b->beta})
    if (p) cudaFree(p);
  b->magic = 0;
  delete b;
}

// Row-major C[M][N] (ldc) = A[M][K] (lda) * B[K][N] (ldb) on the library's
// GEMM; a wait that runs out is recorded in the layer's error word.
arl2_status gemm(const arl2_block* b, int M, int N, int K, const void* A, int64_t lda, const void* B, int64_t ldb,
                 void* C, int64_t ldc, cudaStream_t st) {
  arl2::GemmParams p{};
  p.M = M;
  p.N = N;
  p.K = K;
  p.err = arl2::layer_error_word(b->layer);
  p.wait_limit_ns = arl2::layer_wait_limit(b->layer);
  return arl2::gemm_bf16(A, lda, B, ldb, C, ldc, p, b->sms, st) == cudaSuccess ? ARL2_OK : ARL2_ERR_CUDA;
}

// Q | K | V | gate logits = X [W_qkv | W_gate], one token row each.
arl2_status project_in(arl2_block* b, const void* x, cudaStream_t st) {
  const int D = b->cfg.heads * b->cfg.head_dim, M = b->cfg.batch * b->cfg.tokens_per_frame;
  return gemm(b, M, int(b->ldw), D, x, D, b->w_all, b->ldw, b->qkvg, b->ldw, st);
}

arl2_status project_out(arl2_block* b, void* y, cudaStream_t st) {
  const int D = b->cfg.heads * b->cfg.head_dim, M = b->cfg.batch * b->cfg.tokens_per_frame;
  return gemm(b, M, D, D, b->o, D, b->w_o, D, y, D, st);
}

bool overlap(const void* a, const void* c, size_t n) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(c);
  return x < y + n && y < x + n;
}

arl2_status check_xy(const arl2_block* b, const void* x, const void* y) {
  if (!x || !y || !aligned(x) || !aligned(y)) return ARL2_ERR_INVALID_ARGUMENT;
  const size_t n = size_t(b->cfg.batch) * b->cfg.tokens_per_frame * b->cfg.heads * b->cfg.head_dim * 2;
  return overlap(x, y, n) ? ARL2_ERR_INVALID_ARGUMENT : ARL2_OK;
}

}  // namespace

extern "C" {

arl2_status arl2_block_init(const arl2_config* cfg, const void* w_qkv, const void* w_o, const void* w_gate,
                            const void* phi_q, const void* phi_k, const void* phi_v, void* stream,
                            arl2_block_t* out) {
  if (!out) return ARL2_ERR_INVALID_ARGUMENT;
  *out = nullptr;
  if (!cfg || !w_qkv || !w_o || !w_gate || !aligned(w_qkv) || !aligned(w_o) || !aligned(w_gate))
    return ARL2_ERR_INVALID_ARGUMENT;
  if (cfg->batch < 1 || cfg->heads < 1 || cfg->tokens_per_frame < 1) return ARL2_ERR_INVALID_ARGUMENT;
  if (cfg->dtype != ARL2_BF16 || cfg->head_dim != 128) return ARL2_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  arl2_block* b = new (std::nothrow) arl2_block();
  if (!b) return ARL2_ERR_OUT_OF_MEMORY;
  b->cfg = *cfg;
  arl2_status s = arl2_state_init(cfg, phi_q, phi_k, phi_v, stream, &b->layer);
  if (s != ARL2_OK) {
    b->layer = nullptr;
    free_block(b);
    return s;
  }
  const size_t D = size_t(cfg->heads) * cfg->head_dim, H = cfg->heads;
  const size_t M = size_t(cfg->batch) * cfg->tokens_per_frame;
  b->ldw = int64_t(3 * D + ((2 * H + 7) / 8) * 8);
  const size_t ldw = size_t(b->ldw);
  cudaError_t e = cudaSuccess;
  auto alloc = [&](void** p, size_t n) {
    if (e == cudaSuccess) e = cudaMalloc(p, n);
  };
  alloc(&b->w_all, D * ldw * 2);
  alloc(&b->w_o, D * D * 2);
  alloc(&b->qkvg, M * ldw * 2);
  alloc(&b->o, M * D * 2);
  alloc(reinterpret_cast<void**>(&b->alpha), size_t(cfg->batch) * H * sizeof(float));
  alloc(reinterpret_cast<void**>(&b->beta), M * H * sizeof(float));
  auto* wa = static_cast<__nv_bfloat16*>(b->w_all);
  if (e == cudaSuccess) e = cudaMemsetAsync(b->w_all, 0, D * ldw * 2, st);
  if (e == cudaSuccess)
    e = cudaMemcpy2DAsync(wa, ldw * 2, w_qkv, 3 * D * 2, 3 * D * 2, D, cudaMemcpyDeviceToDevice, st);
  if (e == cudaSuccess)
    e = cudaMemcpy2DAsync(wa + 3 * D, ldw * 2, w_gate, 2 * H * 2, 2 * H * 2, D, cudaMemcpyDeviceToDevice, st);
  if (e == cudaSuccess) e = cudaMemcpyAsync(b->w_o, w_o, D * D * 2, cudaMemcpyDeviceToDevice, st);
  if (e != cudaSuccess) {
    free_block(b);
    return from_cuda_e(e);
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&b->sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || b->sms < 1) {
    free_block(b);
    return ARL2_ERR_CUDA;
  }
  b->magic = kBlockMagic;
  {
    std::lock_guard<std::mutex> lk(g_block_mu);
    g_blocks.insert(b);
  }
  *out = b;
  return ARL2_OK;
}

arl2_status arl2_block_query(arl2_block_t b, const void* x, void* y, void* stream) {
  if (!live_block(b)) return ARL2_ERR_INVALID_ARGUMENT;
  arl2_status s = check_xy(b, x, y);
  if (s != ARL2_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((s = project_in(b, x, st)) != ARL2_OK) return s;
  const int D = b->cfg.heads * b->cfg.head_dim;
  const auto* in = static_cast<const __nv_bfloat16*>(b->qkvg);
  if ((s = arl2::layer_query_ld(b->layer, in, in + D, in + 2 * D, b->ldw, b->o, st)) != ARL2_OK) return s;
  return project_out(b, y, st);
}

arl2_status arl2_block_commit(arl2_block_t b, const void* x, void* y, void* stream) {
  if (!live_block(b)) return ARL2_ERR_INVALID_ARGUMENT;
  arl2_status s = check_xy(b, x, y);
  if (s != ARL2_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((s = project_in(b, x, st)) != ARL2_OK) return s;
  const int D = b->cfg.heads * b->cfg.head_dim, H = b->cfg.heads;
  const auto* in = static_cast<const __nv_bfloat16*>(b->qkvg);
  arl2::block_gates_kernel<<<b->cfg.batch * H, 256, 0, st>>>(in + 3 * D, b->ldw, b->alpha, b->beta,
                                                             b->cfg.tokens_per_frame, H);
  if (cudaGetLastError() != cudaSuccess) return ARL2_ERR_CUDA;
  if ((s = arl2::layer_commit_ld(b->layer, in, in + D, in + 2 * D, b->ldw, b->alpha, b->beta, b->o, st)) != ARL2_OK)
    return s;
  return project_out(b, y, st);
}

arl2_state_t arl2_block_layer(arl2_block_t b) { return live_block(b) ? b->layer : nullptr; }

arl2_status arl2_block_destroy(arl2_block_t b) {
  if (!live_block(b)) return ARL2_ERR_INVALID_ARGUMENT;
  {
    std::lock_guard<std::mutex> lk(g_block_mu);
    g_blocks.erase(b);
  }
  free_block(b);  // the layer's destroy first synchronises the stream of its (and the GEMMs') last call
  return ARL2_OK;
}

}  // extern "C"
