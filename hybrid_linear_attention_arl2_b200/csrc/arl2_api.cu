// C ABI of libarl2.so (declared in include/arl2.h): handles, argument
// validation, device allocations, TMA descriptors and kernel dispatch.
// Every step of the hot path runs in this library's kernels; the host code
// here only checks arguments, encodes descriptors and enqueues launches.

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <algorithm>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>
#include <set>

#include "../../include/arl2.h"

#include "layer.h"
#include "params.h"

using namespace arl2;

namespace {

constexpr uint64_t kStateMagic = 0x41524c3253544154ull;  // "ARL2STAT"
constexpr uint64_t kKvMagic = 0x41524c324b564341ull;     // "ARL2KVCA"
constexpr uint64_t kDefaultWaitNs = 1000000000ull;

std::mutex g_mu;
std::set<const void*> g_live;  // live handles, to reject destroyed or foreign pointers

// Allocation failure injection for the out-of-memory tests: ARL2_FAIL_ALLOC_AT=n
// makes the n-th device allocation of the process (1-based) fail.
std::atomic<long> g_alloc_count{0};

cudaError_t dev_alloc(void** p, size_t bytes) {
  const long n = ++g_alloc_count;
  const char* s = std::getenv("ARL2_FAIL_ALLOC_AT");
  if (s && *s && std::atol(s) == n) {
    *p = nullptr;
    return cudaErrorMemoryAllocation;
  }
  return cudaMalloc(p, bytes);
}

bool log_enabled() {
  static int v = -1;
  if (v < 0) {
    const char* s = std::getenv("ARL2_LOG");
    v = (s && *s && *s != '0') ? 1 : 0;
  }
  return v == 1;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 3-D bf16 map, 128-byte swizzle, box {64, rows, 1}; out-of-range elements read as 0.
bool make_map(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t stride1,
              uint64_t stride2, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {stride1, stride2};
  cuuint32_t box[3] = {64, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Token-major activations [B, tokens, H, 128] as a map over (H*128, tokens, B),
// boxes of 64 columns x `rows` tokens.
// `ld`: elements from one token's row to the next (0: H * 128, contiguous).
bool make_act_map(CUtensorMap* m, const void* base, int B, int64_t tokens, int H, uint32_t rows = 128,
                  int64_t ld = 0) {
  const uint64_t row = uint64_t(ld > 0 ? ld : int64_t(H) * 128) * 2;
  return make_map(m, base, uint64_t(H) * 128, uint64_t(tokens), uint64_t(B), row, row * uint64_t(tokens), rows);
}

// Stacked 128 x 128 bf16 matrices [slabs, 128, 128] as a map over (128, 128, slabs).
bool make_mat_map(CUtensorMap* m, const void* base, int slabs, uint32_t rows = 128) {
  return make_map(m, base, 128, 128, uint64_t(slabs), 256, 256 * 128, rows);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

arl2_status from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return ARL2_OK;
  if (e == cudaErrorMemoryAllocation) return ARL2_ERR_OUT_OF_MEMORY;
  if (e == cudaErrorNoDevice || e == cudaErrorInsufficientDriver) return ARL2_ERR_NO_DEVICE;
  return ARL2_ERR_CUDA;
}

arl2_status check_config(const arl2_config* c) {
  if (!c) return ARL2_ERR_INVALID_ARGUMENT;
  if (c->batch < 1 || c->heads < 1 || c->head_dim < 1 || c->tokens_per_frame < 1) return ARL2_ERR_INVALID_ARGUMENT;
  if (c->dtype != ARL2_F32 && c->dtype != ARL2_BF16) return ARL2_ERR_UNSUPPORTED;
  if (c->flags & ~(ARL2_INTRA_ONLY | ARL2_INTER_ONLY)) return ARL2_ERR_INVALID_ARGUMENT;
  if (c->flags == (ARL2_INTRA_ONLY | ARL2_INTER_ONLY)) return ARL2_ERR_INVALID_ARGUMENT;
  if (!(std::isfinite(c->softmax_scale)) || c->softmax_scale < 0.f) return ARL2_ERR_INVALID_ARGUMENT;
  if (!std::isfinite(c->corr_scale)) return ARL2_ERR_INVALID_ARGUMENT;
  if (c->dtype == ARL2_BF16) {
    if (c->head_dim != 128) return ARL2_ERR_UNSUPPORTED;
    if (c->tokens_per_frame > (1 << 24)) return ARL2_ERR_UNSUPPORTED;
    if (int64_t(c->batch) * c->heads > 65535) return ARL2_ERR_UNSUPPORTED;
  } else {
    if (c->head_dim > 128 || c->tokens_per_frame > 4096) return ARL2_ERR_UNSUPPORTED;
    if (int64_t(c->batch) * c->heads > 65535) return ARL2_ERR_UNSUPPORTED;
  }
  return ARL2_OK;
}

float softmax_scale(const arl2_config& c) {
  return c.softmax_scale > 0.f ? c.softmax_scale : 1.f / std::sqrt(float(c.head_dim));
}

}  // namespace

struct arl2_state {
  uint64_t magic;
  arl2_config cfg;
  int device;
  float scale;
  float corr;
  uint64_t wait_ns;
  // f32: phi as given [H,d,d]; bf16: phi_q [H][i][k] as given, phi_k^T and phi_v^T [H][j][i]
  void* phi[3];
  float* S[2];
  int cur;
  __nv_bfloat16* S_bf;   // bf16 copy of S[cur] (bf16 path)
  __nv_bfloat16* mqt;    // two slots of (phi_q S[i])^T, slot cur in use (bf16 path)
  float* partial;        // per-chunk state-write partials (bf16 path)
  int n_chunks;
  float* attn_scratch;   // partial rows of split query blocks (bf16 path)
  unsigned* attn_ready;  // their ready flags, zero between launches
  int sms;
  int pairs;             // CTA pairs of the attention kernel resident at once
  bool state_fused;      // the state write runs as one cluster launch (<= 16 chunks)
  uint32_t* err;
  int64_t frame;
  int64_t bytes;
  cudaStream_t last_stream;
  // The commit's state-write kernels run on `side`, forked from and joined
  // back to the caller's stream (bf16 path).
  cudaStream_t side;
  cudaEvent_t ev_fork, ev_join;
  CUtensorMap tm_phiq, tm_phik_t, tm_phiv_t, tm_s_bf, tm_mqt[2];
  CUtensorMap tm_mqt64[2];  // the same MqT slots in 64-row boxes (a CTA's half for the pair kernel)
  float* tok;  // scratch of the token-level calls, allocated by the first one (bf16 path)
};

struct arl2_kv {
  uint64_t magic;
  arl2_config cfg;
  int device;
  float scale;
  uint64_t wait_ns;
  int32_t max_frames;
  int64_t frames;
  void* kc;  // [B, max_frames*L, H, d]
  void* vc;
  float* attn_scratch;
  unsigned* attn_ready;
  int sms;
  int pairs;  // CTA pairs of the attention kernel resident at once
  uint32_t* err;
  int64_t bytes;
  cudaStream_t last_stream;
};

namespace {

template <class T>
bool live(const T* h, uint64_t magic) {
  if (!h) return false;
  std::lock_guard<std::mutex> g(g_mu);
  return g_live.count(h) && h->magic == magic;
}

void free_state(arl2_state* h) {
  for (void* p : {h->phi[0], h->phi[1], h->phi[2], (void*)h->S[0], (void*)h->S[1], (void*)h->S_bf, (void*)h->mqt,
                  (void*)h->partial, (void*)h->attn_scratch, (void*)h->attn_ready, (void*)h->err, (void*)h->tok})
    if (p) cudaFree(p);
  if (h->ev_fork) cudaEventDestroy(h->ev_fork);
  if (h->ev_join) cudaEventDestroy(h->ev_join);
  if (h->side) cudaStreamDestroy(h->side);
  h->magic = 0;
  delete h;
}

void free_kv(arl2_kv* h) {
  for (void* p : {h->kc, h->vc, (void*)h->attn_scratch, (void*)h->attn_ready, (void*)h->err})
    if (p) cudaFree(p);
  h->magic = 0;
  delete h;
}

#define ARL2_TRY(expr)                          \
  do {                                          \
    cudaError_t e_ = (expr);                    \
    if (e_ != cudaSuccess) return from_cuda(e_); \
  } while (0)

__nv_bfloat16* mqt_slot(const arl2_state* h, int i) {
  return h->mqt + size_t(i) * h->cfg.batch * h->cfg.heads * h->cfg.head_dim * h->cfg.head_dim;
}

arl2_status prepare_readout(arl2_state* h, cudaStream_t st) {
  // MqT = (phi_q S[cur])^T from the bf16 copy of S[cur].
  StateParams sp{};
  sp.mqt = mqt_slot(h, h->cur);
  sp.heads = h->cfg.heads;
  sp.batch = h->cfg.batch;
  sp.err = h->err;
  sp.wait_limit_ns = h->wait_ns;
  ARL2_TRY(launch_readout_prep(h->tm_s_bf, h->tm_phiq, sp, h->cfg.batch, st));
  return ARL2_OK;
}

// inter = false: the intra-frame branch alone (the token-level calls add
// their own read-out afterwards).
arl2_status run_attention(arl2_state* h, const void* q, const void* k, const void* v, void* o, cudaStream_t st,
                          int64_t ld = 0, bool inter = true) {
  const arl2_config& c = h->cfg;
  if (c.dtype == ARL2_F32) {
    F32AttnParams p{};
    p.q = static_cast<const float*>(q);
    p.k = static_cast<const float*>(k);
    p.v = static_cast<const float*>(v);
    p.o = static_cast<float*>(o);
    p.phi_q = static_cast<const float*>(h->phi[0]);
    p.S = h->S[h->cur];
    p.q_len = p.kv_len = p.kv_stride = c.tokens_per_frame;
    p.heads = c.heads;
    p.d = c.head_dim;
    p.scale = h->scale;
    p.flags = c.flags;
    ARL2_TRY(launch_f32_attn(p, c.batch, st));
    return ARL2_OK;
  }
  CUtensorMap tq, tk, tv, to;
  if (!make_act_map(&tq, q, c.batch, c.tokens_per_frame, c.heads, 128, ld) ||
      !make_act_map(&tk, k, c.batch, c.tokens_per_frame, c.heads, 64, ld) ||
      !make_act_map(&tv, v, c.batch, c.tokens_per_frame, c.heads, 128, ld) ||
      !make_act_map(&to, o, c.batch, c.tokens_per_frame, c.heads, 32))
    return ARL2_ERR_CUDA;
  AttnParams p{};
  p.q_len = p.kv_len = c.tokens_per_frame;
  p.heads = c.heads;
  p.scale_log2 = h->scale * 1.4426950408889634f;
  p.flags = c.flags;
  p.has_inter = inter ? 1 : 0;
  p.scratch = h->attn_scratch;
  p.ready = h->attn_ready;
  p.err = h->err;
  p.wait_limit_ns = h->wait_ns;
  if (!attn_pair_partition(p, c.batch, h->pairs)) return ARL2_ERR_UNSUPPORTED;
  ARL2_TRY(launch_attn_pair(tq, tk, tv, h->tm_mqt64[h->cur], to, p, st));
  return ARL2_OK;
}

// [a, a + na) and [b, b + nb) share a byte.
bool overlaps2(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

arl2_status check_io(const arl2_config& c, const void* q, const void* k, const void* v, const void* o,
                     int64_t ld = 0) {
  if (!q || !k || !v || !o) return ARL2_ERR_INVALID_ARGUMENT;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return ARL2_ERR_INVALID_ARGUMENT;
  const size_t esz = c.dtype == ARL2_F32 ? 4 : 2;
  const size_t rows = size_t(c.batch) * c.tokens_per_frame, row = size_t(c.heads) * c.head_dim;
  const size_t n = rows * row * esz;
  // a strided view spans (rows - 1) pitches plus one row
  const size_t n_in = ld > 0 ? ((rows - 1) * size_t(ld) + row) * esz : n;
  auto clash = [&](const void* in) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(o), b = reinterpret_cast<uintptr_t>(in);
    return a < b + n_in && b < a + n;
  };
  if (clash(q) || clash(k) || clash(v)) return ARL2_ERR_INVALID_ARGUMENT;
  return ARL2_OK;
}

}  // namespace

extern "C" {

const char* arl2_status_string(arl2_status s) {
  switch (s) {
    case ARL2_OK: return "ok";
    case ARL2_ERR_INVALID_ARGUMENT: return "invalid argument";
    case ARL2_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case ARL2_ERR_OUT_OF_MEMORY: return "out of device memory";
    case ARL2_ERR_CUDA: return "CUDA error";
    case ARL2_ERR_TIMEOUT: return "device-side wait timed out";
    case ARL2_ERR_NO_DEVICE: return "no CUDA device";
    case ARL2_ERR_SCRATCH_LIMIT: return "sizes exceed the fixed scratch of the allocation-free state write";
    case ARL2_ERR_BOUNDS: return "a kernel index check failed (debug build)";
  }
  return "unknown status";
}

int32_t arl2_abi_version(void) { return 1; }

int32_t arl2_debug_bounds_enabled(void) {
#ifdef ARL2_DEBUG_BOUNDS
  return 1;
#else
  return 0;
#endif
}

arl2_status arl2_state_init(const arl2_config* cfg, const void* phi_q, const void* phi_k, const void* phi_v,
                            void* stream, arl2_state_t* out) {
  if (!out) return ARL2_ERR_INVALID_ARGUMENT;
  *out = nullptr;
  arl2_status s = check_config(cfg);
  if (s != ARL2_OK) return s;
  if (!phi_q || !phi_k || !phi_v || !aligned16(phi_q) || !aligned16(phi_k) || !aligned16(phi_v))
    return ARL2_ERR_INVALID_ARGUMENT;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ARL2_ERR_NO_DEVICE;
  if (cfg->dtype == ARL2_BF16 && !encode_fn()) return ARL2_ERR_NO_DEVICE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  arl2_state* h = new (std::nothrow) arl2_state();
  if (!h) return ARL2_ERR_OUT_OF_MEMORY;
  h->cfg = *cfg;
  h->device = dev;
  h->scale = softmax_scale(*cfg);
  h->corr = cfg->corr_scale < 0.f ? 1.f / float(cfg->tokens_per_frame) : cfg->corr_scale;
  h->wait_ns = kDefaultWaitNs;
  h->last_stream = st;
  const int B = cfg->batch, H = cfg->heads, d = cfg->head_dim;
  const size_t esz = cfg->dtype == ARL2_F32 ? 4 : 2;
  const size_t phi_bytes = size_t(H) * d * d * esz;
  const size_t s_bytes = size_t(B) * H * d * d * sizeof(float);
  h->n_chunks = (cfg->tokens_per_frame + 127) / 128;
  cudaError_t e = cudaSuccess;
  auto alloc = [&](void** p, size_t n) {
    if (e == cudaSuccess) {
      e = dev_alloc(p, n);
      if (e == cudaSuccess) h->bytes += int64_t(n);
    }
  };
  for (int i = 0; i < 3; ++i) alloc(&h->phi[i], phi_bytes);
  alloc(reinterpret_cast<void**>(&h->S[0]), s_bytes);
  alloc(reinterpret_cast<void**>(&h->S[1]), s_bytes);
  alloc(reinterpret_cast<void**>(&h->err), 256);
  if (cfg->dtype == ARL2_BF16) {
    if (cudaDeviceGetAttribute(&h->sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || h->sms < 1) h->sms = 1;
    h->pairs = std::min(h->sms / 2, attn_pair_capacity());
    h->state_fused = state_fused_supported(h->n_chunks, H, B);
    alloc(reinterpret_cast<void**>(&h->attn_scratch), attn_scratch_floats(h->sms) * sizeof(float));
    alloc(reinterpret_cast<void**>(&h->attn_ready), attn_ready_words(h->sms) * sizeof(unsigned));
    alloc(reinterpret_cast<void**>(&h->S_bf), size_t(B) * H * d * d * 2);
    alloc(reinterpret_cast<void**>(&h->mqt), 2 * size_t(B) * H * d * d * 2);
    alloc(reinterpret_cast<void**>(&h->partial), size_t(B) * H * h->n_chunks * d * d * sizeof(float));
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&h->side, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&h->ev_fork, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&h->ev_join, cudaEventDisableTiming);
  }
  if (e != cudaSuccess) {
    free_state(h);
    return from_cuda(e);
  }
  const void* src[3] = {phi_q, phi_k, phi_v};
  if (cfg->dtype == ARL2_F32) {
    for (int i = 0; i < 3 && e == cudaSuccess; ++i)
      e = cudaMemcpyAsync(h->phi[i], src[i], phi_bytes, cudaMemcpyDeviceToDevice, st);
  } else {
    e = cudaMemcpyAsync(h->phi[0], phi_q, phi_bytes, cudaMemcpyDeviceToDevice, st);
    if (e == cudaSuccess)
      e = launch_transpose_bf16(static_cast<const __nv_bfloat16*>(phi_k), static_cast<__nv_bfloat16*>(h->phi[1]), H,
                                st);
    if (e == cudaSuccess)
      e = launch_transpose_bf16(static_cast<const __nv_bfloat16*>(phi_v), static_cast<__nv_bfloat16*>(h->phi[2]), H,
                                st);
  }
  if (e == cudaSuccess) e = cudaMemsetAsync(h->S[0], 0, s_bytes, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(h->S[1], 0, s_bytes, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(h->err, 0, 256, st);
  if (cfg->dtype == ARL2_BF16) {
    if (e == cudaSuccess) e = cudaMemsetAsync(h->S_bf, 0, size_t(B) * H * d * d * 2, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(h->mqt, 0, 2 * size_t(B) * H * d * d * 2, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(h->attn_ready, 0, attn_ready_words(h->sms) * sizeof(unsigned), st);
    if (e == cudaSuccess &&
        !(make_mat_map(&h->tm_phiq, h->phi[0], H) && make_mat_map(&h->tm_phik_t, h->phi[1], H) &&
          make_mat_map(&h->tm_phiv_t, h->phi[2], H) && make_mat_map(&h->tm_s_bf, h->S_bf, B * H) &&
          make_mat_map(&h->tm_mqt[0], mqt_slot(h, 0), B * H) && make_mat_map(&h->tm_mqt[1], mqt_slot(h, 1), B * H) &&
          make_mat_map(&h->tm_mqt64[0], mqt_slot(h, 0), B * H, 64) &&
          make_mat_map(&h->tm_mqt64[1], mqt_slot(h, 1), B * H, 64)))
      e = cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) {
    free_state(h);
    return from_cuda(e);
  }
  h->magic = kStateMagic;
  {
    std::lock_guard<std::mutex> g(g_mu);
    g_live.insert(h);
  }
  if (log_enabled())
    std::fprintf(stderr, "[arl2] state_init B=%d H=%d d=%d L=%d dtype=%d bytes=%lld\n", B, H, d,
                 cfg->tokens_per_frame, cfg->dtype, (long long)h->bytes);
  *out = h;
  return ARL2_OK;
}

arl2_status arl2_frame_query(arl2_state_t h, const void* q, const void* k, const void* v, void* o, void* stream) {
  return arl2::layer_query_ld(h, q, k, v, 0, o, static_cast<cudaStream_t>(stream));
}

arl2_status arl2_frame_commit(arl2_state_t h, const void* q, const void* k, const void* v, const float* alpha,
                              const float* beta, void* o, void* stream) {
  return arl2::layer_commit_ld(h, q, k, v, 0, alpha, beta, o, static_cast<cudaStream_t>(stream));
}

arl2_status arl2_frame_query_strided(arl2_state_t h, const void* q, const void* k, const void* v, int64_t ld,
                                     void* o, void* stream) {
  if (ld < 0) return ARL2_ERR_INVALID_ARGUMENT;
  return arl2::layer_query_ld(h, q, k, v, ld, o, static_cast<cudaStream_t>(stream));
}

arl2_status arl2_frame_commit_strided(arl2_state_t h, const void* q, const void* k, const void* v, int64_t ld,
                                      const float* alpha, const float* beta, void* o, void* stream) {
  if (ld < 0) return ARL2_ERR_INVALID_ARGUMENT;
  return arl2::layer_commit_ld(h, q, k, v, ld, alpha, beta, o, static_cast<cudaStream_t>(stream));
}

arl2_status arl2_token_query(arl2_state_t h, const void* q, const void* k, const void* v, const float* alpha_tok,
                             const float* beta, void* o, void* stream) {
  return arl2::token_pass(h, q, k, v, alpha_tok, beta, o, static_cast<cudaStream_t>(stream), false);
}

arl2_status arl2_token_commit(arl2_state_t h, const void* q, const void* k, const void* v, const float* alpha_tok,
                              const float* beta, void* o, void* stream) {
  return arl2::token_pass(h, q, k, v, alpha_tok, beta, o, static_cast<cudaStream_t>(stream), true);
}

}  // extern "C"

namespace arl2 {

arl2_status layer_query_ld(arl2_state* h, const void* q, const void* k, const void* v, int64_t ld, void* o,
                           cudaStream_t st) {
  if (!live(h, kStateMagic)) return ARL2_ERR_INVALID_ARGUMENT;
  if (ld != 0 && (h->cfg.dtype != ARL2_BF16 || ld < int64_t(h->cfg.heads) * 128 || ld % 8 != 0))
    return ARL2_ERR_INVALID_ARGUMENT;
  arl2_status s = check_io(h->cfg, q, k, v, o, ld);
  if (s != ARL2_OK) return s;
  h->last_stream = st;
  return run_attention(h, q, k, v, o, st, ld);
}

arl2_status layer_commit_ld(arl2_state* h, const void* q, const void* k, const void* v, int64_t ld, const float* alpha,
                            const float* beta, void* o, cudaStream_t st) {
  if (!live(h, kStateMagic)) return ARL2_ERR_INVALID_ARGUMENT;
  if (ld != 0 && (h->cfg.dtype != ARL2_BF16 || ld < int64_t(h->cfg.heads) * 128 || ld % 8 != 0))
    return ARL2_ERR_INVALID_ARGUMENT;
  arl2_status s = check_io(h->cfg, q, k, v, o, ld);
  if (s != ARL2_OK) return s;
  if (!alpha || !beta || !aligned16(alpha) || !aligned16(beta)) return ARL2_ERR_INVALID_ARGUMENT;
  h->last_stream = st;
  const bool fork = h->cfg.dtype == ARL2_BF16;
  // The state write needs nothing from the output's attention launch and
  // writes nothing it reads (S_N, its bf16 copy and MqT go to the other slots):
  // its three kernels run on the side stream, forked before that launch, so
  // that their CTAs take the SMs the attention launch frees in its tail; the
  // caller's stream joins them before its next work.
  if (fork) ARL2_TRY(cudaEventRecord(h->ev_fork, st));
  s = run_attention(h, q, k, v, o, st, ld);  // the output reads S_{N-1}
  if (s != ARL2_OK) return s;
  const arl2_config& c = h->cfg;
  const int nxt = h->cur ^ 1;
  if (c.dtype == ARL2_F32) {
    F32CommitParams p{};
    p.k = static_cast<const float*>(k);
    p.v = static_cast<const float*>(v);
    p.phi_k = static_cast<const float*>(h->phi[1]);
    p.phi_v = static_cast<const float*>(h->phi[2]);
    p.S_prev = h->S[h->cur];
    p.S_next = h->S[nxt];
    p.alpha = alpha;
    p.beta = beta;
    p.L = c.tokens_per_frame;
    p.heads = c.heads;
    p.d = c.head_dim;
    p.corr = h->corr;
    ARL2_TRY(launch_f32_commit(p, c.batch, st));
  } else {
    CUtensorMap tk, tv;
    if (!make_act_map(&tk, k, c.batch, c.tokens_per_frame, c.heads, 128, ld) ||
        !make_act_map(&tv, v, c.batch, c.tokens_per_frame, c.heads, 128, ld))
      return ARL2_ERR_CUDA;
    StateParams sp{};
    sp.S_prev = h->S[h->cur];
    sp.alpha = alpha;
    sp.beta = beta;
    sp.partial = h->partial;
    sp.S_next = h->S[nxt];
    sp.S_next_bf = h->S_bf;
    sp.mqt = mqt_slot(h, nxt);
    sp.L = c.tokens_per_frame;
    sp.heads = c.heads;
    sp.batch = c.batch;
    sp.n_chunks = h->n_chunks;
    sp.corr = h->corr;
    sp.err = h->err;
    sp.wait_limit_ns = h->wait_ns;
    ARL2_TRY(cudaStreamWaitEvent(h->side, h->ev_fork, 0));
    if (h->state_fused) {  // one launch: partials reduced on chip, MqT formed by each cluster's rank 0
      ARL2_TRY(launch_state_fused(tk, tv, h->tm_phik_t, h->tm_phiv_t, h->tm_s_bf, h->tm_phiq, sp, c.batch,
                                  h->side));
    } else {
      ARL2_TRY(launch_state_partial(tk, tv, h->tm_phik_t, h->tm_phiv_t, h->tm_s_bf, sp, c.batch, h->side));
      ARL2_TRY(launch_state_finalize(sp, c.batch, h->side));
      ARL2_TRY(launch_readout_prep(h->tm_s_bf, h->tm_phiq, sp, c.batch, h->side));
    }
    ARL2_TRY(cudaEventRecord(h->ev_join, h->side));
    ARL2_TRY(cudaStreamWaitEvent(st, h->ev_join, 0));
  }
  h->cur = nxt;
  h->frame += 1;
  return ARL2_OK;
}

uint32_t* layer_error_word(arl2_state* h) { return h->err; }
uint64_t layer_wait_limit(arl2_state* h) { return h->wait_ns; }

arl2_status token_pass(arl2_state* h, const void* q, const void* k, const void* v, const float* alpha_tok,
                       const float* beta, void* o, cudaStream_t st, bool commit) {
  if (!live(h, kStateMagic)) return ARL2_ERR_INVALID_ARGUMENT;
  const arl2_config& c = h->cfg;
  if (c.dtype != ARL2_BF16) return ARL2_ERR_UNSUPPORTED;
  arl2_status s = check_io(c, q, k, v, o);
  if (s != ARL2_OK) return s;
  if (!alpha_tok || !beta || !aligned16(alpha_tok) || !aligned16(beta)) return ARL2_ERR_INVALID_ARGUMENT;
  if (!h->tok) {
    const size_t n = token_scratch_floats(c.batch, c.heads, c.tokens_per_frame) * sizeof(float);
    void* mem = nullptr;
    const cudaError_t e = cudaMalloc(&mem, n);
    if (e != cudaSuccess) {  // out of memory, or (say) an allocation inside a stream capture
      cudaGetLastError();
      return from_cuda(e);
    }
    h->tok = static_cast<float*>(mem);
    h->bytes += int64_t(n);
  }
  h->last_stream = st;
  s = run_attention(h, q, k, v, o, st, 0, false);  // the intra-frame branch into o
  if (s != ARL2_OK) return s;
  const int nxt = h->cur ^ 1;
  TokenParams p{};
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k = static_cast<const __nv_bfloat16*>(k);
  p.v = static_cast<const __nv_bfloat16*>(v);
  p.phi_q = static_cast<const __nv_bfloat16*>(h->phi[0]);
  p.phi_k_t = static_cast<const __nv_bfloat16*>(h->phi[1]);
  p.phi_v_t = static_cast<const __nv_bfloat16*>(h->phi[2]);
  p.alpha_tok = alpha_tok;
  p.beta = beta;
  p.corr = h->corr;
  p.B = c.batch;
  p.L = c.tokens_per_frame;
  p.H = c.heads;
  p.n_chunks = h->n_chunks;
  token_bind_scratch(p, h->tok);
  p.s_in = h->S[h->cur];
  p.s_out = commit ? h->S[nxt] : nullptr;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.err = h->err;
  p.wait_limit_ns = h->wait_ns;
  ARL2_TRY(launch_token_level(p, !(c.flags & ARL2_INTRA_ONLY), st));
  if (commit) {  // S_N becomes the current state; its bf16 copy and read-out operand follow it
    h->cur = nxt;
    ARL2_TRY(launch_to_bf16(h->S[h->cur], h->S_bf, size_t(c.batch) * c.heads * 128 * 128, st));
    s = prepare_readout(h, st);
    if (s != ARL2_OK) return s;
    h->frame += 1;
  }
  return ARL2_OK;
}

}  // namespace arl2

extern "C" {

arl2_status arl2_state_get(arl2_state_t h, float* dst, int64_t* frame, void* stream) {
  if (!live(h, kStateMagic)) return ARL2_ERR_INVALID_ARGUMENT;
  if (frame) *frame = h->frame;
  if (!dst) return frame ? ARL2_OK : ARL2_ERR_INVALID_ARGUMENT;
  const arl2_config& c = h->cfg;
  const size_t n = size_t(c.batch) * c.heads * c.head_dim * c.head_dim * sizeof(float);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  h->last_stream = st;
  ARL2_TRY(cudaMemcpyAsync(dst, h->S[h->cur], n, cudaMemcpyDeviceToDevice, st));
  return ARL2_OK;
}

arl2_status arl2_state_set(arl2_state_t h, const float* src, int64_t frame, void* stream) {
  if (!live(h, kStateMagic)) return ARL2_ERR_INVALID_ARGUMENT;
  if (!src || frame < 0 || !aligned16(src)) return ARL2_ERR_INVALID_ARGUMENT;
  const arl2_config& c = h->cfg;
  const size_t cnt = size_t(c.batch) * c.heads * c.head_dim * c.head_dim;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  h->last_stream = st;
  ARL2_TRY(cudaMemcpyAsync(h->S[h->cur], src, cnt * sizeof(float), cudaMemcpyDeviceToDevice, st));
  if (c.dtype == ARL2_BF16) {
    ARL2_TRY(launch_to_bf16(h->S[h->cur], h->S_bf, cnt, st));
    arl2_status s = prepare_readout(h, st);
    if (s != ARL2_OK) return s;
  }
  h->frame = frame;
  return ARL2_OK;
}

arl2_status arl2_last_error(arl2_state_t h) {
  if (!live(h, kStateMagic)) return ARL2_ERR_INVALID_ARGUMENT;
  ARL2_TRY(cudaStreamSynchronize(h->last_stream));
  uint32_t w = 0;
  ARL2_TRY(cudaMemcpy(&w, h->err, sizeof(w), cudaMemcpyDeviceToHost));
  if (w) {
    // a kernel that gave up may have left partial-ready flags raised
    ARL2_TRY(cudaMemset(h->err, 0, sizeof(w)));
    if (h->attn_ready) ARL2_TRY(cudaMemset(h->attn_ready, 0, attn_ready_words(h->sms) * sizeof(unsigned)));
  }
  return static_cast<arl2_status>(w);
}

int64_t arl2_state_device_bytes(arl2_state_t h) { return live(h, kStateMagic) ? h->bytes : -1; }

arl2_status arl2_state_set_wait_limit(arl2_state_t h, uint64_t limit_ns) {
  if (!live(h, kStateMagic)) return ARL2_ERR_INVALID_ARGUMENT;
  h->wait_ns = limit_ns ? limit_ns : kDefaultWaitNs;
  return ARL2_OK;
}

arl2_status arl2_state_destroy(arl2_state_t h) {
  if (!live(h, kStateMagic)) return ARL2_ERR_INVALID_ARGUMENT;
  {
    std::lock_guard<std::mutex> g(g_mu);
    g_live.erase(h);
  }
  cudaStreamSynchronize(h->last_stream);
  free_state(h);
  return ARL2_OK;
}

// ---------------------------------------------------------------- KV-cache layers
arl2_status arl2_kv_init(const arl2_config* cfg, int32_t max_frames, void* stream, arl2_kv_t* out) {
  if (!out) return ARL2_ERR_INVALID_ARGUMENT;
  *out = nullptr;
  arl2_status s = check_config(cfg);
  if (s != ARL2_OK) return s;
  if (max_frames < 1) return ARL2_ERR_INVALID_ARGUMENT;
  const int64_t tokens = int64_t(max_frames) * cfg->tokens_per_frame;
  if (cfg->dtype == ARL2_BF16 && tokens > (int64_t(1) << 31)) return ARL2_ERR_UNSUPPORTED;
  if (cfg->dtype == ARL2_F32 && tokens > (int64_t(1) << 31)) return ARL2_ERR_UNSUPPORTED;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ARL2_ERR_NO_DEVICE;
  if (cfg->dtype == ARL2_BF16 && !encode_fn()) return ARL2_ERR_NO_DEVICE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  arl2_kv* h = new (std::nothrow) arl2_kv();
  if (!h) return ARL2_ERR_OUT_OF_MEMORY;
  h->cfg = *cfg;
  h->device = dev;
  h->scale = softmax_scale(*cfg);
  h->wait_ns = kDefaultWaitNs;
  h->max_frames = max_frames;
  h->last_stream = st;
  const size_t esz = cfg->dtype == ARL2_F32 ? 4 : 2;
  const size_t bytes = size_t(cfg->batch) * size_t(tokens) * cfg->heads * cfg->head_dim * esz;
  if (cudaDeviceGetAttribute(&h->sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || h->sms < 1) h->sms = 1;
  h->pairs = cfg->dtype == ARL2_BF16 ? std::min(h->sms / 2, attn_pair_capacity()) : 0;
  const size_t scratch_bytes = attn_scratch_floats(h->sms) * sizeof(float);
  const size_t ready_bytes = attn_ready_words(h->sms) * sizeof(unsigned);
  cudaError_t e = dev_alloc(&h->kc, bytes);
  if (e == cudaSuccess) e = dev_alloc(&h->vc, bytes);
  if (e == cudaSuccess && cfg->dtype == ARL2_BF16) e = dev_alloc(reinterpret_cast<void**>(&h->attn_scratch), scratch_bytes);
  if (e == cudaSuccess && cfg->dtype == ARL2_BF16) e = dev_alloc(reinterpret_cast<void**>(&h->attn_ready), ready_bytes);
  if (e == cudaSuccess && cfg->dtype == ARL2_BF16) e = cudaMemsetAsync(h->attn_ready, 0, ready_bytes, st);
  if (e == cudaSuccess) e = dev_alloc(reinterpret_cast<void**>(&h->err), 256);
  if (e == cudaSuccess) e = cudaMemsetAsync(h->kc, 0, bytes, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(h->vc, 0, bytes, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(h->err, 0, 256, st);
  if (e != cudaSuccess) {
    free_kv(h);
    return from_cuda(e);
  }
  h->bytes = int64_t(2 * bytes + 256) + (cfg->dtype == ARL2_BF16 ? int64_t(scratch_bytes + ready_bytes) : 0);
  h->magic = kKvMagic;
  {
    std::lock_guard<std::mutex> g(g_mu);
    g_live.insert(h);
  }
  *out = h;
  return ARL2_OK;
}

namespace {

// Copy this pass's K and V into cache slot `frames` (the slot after the
// committed frames), then attend over frames 0..frames of the cache.
arl2_status kv_pass(arl2_kv* h, const void* q, const void* k, const void* v, void* o, cudaStream_t st,
                    int64_t ld = 0) {
  const arl2_config& c = h->cfg;
  if (h->frames >= h->max_frames) return ARL2_ERR_INVALID_ARGUMENT;
  const size_t esz = c.dtype == ARL2_F32 ? 4 : 2;
  const size_t row_bytes = size_t(c.heads) * c.head_dim * esz;
  const size_t frame_bytes = size_t(c.tokens_per_frame) * row_bytes;
  const size_t stream_bytes = frame_bytes * size_t(h->max_frames);
  char* kc = static_cast<char*>(h->kc);
  char* vc = static_cast<char*>(h->vc);
  if (ld == 0) {  // one copy per tensor: B frames of contiguous rows
    ARL2_TRY(cudaMemcpy2DAsync(kc + frame_bytes * h->frames, stream_bytes, k, frame_bytes, frame_bytes, c.batch,
                               cudaMemcpyDeviceToDevice, st));
    ARL2_TRY(cudaMemcpy2DAsync(vc + frame_bytes * h->frames, stream_bytes, v, frame_bytes, frame_bytes, c.batch,
                               cudaMemcpyDeviceToDevice, st));
  } else {  // one copy per stream and tensor: L token rows `ld` elements apart
    const size_t pitch = size_t(ld) * esz;
    for (int b = 0; b < c.batch; ++b) {
      const size_t src_off = size_t(b) * c.tokens_per_frame * pitch;
      ARL2_TRY(cudaMemcpy2DAsync(kc + stream_bytes * b + frame_bytes * h->frames, row_bytes,
                                 static_cast<const char*>(k) + src_off, pitch, row_bytes, c.tokens_per_frame,
                                 cudaMemcpyDeviceToDevice, st));
      ARL2_TRY(cudaMemcpy2DAsync(vc + stream_bytes * b + frame_bytes * h->frames, row_bytes,
                                 static_cast<const char*>(v) + src_off, pitch, row_bytes, c.tokens_per_frame,
                                 cudaMemcpyDeviceToDevice, st));
    }
  }
  const int64_t kv_tokens = int64_t(h->frames + 1) * c.tokens_per_frame;
  const int64_t stride_tokens = int64_t(h->max_frames) * c.tokens_per_frame;
  if (c.dtype == ARL2_F32) {
    F32AttnParams p{};
    p.q = static_cast<const float*>(q);
    p.k = static_cast<const float*>(h->kc);
    p.v = static_cast<const float*>(h->vc);
    p.o = static_cast<float*>(o);
    p.phi_q = nullptr;
    p.S = nullptr;
    p.q_len = c.tokens_per_frame;
    p.kv_len = int(kv_tokens);
    p.kv_stride = int(stride_tokens);
    p.heads = c.heads;
    p.d = c.head_dim;
    p.scale = h->scale;
    p.flags = 0;
    ARL2_TRY(launch_f32_attn(p, c.batch, st));
    return ARL2_OK;
  }
  CUtensorMap tq, tk, tv, to;
  if (!make_act_map(&tq, q, c.batch, c.tokens_per_frame, c.heads, 128, ld) ||
      !make_act_map(&tk, h->kc, c.batch, stride_tokens, c.heads, 64) ||
      !make_act_map(&tv, h->vc, c.batch, stride_tokens, c.heads, 128) ||
      !make_act_map(&to, o, c.batch, c.tokens_per_frame, c.heads, 32))
    return ARL2_ERR_CUDA;
  AttnParams p{};
  p.q_len = c.tokens_per_frame;
  p.kv_len = int(kv_tokens);
  p.heads = c.heads;
  p.scale_log2 = h->scale * 1.4426950408889634f;
  p.flags = 0;
  p.has_inter = 0;
  p.scratch = h->attn_scratch;
  p.ready = h->attn_ready;
  p.err = h->err;
  p.wait_limit_ns = h->wait_ns;
  if (!attn_pair_partition(p, c.batch, h->pairs)) return ARL2_ERR_UNSUPPORTED;
  ARL2_TRY(launch_attn_pair(tq, tk, tv, tq, to, p, st));
  return ARL2_OK;
}

}  // namespace

arl2_status arl2_kv_query(arl2_kv_t h, const void* q, const void* k, const void* v, void* o, void* stream) {
  if (!live(h, kKvMagic)) return ARL2_ERR_INVALID_ARGUMENT;
  arl2_status s = check_io(h->cfg, q, k, v, o);
  if (s != ARL2_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  h->last_stream = st;
  return kv_pass(h, q, k, v, o, st);
}

arl2_status arl2_kv_commit(arl2_kv_t h, const void* q, const void* k, const void* v, void* o, void* stream) {
  if (!live(h, kKvMagic)) return ARL2_ERR_INVALID_ARGUMENT;
  arl2_status s = check_io(h->cfg, q, k, v, o);
  if (s != ARL2_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  h->last_stream = st;
  s = kv_pass(h, q, k, v, o, st);
  if (s == ARL2_OK) h->frames += 1;
  return s;
}

arl2_status arl2_kv_query_strided(arl2_kv_t h, const void* q, const void* k, const void* v, int64_t ld, void* o,
                                  void* stream) {
  if (!live(h, kKvMagic)) return ARL2_ERR_INVALID_ARGUMENT;
  if (ld < 0 || (ld != 0 && (h->cfg.dtype != ARL2_BF16 || ld < int64_t(h->cfg.heads) * h->cfg.head_dim || ld % 8 != 0)))
    return ARL2_ERR_INVALID_ARGUMENT;
  arl2_status s = check_io(h->cfg, q, k, v, o, ld);
  if (s != ARL2_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  h->last_stream = st;
  return kv_pass(h, q, k, v, o, st, ld);
}

arl2_status arl2_kv_commit_strided(arl2_kv_t h, const void* q, const void* k, const void* v, int64_t ld, void* o,
                                   void* stream) {
  if (!live(h, kKvMagic)) return ARL2_ERR_INVALID_ARGUMENT;
  if (ld < 0 || (ld != 0 && (h->cfg.dtype != ARL2_BF16 || ld < int64_t(h->cfg.heads) * h->cfg.head_dim || ld % 8 != 0)))
    return ARL2_ERR_INVALID_ARGUMENT;
  arl2_status s = check_io(h->cfg, q, k, v, o, ld);
  if (s != ARL2_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  h->last_stream = st;
  s = kv_pass(h, q, k, v, o, st, ld);
  if (s == ARL2_OK) h->frames += 1;
  return s;
}

int64_t arl2_kv_frames(arl2_kv_t h) { return live(h, kKvMagic) ? h->frames : -1; }
int64_t arl2_kv_device_bytes(arl2_kv_t h) { return live(h, kKvMagic) ? h->bytes : -1; }

arl2_status arl2_kv_last_error(arl2_kv_t h) {
  if (!live(h, kKvMagic)) return ARL2_ERR_INVALID_ARGUMENT;
  ARL2_TRY(cudaStreamSynchronize(h->last_stream));
  uint32_t w = 0;
  ARL2_TRY(cudaMemcpy(&w, h->err, sizeof(w), cudaMemcpyDeviceToHost));
  if (w) {
    // a kernel that gave up may have left partial-ready flags raised
    ARL2_TRY(cudaMemset(h->err, 0, sizeof(w)));
    if (h->attn_ready) ARL2_TRY(cudaMemset(h->attn_ready, 0, attn_ready_words(h->sms) * sizeof(unsigned)));
  }
  return static_cast<arl2_status>(w);
}

arl2_status arl2_kv_destroy(arl2_kv_t h) {
  if (!live(h, kKvMagic)) return ARL2_ERR_INVALID_ARGUMENT;
  {
    std::lock_guard<std::mutex> g(g_mu);
    g_live.erase(h);
  }
  cudaStreamSynchronize(h->last_stream);
  free_kv(h);
  return ARL2_OK;
}

arl2_status arl2_selftest_wait_timeout(uint64_t limit_ns, void* stream) {
  if (limit_ns == 0 || limit_ns > 10000000000ull) return ARL2_ERR_INVALID_ARGUMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t* err = nullptr;
  ARL2_TRY(dev_alloc(reinterpret_cast<void**>(&err), sizeof(uint32_t)));
  cudaError_t e = cudaMemsetAsync(err, 0, sizeof(uint32_t), st);
  if (e == cudaSuccess) e = launch_wait_selftest(err, limit_ns, st);
  uint32_t w = 0;
  if (e == cudaSuccess) e = cudaMemcpyAsync(&w, err, sizeof(uint32_t), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  cudaFree(err);
  if (e != cudaSuccess) return from_cuda(e);
  return static_cast<arl2_status>(w);
}

arl2_status arl2_attn_partition(int batch, int heads, int q_len, int kv_len, int pairs, int32_t* segs, int max_segs,
                                int32_t* seg_first, int* n_segs, int* n_pairs) {
  if (!segs || !seg_first || !n_segs || !n_pairs || batch < 1 || heads < 1 || q_len < 1 || kv_len < 1 || pairs < 1 ||
      pairs > arl2::kAttnMaxGrid / 2 || max_segs < 1)
    return ARL2_ERR_INVALID_ARGUMENT;
  arl2::AttnParams p{};
  p.q_len = q_len;
  p.kv_len = kv_len;
  p.heads = heads;
  if (!arl2::attn_pair_partition(p, batch, pairs) || p.n_segs > max_segs) return ARL2_ERR_UNSUPPORTED;
  const int np = p.grid / 2;
  for (int c = 0; c <= np; ++c) seg_first[c] = int32_t(p.seg_first[c]);
  for (int i = 0; i < p.n_segs; ++i) {
    const uint2 e = p.seg[i];
    const int j0 = int((e.y >> 10) & 2047u);
    segs[5 * i + 0] = int32_t(e.x & 0x0FFFFFFFu);
    segs[5 * i + 1] = int32_t(e.y & 1023u);
    segs[5 * i + 2] = j0;
    segs[5 * i + 3] = j0 + int32_t(e.y >> 21);
    segs[5 * i + 4] = int32_t(e.x >> 28);
  }
  *n_segs = p.n_segs;
  *n_pairs = np;
  return ARL2_OK;
}

arl2_status arl2_gemm_bf16(const void* a, int64_t lda, const void* b, int64_t ldb, void* c, int64_t ldc, int64_t m,
                           int64_t n, int64_t k, void* stream) {
  if (!a || !b || !c || !aligned16(a) || !aligned16(b) || !aligned16(c)) return ARL2_ERR_INVALID_ARGUMENT;
  if (m < 0 || n < 0 || k < 0 || m > (1 << 30) || n > (1 << 30) || k > (1 << 30)) return ARL2_ERR_INVALID_ARGUMENT;
  if (lda < k || ldb < n || ldc < n || lda % 8 || ldb % 8 || ldc % 8) return ARL2_ERR_INVALID_ARGUMENT;
  if (m == 0 || n == 0) return ARL2_OK;
  const size_t nc = (size_t(m - 1) * size_t(ldc) + size_t(n)) * 2;
  if (overlaps2(c, nc, a, (size_t(m - 1) * size_t(lda) + size_t(k)) * 2) ||
      overlaps2(c, nc, b, (size_t(k > 0 ? k - 1 : 0) * size_t(ldb) + size_t(n)) * 2))
    return ARL2_ERR_INVALID_ARGUMENT;
  if (!encode_fn()) return ARL2_ERR_NO_DEVICE;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return ARL2_ERR_NO_DEVICE;
  GemmParams p{};
  p.M = int(m);
  p.N = int(n);
  p.K = int(k);
  p.err = nullptr;
  p.wait_limit_ns = kDefaultWaitNs;
  ARL2_TRY(gemm_bf16(a, lda, b, ldb, c, ldc, p, sms, static_cast<cudaStream_t>(stream)));
  return ARL2_OK;
}

arl2_status arl2_selftest_exp2(const float* x, float* y, int64_t n, void* stream) {
  if (!x || !y || n < 0) return ARL2_ERR_INVALID_ARGUMENT;
  if (n == 0) return ARL2_OK;
  ARL2_TRY(launch_exp2_poly(x, y, n, static_cast<cudaStream_t>(stream)));
  return ARL2_OK;
}

}  // extern "C"

// ---------------------------------------------------------------- state write without allocation
// For callers that must not allocate device memory (inside a stream capture,
// under a fixed memory budget, or beside a runtime that owns the allocator),
// arl2_state_write_noalloc runs the commit's state-write kernels with their
// work space in this static array instead of cudaMalloc'd buffers.  The array
// is part of the library's device image: every GPU that loads the library
// holds it until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[ARL2_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_addr[kNoAllocMaxDevices] = {};

// Host code cannot use g_noalloc_scratch as a pointer: on the host the name is
// only a stand-in for the device symbol.  Look up its device address once per
// device, with that device current.
arl2_status noalloc_scratch(int dev, unsigned char** out) {
  if (dev < 0 || dev >= kNoAllocMaxDevices) return ARL2_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> g(g_noalloc_mu);
  if (!g_noalloc_addr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) return e != cudaSuccess ? from_cuda(e) : ARL2_ERR_CUDA;
    g_noalloc_addr[dev] = p;
  }
  *out = static_cast<unsigned char*>(g_noalloc_addr[dev]);
  return ARL2_OK;
}

size_t round_kib(size_t n) { return (n + 1023) & ~size_t(1023); }

}  // namespace

extern "C" arl2_status arl2_state_write_noalloc(const arl2_config* cfg, const void* k, const void* v,
                                                const void* phi_k, const void* phi_v, const float* S_prev,
                                                const float* alpha, const float* beta, float* S_next,
                                                uint32_t* dev_error, void* stream) {
  arl2_status s = check_config(cfg);
  if (s != ARL2_OK) return s;
  if (cfg->dtype != ARL2_BF16) return ARL2_ERR_UNSUPPORTED;
  const void* ptrs[] = {k, v, phi_k, phi_v, S_prev, alpha, beta, S_next, dev_error};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return ARL2_ERR_INVALID_ARGUMENT;
  const int B = cfg->batch, H = cfg->heads, L = cfg->tokens_per_frame;
  const size_t mat_bf = size_t(128) * 128 * 2;
  const size_t state_bytes = size_t(B) * H * 128 * 128 * sizeof(float);
  // The outputs (S_next, dev_error) may share no byte with any input or with
  // each other: the kernels read every input after the first output byte is
  // written.
  {
    const size_t act = size_t(B) * L * H * 128 * 2, phi = size_t(H) * 128 * 128 * 2;
    const struct { const void* p; size_t n; } in[] = {
        {k, act}, {v, act}, {phi_k, phi}, {phi_v, phi}, {S_prev, state_bytes},
        {alpha, size_t(B) * H * sizeof(float)}, {beta, size_t(B) * H * L * sizeof(float)}};
    for (const auto& r : in)
      if (overlaps2(S_next, state_bytes, r.p, r.n) || overlaps2(dev_error, sizeof(uint32_t), r.p, r.n))
        return ARL2_ERR_INVALID_ARGUMENT;
    if (overlaps2(S_next, state_bytes, dev_error, sizeof(uint32_t))) return ARL2_ERR_INVALID_ARGUMENT;
  }
  const int n_chunks = (L + 127) / 128;
  // Scratch layout: phi_k^T, phi_v^T [H,128,128] bf16; S_prev and S_next in
  // bf16 [B,H,128,128]; per-chunk partials [B,H,n_chunks,128,128] fp32.
  const size_t off_pk = 0;
  const size_t off_pv = off_pk + round_kib(size_t(H) * mat_bf);
  const size_t off_sb = off_pv + round_kib(size_t(H) * mat_bf);
  const size_t off_nb = off_sb + round_kib(size_t(B) * H * mat_bf);
  const size_t off_part = off_nb + round_kib(size_t(B) * H * mat_bf);
  const size_t need = off_part + round_kib(size_t(B) * H * n_chunks * 128 * 128 * sizeof(float));
  if (need > size_t(ARL2_NOALLOC_SCRATCH_BYTES)) return ARL2_ERR_SCRATCH_LIMIT;
  if (!encode_fn()) return ARL2_ERR_NO_DEVICE;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ARL2_ERR_NO_DEVICE;
  unsigned char* scratch = nullptr;
  s = noalloc_scratch(dev, &scratch);
  if (s != ARL2_OK) return s;
  auto* pk_t = reinterpret_cast<__nv_bfloat16*>(scratch + off_pk);
  auto* pv_t = reinterpret_cast<__nv_bfloat16*>(scratch + off_pv);
  auto* s_bf = reinterpret_cast<__nv_bfloat16*>(scratch + off_sb);
  auto* next_bf = reinterpret_cast<__nv_bfloat16*>(scratch + off_nb);
  auto* partial = reinterpret_cast<float*>(scratch + off_part);

  CUtensorMap tk, tv, tpk, tpv, ts;
  if (!make_act_map(&tk, k, B, L, H) || !make_act_map(&tv, v, B, L, H) || !make_mat_map(&tpk, pk_t, H) ||
      !make_mat_map(&tpv, pv_t, H) || !make_mat_map(&ts, s_bf, B * H))
    return ARL2_ERR_CUDA;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // Only the error word must start at zero: every other scratch byte the
  // kernels read is written earlier in this same call.
  ARL2_TRY(cudaMemsetAsync(dev_error, 0, sizeof(uint32_t), st));
  ARL2_TRY(launch_transpose_bf16(static_cast<const __nv_bfloat16*>(phi_k), pk_t, H, st));
  ARL2_TRY(launch_transpose_bf16(static_cast<const __nv_bfloat16*>(phi_v), pv_t, H, st));
  ARL2_TRY(launch_to_bf16(S_prev, s_bf, size_t(B) * H * 128 * 128, st));
  StateParams sp{};
  sp.S_prev = S_prev;
  sp.alpha = alpha;
  sp.beta = beta;
  sp.partial = partial;
  sp.S_next = S_next;
  sp.S_next_bf = next_bf;
  sp.mqt = nullptr;
  sp.L = L;
  sp.heads = H;
  sp.batch = B;
  sp.n_chunks = n_chunks;
  sp.corr = cfg->corr_scale < 0.f ? 1.f / float(L) : cfg->corr_scale;
  sp.err = dev_error;
  sp.wait_limit_ns = kDefaultWaitNs;
  ARL2_TRY(launch_state_partial(tk, tv, tpk, tpv, ts, sp, B, st));
  ARL2_TRY(launch_state_finalize(sp, B, st));
  return ARL2_OK;
}
