// Intra-frame softmax attention with the inter-frame read-out fused into its
// epilogue, on CTA pairs (tcgen05 cta_group::2), bf16 operands, fp32
// accumulation in tensor memory (sm_100a).
//
//   O = softmax(Q K^T * scale) V  +  Q MqT^T        (MqT = (phi_q S_{N-1})^T)
//
// The first term is the intra-frame branch (ARL2 summary, section 2.1: the
// original bidirectional softmax attention within each frame).  The second is
// the inter-frame read-out O_inter = Q' S_{N-1} = (Q phi_q) S_{N-1}, computed
// as Q (phi_q S_{N-1}), one extra 256 x 128 x 128 MMA per 256 query rows.
//
// Work decomposition.  A cluster of two CTAs owns a block of 256 query rows of
// one (stream, head): query tile 2b in rank 0, tile 2b + 1 in rank 1.  Every
// MMA covers both CTAs' rows (M = 256): rank 0 issues it, each CTA supplies
// its own 128 rows of the A operand and half of the B operand (64 keys of a K
// tile, 64 head dimensions of a V tile) and keeps its 128 rows of the
// accumulator in its own tensor memory.  S and P are double-buffered in tensor
// memory and S is issued two key tiles ahead of the PV that consumes the
// matching P, so the softmax of tile i finds S(i) ready as soon as it is done
// with tile i - 2: it never waits for a PV, and the tensor core never waits
// for the softmax of the tile it is about to compute.  The two softmax
// warpgroups take alternate key tiles of the same 128 rows (the running row
// max is handed from tile to tile through shared memory), so that one's waits
// hide behind the other's exponentials.  Each pair walks its own list of
// segments (a run of key tiles of one block), made on the host: whole blocks
// where the blocks divide evenly over the pairs, the rest cut into pieces
// (or plain equal ranges of the (block, key tile) sequence, "stream-K", when
// that costs less).  A block whose key range is split across pairs is
// finished by the pair holding its key tile 0 (always that pair's last
// segment); the pairs continuing it (their first segment, or on long key
// ranges their last) store their normalised partial output in bf16 with
// (m, l) in fp32 and raise ready flags, and the finishing pair combines the
// pieces in key order (deterministic).
//
// Roles per CTA (512 threads, four warpgroups):
//   warp 0       TMA producer: per segment the CTA's Q tile (two slots, so the
//                next segment's Q loads during the current one), then its
//                halves of K_j, V_j (and of MqT for blocks it finishes)
//                through a ring of 16 KB slots; the loads of both CTAs count
//                on rank 0's barriers;
//   warp 1       (rank 0 only) tcgen05 issuer of S(i) = Q K_i^T;
//   warp 2       tensor-memory allocator (both CTAs, cta_group::2);
//   warp 3       (rank 0 only) tcgen05 issuer of O += P(i) V_i and X = Q MqT^T;
//   warps 4..7   softmax of the even key tiles (one query row per thread);
//   warps 8..11  softmax of the odd key tiles;
//   warps 12..15 epilogue: at the end of a segment reads O (and X) from
//                tensor memory, hands it back at once, merges the other pairs'
//                pieces of a split block and writes the output with TMA tile
//                stores, or stores the partial.
// Tensor memory (512 columns per CTA): S[0] [0,128), S[1] [128,256) (fp32);
// P[0] [256,320), P[1] [320,384) (bf16 pairs; X = Q MqT^T overlays [256,384)
// at the end of a segment); O [384,512).
//
// Every wait is bounded (mbarriers and peer flags): on expiry the CTA raises
// its abort flag and records a timeout; there is no named barrier, so a role
// that leaves early never strands another.  The same kernel without the
// read-out serves the softmax layers that keep a growing KV cache.

#include <algorithm>
#include <vector>

#include "params.h"
#include "sm100.cuh"

namespace arl2 {

namespace {

constexpr int kThreads = 512;
constexpr int kRing = 7;
constexpr uint32_t kQTile = 32768;  // 128 rows x 128 bf16
constexpr uint32_t kBox = 16384;    // 128 rows x 64 bf16
constexpr uint32_t kSlot = 16384;   // a half tile: 64 keys x 128 dims, 128 keys x 64 dims, or 64 rows of MqT
constexpr uint32_t kTilesBytes = 2 * kQTile + kRing * kSlot + kQTile;  // Q x2, ring, output staging
constexpr uint32_t kBarBytes = 512;
constexpr uint32_t kStatsBytes = 4 * 128 * 4 + 2 * 128 * 4;  // (m, l) per softmax warpgroup; running max hand-off [2]
constexpr int kSmem = 232448;
static_assert(kTilesBytes + kBarBytes + kStatsBytes + 1024 <= uint32_t(kSmem), "shared memory layout too large");
constexpr int kMaxContrib = 8;
constexpr int kLaunchRegs = 128;
constexpr int kCtlRegs = 56;
constexpr int kSoftmaxRegs = 168;
constexpr int kEpiRegs = 112;
static_assert(128 * kCtlRegs + 256 * kSoftmaxRegs + 128 * kEpiRegs <= kThreads * kLaunchRegs,
              "register split too large");

enum {
  B_QF = 0,              // [2] Q slot loaded (rank 0: both CTAs' bytes)
  B_QE = 2,              // [2] Q slot free (commit, both CTAs)
  B_RF = 4,              // [kRing] ring slot loaded (rank 0: both CTAs' bytes)
  B_RE = 4 + kRing,      // [kRing] ring slot free (commit, both CTAs)
  B_SF = 4 + 2 * kRing,  // [2] S(i) in S[i & 1] (commit, both CTAs)
  B_SC = B_SF + 2,       // [2] S[i & 1] read by the softmax (rank 0: the owning warpgroup's 4 warps x 2 CTAs)
  B_PF = B_SC + 2,       // [2] P(i) in P[i & 1] (rank 0: the owning warpgroup's 4 warps x 2 CTAs)
  B_PD = B_PF + 2,       // [2] PV(i) done: P[i & 1] free, O current (commit, both CTAs)
  B_MX = B_PD + 2,       // [2 tile parities][4 quarters] running max after tile i published (local: 1 warp)
  B_SD = B_MX + 8,       // every MMA of the segment completed (commit, both CTAs)
  B_ST = B_SD + 1,       // the segment's statistics in shared memory (local: 8 warps)
  B_STC = B_ST + 1,      // statistics read by the epilogue (local: 4 warps)
  B_EO = B_STC + 1,      // epilogues done with O and X (rank 0: 4 warps x 2 CTAs)
  B_EL = B_EO + 1,       // this CTA's epilogue done with O and X (local: 4 warps)
  B_PQ = B_EL + 1,       // [4] a contributor's piece of this warp's rows in shared memory (local: bytes)
  B_DRAIN = B_PQ + 4,
  B_COUNT
};
static_assert(B_COUNT * 8 + 8 <= int(kBarBytes), "barrier area too small");

struct Seg {
  int bh, blk, j0, j1, n_contrib;
};

__device__ __forceinline__ bool next_seg(const AttnParams& p, unsigned& u, unsigned u_end, Seg& s) {
  if (u >= u_end) return false;
  const uint2 e = p.seg[u++];
  s.bh = int(e.x & 0x0FFFFFFFu);
  s.n_contrib = int(e.x >> 28);
  s.blk = int(e.y & 1023u);
  s.j0 = int((e.y >> 10) & 2047u);
  s.j1 = s.j0 + int(e.y >> 21);
  // (debug build) the segment lies inside the problem and the pairs whose
  // pieces it merges are pairs of this launch; every role decodes the same
  // list, so all of them stop at the same segment
  if (!ARL2_IN_BOUNDS(p.err, s.blk < p.n_blk && s.j0 < s.j1 && s.j1 <= p.nkv && s.n_contrib <= kMaxContrib &&
                                 2 * (int(blockIdx.x >> 1) + s.n_contrib) + 1 < p.grid &&
                                 (long long)(s.bh + 1) * p.n_blk * p.nkv <= p.total_units))
    return false;
  return true;
}

// Ring positions within a segment of n key tiles, in the order the issuers
// consume them (S about two tiles ahead of PV): K_0, K_1, K_2, V_0, K_3, V_1, ...,
// K_{n-1}, V_{n-3}, V_{n-2}, V_{n-1}, then MqT.
__device__ __forceinline__ int pos_k(int i) { return i < 2 ? i : 2 * i - 2; }
__device__ __forceinline__ int pos_v(int i, int n) {
  if (n == 1) return 1;
  return i + 2 < n ? 2 * i + 3 : 2 * n - 2 + (i - (n - 2));
}

__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release(unsigned* p, unsigned v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const WaitCtl& w) {
  const bool ok = mbar_wait(bar, parity, w);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ float* slot_of(const AttnParams& p, int cta) {
  return p.scratch + size_t(cta) * kAttnPairSlotFloats;
}

// ------------------------------------------------------------------ producer
// One thread per CTA.  Rank 0 announces the bytes of both CTAs on its own
// barriers; each CTA loads its own halves with rank 0's barrier as the target.
__device__ __forceinline__ void producer(const AttnParams& p, uint64_t* bars, uint8_t* sQ, uint8_t* sR,
                                         const CUtensorMap* tm_q, const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                                         const CUtensorMap* tm_mq, const int rank, const unsigned u_begin,
                                         const unsigned u_end, const WaitCtl& w) {
  uint32_t ring = 0, k = 0;
  unsigned u = u_begin;
  Seg s;
  const bool lead = rank == 0;
  while (next_seg(p, u, u_end, s)) {
    const int b = s.bh / p.heads, h = s.bh % p.heads;
    const int n = s.j1 - s.j0;
    const bool writer = s.j0 == 0;
    const int ntiles = 2 * n + ((writer && p.has_inter) ? 1 : 0);
    const int x0 = h * 128;
    const uint32_t qs = k & 1;
    // Q of this segment, once the MMAs of segment k - 2 have released the slot
    if (k >= 2 && !mbar_wait(&bars[B_QE + qs], ((k >> 1) - 1) & 1, w)) return;
    if (lead) mbar_expect_tx(&bars[B_QF + qs], 2 * kQTile);
    const int qrow = (2 * s.blk + rank) * 128;
    tma_load_3d_pair(sQ + qs * kQTile, tm_q, &bars[B_QF + qs], x0, qrow, b);
    tma_load_3d_pair(sQ + qs * kQTile + kBox, tm_q, &bars[B_QF + qs], x0 + 64, qrow, b);
    for (int t = 0; t < ntiles; ++t) {
      const uint32_t slot = ring % kRing;
      if (ring >= kRing && !mbar_wait(&bars[B_RE + slot], ((ring / kRing) - 1) & 1, w)) return;
      uint8_t* dst = sR + slot * kSlot;
      if (lead) mbar_expect_tx(&bars[B_RF + slot], 2 * kSlot);
      if (t < 2 * n) {
        // position t holds K_i or V_i (the inverse of pos_k / pos_v)
        int i, is_v;
        if (n == 1) {
          i = 0, is_v = t;
        } else if (t < 2) {
          i = t, is_v = 0;
        } else if (t >= 2 * n - 2) {
          i = t - n, is_v = 1;
        } else if ((t & 1) == 0) {
          i = t / 2 + 1, is_v = 0;
        } else {
          i = (t + 1) / 2 - 2, is_v = 1;
        }
        const int j = s.j0 + i;
        if (is_v) {  // all 128 keys, this CTA's 64 head dimensions
          tma_load_3d_pair(dst, tm_v, &bars[B_RF + slot], x0 + 64 * rank, j * 128, b);
        } else {     // this CTA's 64 keys, all 128 head dimensions
          tma_load_3d_pair(dst, tm_k, &bars[B_RF + slot], x0, j * 128 + 64 * rank, b);
          tma_load_3d_pair(dst + kSlot / 2, tm_k, &bars[B_RF + slot], x0 + 64, j * 128 + 64 * rank, b);
        }
      } else {  // this CTA's 64 rows of MqT
        tma_load_3d_pair(dst, tm_mq, &bars[B_RF + slot], 0, 64 * rank, s.bh);
        tma_load_3d_pair(dst + kSlot / 2, tm_mq, &bars[B_RF + slot], 64, 64 * rank, s.bh);
      }
      ++ring;
    }
    ++k;
  }
}

// ------------------------------------------------------------------ MMA issuer
// S (or X) over K = 128: A = the CTA's 128 query rows (two 64-column boxes
// 16 KB apart), B = its half of a K tile or of MqT (64 rows, boxes 8 KB apart).
__device__ __forceinline__ void mma_s_group(const uint32_t d, const uint32_t a_lo, const uint32_t b_lo,
                                            const uint32_t hi, const uint32_t idesc) {
#pragma unroll
  for (int kk = 0; kk < 8; ++kk)
    mma_pair_ss(d, a_lo + (kk >> 2) * (kBox >> 4) + (kk & 3) * 2, b_lo + (kk >> 2) * ((kSlot / 2) >> 4) + (kk & 3) * 2,
                hi, idesc, kk > 0);
}

// O (+)= P V over nk 16-key steps: P from tensor memory, V MN-major (the
// CTA's 64 head dimensions, one 128-byte row per key).
__device__ __forceinline__ void mma_pv_group(const uint32_t d, const uint32_t p_tmem, const uint32_t v_lo,
                                             const uint32_t hi, const uint32_t idesc, const int nk, const bool acc0) {
  if (nk == 8) {
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) mma_pair_ts(d, p_tmem + kk * 8, v_lo + kk * 128, hi, idesc, kk > 0 || acc0);
  } else {
    for (int kk = 0; kk < nk; ++kk) mma_pair_ts(d, p_tmem + kk * 8, v_lo + kk * 128, hi, idesc, kk > 0 || acc0);
  }
}

// Two threads of rank 0 issue the MMAs, so that a PV whose P is ready never
// queues behind the issue of an S (a thread issuing tcgen05.mma stalls while
// the tensor pipe's queue is full, ~the execution time of what it issues).
// Tiles are counted over the whole launch (g).
//
// S issuer: S(g) goes to S[g & 1] once the softmax of both CTAs has read
// S(g - 2) out of it (B_SC); it runs up to two tiles ahead of the softmax.
__device__ __forceinline__ void s_issuer(const AttnParams& p, uint64_t* bars, const uint32_t tmem,
                                         const uint32_t q_addr, const uint32_t r_addr, const unsigned u_begin,
                                         const unsigned u_end, const WaitCtl& w) {
  constexpr uint32_t kQ16 = kQTile >> 4, kSlot16 = kSlot >> 4;
  const uint32_t id_s = idesc_bf16(256, 128, 0, 0);
  const uint64_t dq64 = smem_desc_sw128(q_addr, 16, 1024);
  const uint32_t hi = uint32_t(dq64 >> 32);
  const uint32_t dq0 = uint32_t(dq64);
  const uint32_t dk0 = uint32_t(smem_desc_sw128(r_addr, 16, 1024));  // K-major ring slot
  uint32_t ring = 0, k = 0, gs = 0;
  unsigned u = u_begin;
  Seg s;
  while (next_seg(p, u, u_end, s)) {
    const int n = s.j1 - s.j0;
    const uint32_t qs = k & 1;
    const uint32_t dq = dq0 + qs * kQ16;
    if (!mbar_wait(&bars[B_QF + qs], (k >> 1) & 1, w)) return;
    for (int i = 0; i < n; ++i, ++gs) {
      const uint32_t rk = ring + pos_k(i), buf = gs & 1;
      if (!mbar_wait(&bars[B_RF + rk % kRing], (rk / kRing) & 1, w)) return;
      if (gs >= 2) {
        if (!mbar_wait(&bars[B_SC + buf], ((gs - 2) >> 1) & 1, w)) return;
        tc_fence_after();
      }
      mma_s_group(tmem + buf * 128, dq, dk0 + (rk % kRing) * kSlot16, hi, id_s);
      mma_commit_pair(&bars[B_SF + buf]);
      mma_commit_pair(&bars[B_RE + rk % kRing]);
    }
    ring += 2 * n + ((s.j0 == 0 && p.has_inter) ? 1 : 0);
    ++k;
  }
}

// PV issuer: PV(g) reads P[g & 1] once both CTAs' softmax has written P(g)
// (B_PF); a segment's first PV, which overwrites O, waits until the
// epilogues have read the previous segment's O and X (B_EO).  Then, for
// blocks finished here, X = Q MqT^T over [256, 384) (both P buffers are
// consumed by then).  Every S of the segment has completed before its last
// PV is issued (the softmax read S first), so this thread's commits also
// stand for them: B_SD (the segment's MMAs done) and B_QE (Q slot free).
__device__ __forceinline__ void pv_issuer(const AttnParams& p, uint64_t* bars, const uint32_t tmem,
                                          const uint32_t q_addr, const uint32_t r_addr, const unsigned u_begin,
                                          const unsigned u_end, const WaitCtl& w) {
  constexpr uint32_t kQ16 = kQTile >> 4, kSlot16 = kSlot >> 4;
  const uint32_t id_s = idesc_bf16(256, 128, 0, 0);
  const uint32_t id_o = idesc_bf16(256, 128, 0, 1);
  const uint64_t dq64 = smem_desc_sw128(q_addr, 16, 1024);
  const uint32_t hi = uint32_t(dq64 >> 32);
  const uint32_t dq0 = uint32_t(dq64);
  const uint32_t dk0 = uint32_t(smem_desc_sw128(r_addr, 16, 1024));    // K-major ring slot (MqT)
  const uint32_t dv0 = uint32_t(smem_desc_sw128(r_addr, kBox, 1024));  // MN-major ring slot (V)
  uint32_t ring = 0, k = 0, gp = 0;
  unsigned u = u_begin;
  Seg s;
  while (next_seg(p, u, u_end, s)) {
    const int n = s.j1 - s.j0;
    const uint32_t qs = k & 1;
    for (int j = 0; j < n; ++j, ++gp) {
      const uint32_t rv = ring + pos_v(j, n), buf = gp & 1;
      if (!mbar_wait(&bars[B_RF + rv % kRing], (rv / kRing) & 1, w)) return;
      if (!mbar_wait(&bars[B_PF + buf], (gp >> 1) & 1, w)) return;
      if (j == 0 && k > 0 && !mbar_wait(&bars[B_EO], (k - 1) & 1, w)) return;
      tc_fence_after();
      const int valid = min(128, p.kv_len - (s.j0 + j) * 128);
      mma_pv_group(tmem + 384, tmem + 256 + buf * 64, dv0 + (rv % kRing) * kSlot16, hi, id_o, (valid + 15) >> 4,
                   j > 0);
      mma_commit_pair(&bars[B_PD + buf]);
      mma_commit_pair(&bars[B_RE + rv % kRing]);
    }
    ring += 2 * n;
    if (s.j0 == 0 && p.has_inter) {  // X = Q MqT^T for the rows this pair finishes
      const uint32_t rm = ring;
      // Q is in (the S issuer saw it); waited on here too so that this
      // thread's MMA reads it after observing the load's completion
      if (!mbar_wait(&bars[B_QF + qs], (k >> 1) & 1, w)) return;
      if (!mbar_wait(&bars[B_RF + rm % kRing], (rm / kRing) & 1, w)) return;
      mma_s_group(tmem + 256, dq0 + qs * kQ16, dk0 + (rm % kRing) * kSlot16, hi, id_s);
      mma_commit_pair(&bars[B_RE + rm % kRing]);
      ++ring;
    }
    mma_commit_pair(&bars[B_SD]);
    mma_commit_pair(&bars[B_QE + qs]);
    ++k;
  }
}

// ------------------------------------------------------------------ softmax
// The two softmax warpgroups take alternate key tiles of the same 128 rows:
// warpgroup w owns the tiles g with g & 1 == w, so it always reads S[w] and
// writes P[w], one query row per thread and all 128 columns of the tile.
// While one computes the exponentials of tile g the other is on tile g + 1,
// so each one's waits and tensor-memory round trips hide behind the other's
// arithmetic.  The running row max m is handed along the tiles in order
// through shared memory: the owner of tile g takes m after tile g - 1 (which
// the other warpgroup publishes right after its row max, long before S(g) is
// in), raises it only when the tile's max exceeds it by more than 8 (a factor
// 256, so P <= 256), and publishes it before its exponentials.  A raised m
// rescales O (all 128 columns of the CTA's rows) once PV(g - 1) has completed
// and before P(g) is announced; rare.  Each warpgroup keeps its own row sum l
// against the last m it used; at the end of a segment both (m, l) go to
// shared memory and the epilogue combines them.
// 2^x for a pair on the FMA pipe: x = n + f with n = round(x) (adding
// 1.5 * 2^23 leaves n in the low mantissa bits), 2^f from the degree-3
// polynomial through the four Chebyshev nodes of [-1/2, 1/2] (coefficients of
// exp2_poly, relative error <= 1.0e-4, below the 2^-9 step of the bf16 P it
// feeds), 2^n added to the exponent field.  x is clamped below at -125.
__device__ __forceinline__ float2 exp2_poly_pair(float2 x) {
  constexpr float kRound = 12582912.f;  // 1.5 * 2^23
  constexpr float c0 = 0.999924541f, c1 = 0.693136752f, c2 = 0.242639482f, c3 = 0.0558382832f;
  x.x = fmaxf(x.x, -125.f);
  x.y = fmaxf(x.y, -125.f);
  const float2 t = __fadd2_rn(x, make_float2(kRound, kRound));
  const float2 f = __fadd2_rn(x, __fadd2_rn(make_float2(kRound, kRound), make_float2(-t.x, -t.y)));
  float2 q = __ffma2_rn(make_float2(c3, c3), f, make_float2(c2, c2));
  q = __ffma2_rn(q, f, make_float2(c1, c1));
  q = __ffma2_rn(q, f, make_float2(c0, c0));
  return make_float2(__uint_as_float((__float_as_uint(t.x) << 23) + __float_as_uint(q.x)),
                     __uint_as_float((__float_as_uint(t.y) << 23) + __float_as_uint(q.y)));
}

// Of the 16 pairs of each 32-column chunk, this many take the FMA-pipe
// exponential (pairs 1, 4, 7, ...); the rest take the MUFU.
constexpr int kPolyPerChunk = 3;

// P = 2^(S * scale * log2(e) - m) for 32 columns of a row, packed to bf16
// pairs; returns their sum.
template <bool kPoly>
__device__ __forceinline__ float exp_chunk(const uint32_t* r, const float2 sc, const float2 nm, uint32_t (&pk)[16]) {
  float2 s2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
  for (int x = 0; x < 16; ++x) {
    const float2 y = __ffma2_rn(make_float2(__uint_as_float(r[2 * x]), __uint_as_float(r[2 * x + 1])), sc, nm);
    const bool poly = kPoly && (x % 3 == 1) && (x / 3) < kPolyPerChunk;
    const float2 e = poly ? exp2_poly_pair(y) : make_float2(fast_exp2(y.x), fast_exp2(y.y));
    s2[x & 1] = __fadd2_rn(s2[x & 1], e);
    pk[x] = pack_bf16x2(e.x, e.y);
  }
  const float2 sa = __fadd2_rn(s2[0], s2[1]);
  return sa.x + sa.y;
}

__device__ __forceinline__ void softmax_role(const AttnParams& p, uint64_t* bars, float* stats, float* mchain,
                                             const uint32_t tmem, const int rank, const int wgi, const int quarter,
                                             const int lane, const unsigned u_begin, const unsigned u_end,
                                             const WaitCtl& w) {
  const int row = quarter * 32 + lane;
  const uint32_t lane_off = uint32_t(quarter * 32) << 16;
  const uint32_t tS = tmem + wgi * 128 + lane_off;       // S[wgi]
  const uint32_t tP = tmem + 256 + wgi * 64 + lane_off;  // P[wgi]
  const uint32_t tO = tmem + 384 + lane_off;
  // rank 1's warps arrive on rank 0's barriers themselves: a relaxed
  // cluster-scope arrive after tcgen05.wait and the thread-sync fence (the
  // release form costs each warp ~10^3 cycles)
  const uint32_t sc_lead = cluster_map(smem_u32(&bars[B_SC + wgi]), 0);
  const uint32_t pf_lead = cluster_map(smem_u32(&bars[B_PF + wgi]), 0);
  const float2 sc = make_float2(p.scale_log2, p.scale_log2);
  uint32_t g = 0, k = 0;
  unsigned u = u_begin;
  Seg s;
  while (next_seg(p, u, u_end, s)) {
    const int n = s.j1 - s.j0;
    float m = -INFINITY, l = 0.f;  // the last m this warpgroup used, and its l against it
    bool first = true;
    for (int i = 0; i < n; ++i, ++g) {
      if (int(g & 1) != wgi) continue;
      if (!warp_wait(&bars[B_SF + wgi], (g >> 1) & 1, w)) return;
      tc_fence_after();
      uint32_t r[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tS + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32 * c]));
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {  // S[wgi] may take S(g + 2)
        if (rank == 0) mbar_arrive(&bars[B_SC + wgi]);
        else mbar_arrive_cluster_relaxed(sc_lead);
      }
      const int valid = min(128, p.kv_len - (s.j0 + i) * 128);
      if (valid < 128) {
#pragma unroll
        for (int x = 0; x < 128; ++x)
          if (x >= valid) r[x] = __float_as_uint(-INFINITY);
      }
      float m4[4];
#pragma unroll
      for (int q = 0; q < 4; ++q)
        m4[q] = fmax3(__uint_as_float(r[q]), __uint_as_float(r[4 + q]), __uint_as_float(r[8 + q]));
#pragma unroll
      for (int x = 12; x < 124; x += 8)
#pragma unroll
        for (int q = 0; q < 4; ++q) m4[q] = fmax3(m4[q], __uint_as_float(r[x + q]), __uint_as_float(r[x + 4 + q]));
#pragma unroll
      for (int q = 0; q < 4; ++q) m4[q] = fmaxf(m4[q], __uint_as_float(r[124 + q]));
      const float mx = fmaxf(fmax3(m4[0], m4[1], m4[2]), m4[3]) * sc.x;
      // m after tile g - 1, from the other warpgroup; waited for at a
      // segment's first tile too (value unused) so that the two hand-off
      // slots are never rewritten before they are read
      float m_in = -INFINITY;
      if (g > 0) {
        const uint32_t gq = g - 1;
        if (!warp_wait(&bars[B_MX + (gq & 1) * 4 + quarter], (gq >> 1) & 1, w)) return;
        if (i > 0) m_in = mchain[(gq & 1) * 128 + row];
      }
      const bool need = i > 0 && mx > m_in + 8.f;
      const float mg = (i == 0 || need) ? mx : m_in;
      mchain[(g & 1) * 128 + row] = mg;
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[B_MX + (g & 1) * 4 + quarter]);
      const bool any_rescale = __any_sync(0xffffffffu, need);
      // the exponentials go to registers first: P[wgi] is free only once
      // PV(g - 2) has completed, and a warpgroup's first tile of a segment
      // also waits until the epilogue is done with X, which overlays both P
      // buffers
      const float2 nm = make_float2(-mg, -mg);
      float sum = 0.f;
      uint32_t pk[64];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t(&pc)[16] = *reinterpret_cast<uint32_t(*)[16]>(&pk[16 * c]);
        sum += valid >= 128 ? exp_chunk<true>(&r[32 * c], sc, nm, pc) : exp_chunk<false>(&r[32 * c], sc, nm, pc);
      }
      if (g >= 2 && !warp_wait(&bars[B_PD + wgi], ((g - 2) >> 1) & 1, w)) return;
      if (first && k > 0 && !warp_wait(&bars[B_EL], (k - 1) & 1, w)) return;
      first = false;
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_st16(tP + c * 16, *reinterpret_cast<const uint32_t(*)[16]>(&pk[16 * c]));
      if (any_rescale) {  // O *= 2^(m_in - mg) (1 for rows that keep m) once PV(g - 1) has completed
        if (!warp_wait(&bars[B_PD + (wgi ^ 1)], ((g - 1) >> 1) & 1, w)) return;
        tc_fence_after();
        const float f = fast_exp2(m_in - mg);
#pragma unroll 1
        for (int q = 0; q < 4; ++q) {
          uint32_t o[32];
          tmem_ld32(tO + q * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int x = 0; x < 32; ++x) o[x] = __float_as_uint(__uint_as_float(o[x]) * f);
          tmem_st32(tO + q * 32, o);
        }
      }
      l = fmaf(l, m == mg ? 1.f : fast_exp2(m - mg), sum);
      m = mg;
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {  // P(g) is in
        if (rank == 0) mbar_arrive(&bars[B_PF + wgi]);
        else mbar_arrive_cluster_relaxed(pf_lead);
      }
    }
    // the epilogue has read the previous segment's statistics
    if (k > 0 && !warp_wait(&bars[B_STC], (k - 1) & 1, w)) return;
    stats[wgi * 256 + row] = m;  // -inf, 0 for a warpgroup with no tile in the segment
    stats[wgi * 256 + 128 + row] = l;
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars[B_ST]);
    ++k;
  }
}

// ------------------------------------------------------------------ epilogue
// A contributor's piece: O / l rounded to bf16, rows in four 8 KB quarters
// (one per epilogue warp); within quarter q, 16-byte chunk c (columns
// 8c..8c+7) of row 32q + r lies at byte q * 8192 + (c * 32 + r) * 16, so a
// warp's chunk is one contiguous 512-byte span and a warp's quarter is one
// 8 KB block that the finishing CTA copies into shared memory whole.  (m, l)
// follow in fp32 at float kPartStats.
constexpr int kPartStats = 128 * 128;
constexpr uint32_t kPartQuarter = 8192;

// Acquire the ready flags of this warp's quarter of contributors pair + 1 ..
// pair + n (bounded spin by lane 0, then every lane acquires).
__device__ __forceinline__ bool acquire_pieces(const AttnParams& p, int pair, int rank, int quarter, int lane, int n,
                                               volatile int* abort_flag) {
  if (lane == 0) {
    for (int q = 0; q < n && !*abort_flag; ++q) {
      const unsigned* f = p.ready + (size_t(2 * (pair + 1 + q) + rank)) * 4 + quarter;
      const uint64_t t0 = global_timer_ns();
      while (ld_acquire(f) == 0u) {
        if (*abort_flag || global_timer_ns() - t0 > p.wait_limit_ns) {
          *abort_flag = 1;
          record_error(p.err, kDevTimeout);
          break;
        }
      }
    }
  }
  __syncwarp();
  if (*abort_flag) return false;
  for (int q = 0; q < n; ++q) (void)ld_acquire(p.ready + (size_t(2 * (pair + 1 + q) + rank)) * 4 + quarter);
  return true;
}

// One warpgroup, one query row per thread.  At the end of a segment (its MMAs
// done, the statistics in shared memory):
//  * own piece: m, l = l_lo + l_hi, O / l;
//  * a segment that does not start at key tile 0 (a contributor) stores its
//    piece (O / l in bf16, m, l) and raises this warp's ready flag;
//  * a segment holding a whole block writes O / l (+ X) through per-warp
//    staging boxes and TMA tile stores;
//  * a segment that starts a block continued by the next pairs (always the
//    pair's last segment) merges their pieces in key order before adding X.
//    Those pieces are ready long before the segment's MMAs end, so while they
//    run this warp acquires the flags, reads the pieces' (m, l) and copies the
//    first piece's quarter into the Q slot the segment does not use.
// Tensor memory is handed back (B_EO on rank 0 for the issuer, B_EL locally
// for the softmax) as soon as O and X have been read.
__device__ __forceinline__ bool epilogue_role(const AttnParams& p, uint64_t* bars, const float* stats, uint8_t* stage,
                                              uint8_t* sQ, const CUtensorMap* tm_o, const uint32_t tmem, const int cta,
                                              const int rank, const int quarter, const int lane,
                                              const unsigned u_begin, const unsigned u_end, volatile int* abort_flag,
                                              const WaitCtl& w) {
  const int row = quarter * 32 + lane;
  const uint32_t lane_off = uint32_t(quarter * 32) << 16;
  const uint32_t eo_leader = cluster_map(smem_u32(&bars[B_EO]), 0);
  const bool use_intra = !(p.flags & 2u);
  const bool use_inter = p.has_inter && !(p.flags & 1u);
  const int pair = cta >> 1;
  uint32_t k = 0;
  bool staged = false;
  uint8_t* wst = stage + quarter * 8192;
  unsigned u = u_begin;
  Seg s;
  while (next_seg(p, u, u_end, s)) {
    const int b = s.bh / p.heads, h = s.bh % p.heads;
    const bool writer = s.j0 == 0, full = writer && s.j1 == p.nkv;
    const int qt = 2 * s.blk + rank;
    const bool row_ok = qt * 128 + row < p.q_len;
    const bool warp_on = qt * 128 + quarter * 32 < p.q_len;  // warp-uniform
    const bool with_x = writer && use_inter;
    const int n_contrib = (writer && !full) ? s.n_contrib : 0;  // the host keeps it <= kMaxContrib
    uint8_t* piece = sQ + ((k + 1) & 1) * kQTile + quarter * kPartQuarter;
    float mk[kMaxContrib], lk[kMaxContrib];
#pragma unroll
    for (int q = 0; q < kMaxContrib; ++q) {
      mk[q] = -INFINITY;
      lk[q] = 0.f;
    }
    if (n_contrib > 0) {
      if (!acquire_pieces(p, pair, rank, quarter, lane, n_contrib, abort_flag)) return false;
      // the other Q slot is free once the previous segment's MMAs are done
      if (lane == 0 && (k == 0 || mbar_wait(&bars[B_QE + ((k + 1) & 1)], ((k - 1) >> 1) & 1, w))) {
        fence_async_global();
        mbar_expect_tx(&bars[B_PQ + quarter], kPartQuarter);
        bulk_load(piece, reinterpret_cast<const uint8_t*>(slot_of(p, 2 * (pair + 1) + rank)) + quarter * kPartQuarter,
                  kPartQuarter, &bars[B_PQ + quarter]);
      }
      __syncwarp();
      if (*abort_flag) return false;
#pragma unroll
      for (int q = 0; q < kMaxContrib; ++q) {
        if (q < n_contrib) {
          const float* st = slot_of(p, 2 * (pair + 1 + q) + rank) + kPartStats;
          mk[q] = st[row];
          lk[q] = st[128 + row];
        }
      }
    }
    if (!warp_wait(&bars[B_SD], k & 1, w)) return false;
    if (!warp_wait(&bars[B_ST], k & 1, w)) return false;
    tc_fence_after();
    const float m0 = stats[row], m1 = stats[256 + row], M = fmaxf(m0, m1);
    const float L = stats[128 + row] * fast_exp2(m0 - M) + stats[384 + row] * fast_exp2(m1 - M);
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars[B_STC]);
    float a0 = 0.f, wk[kMaxContrib];
#pragma unroll
    for (int q = 0; q < kMaxContrib; ++q) wk[q] = 0.f;
    if (!writer) {
      a0 = 1.f / L;
    } else if (n_contrib == 0) {
      a0 = row_ok ? 1.f / L : 0.f;
    } else {
      float Mx = M;
#pragma unroll
      for (int q = 0; q < kMaxContrib; ++q) Mx = fmaxf(Mx, mk[q]);
      const float es = fast_exp2(M - Mx);
      float Lx = L * es;
#pragma unroll
      for (int q = 0; q < kMaxContrib; ++q) {
        wk[q] = q < n_contrib ? lk[q] * fast_exp2(mk[q] - Mx) : 0.f;
        Lx += wk[q];
      }
      const float inv = row_ok ? 1.f / Lx : 0.f;
      a0 = es * inv;
#pragma unroll
      for (int q = 0; q < kMaxContrib; ++q) wk[q] *= inv;
    }
    if (!use_intra) a0 = 0.f;
    const float2 A0 = make_float2(a0, a0);
    if (!writer) {  // ------------------------------------------------------ contributor
      float* slot = slot_of(p, cta);
      uint4* d4 = reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(slot) + quarter * kPartQuarter) + lane;
#pragma unroll 1
      for (int q = 0; q < 4; ++q) {  // 32 columns at a time
        uint32_t o0[32];
        tmem_ld32(tmem + 384 + lane_off + q * 32, o0);
        tmem_wait_ld();
        const float2* v = reinterpret_cast<const float2*>(o0);
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const float2 v0 = __fmul2_rn(v[4 * x], A0), v1 = __fmul2_rn(v[4 * x + 1], A0);
          const float2 v2 = __fmul2_rn(v[4 * x + 2], A0), v3 = __fmul2_rn(v[4 * x + 3], A0);
          d4[(4 * q + x) * 32] = make_uint4(pack_bf16x2(v0.x, v0.y), pack_bf16x2(v1.x, v1.y), pack_bf16x2(v2.x, v2.y),
                                            pack_bf16x2(v3.x, v3.y));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bars[B_EL]);
        mbar_arrive_cluster_relaxed(eo_leader);
      }
      slot[kPartStats + row] = M;
      slot[kPartStats + 128 + row] = L;
      __threadfence();
      __syncwarp();
      if (lane == 0) st_release(p.ready + size_t(cta) * 4 + quarter, 1u);
      ++k;
      continue;
    }
    // ------------------------------------------------------------------ writer
    if (lane == 0 && staged) bulk_wait_read0();  // this warp's previous tile store has read its boxes
    __syncwarp();
    if (n_contrib > 0 && !warp_wait(&bars[B_PQ + quarter], 0, w)) return false;  // once per launch
#pragma unroll 1
    for (int q = 0; q < 4; ++q) {  // 32 columns at a time
      uint32_t o0[32], rx[32];
      tmem_ld32(tmem + 384 + lane_off + q * 32, o0);
      if (with_x) tmem_ld32(tmem + 256 + lane_off + q * 32, rx);
      tmem_wait_ld();
      if (q == 3) {  // O and X are read: hand tensor memory back
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&bars[B_EL]);
          mbar_arrive_cluster_relaxed(eo_leader);
        }
      }
      float2* v = reinterpret_cast<float2*>(o0);
#pragma unroll
      for (int x = 0; x < 16; ++x) v[x] = __fmul2_rn(v[x], A0);
      if (n_contrib > 0 && use_intra) {
#pragma unroll 1
        for (int c2 = 0; c2 < n_contrib; ++c2) {
          // the first piece from shared memory, any others from global memory
          const uint4* src =
              c2 == 0 ? reinterpret_cast<const uint4*>(piece) + lane
                      : reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(slot_of(p, 2 * (pair + 1 + c2) + rank)) +
                                                       quarter * kPartQuarter) + lane;
          const float2 W = make_float2(wk[c2], wk[c2]);
          uint4 t4[4];
#pragma unroll
          for (int x = 0; x < 4; ++x) t4[x] = src[(4 * q + x) * 32];
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            const uint32_t w4[4] = {t4[x].x, t4[x].y, t4[x].z, t4[x].w};
#pragma unroll
            for (int e = 0; e < 4; ++e)
              v[4 * x + e] = __ffma2_rn(make_float2(__uint_as_float(w4[e] << 16), __uint_as_float(w4[e] & 0xFFFF0000u)), W,
                                        v[4 * x + e]);
          }
        }
      }
      if (with_x) {
        const float2* x2 = reinterpret_cast<const float2*>(rx);
#pragma unroll
        for (int x = 0; x < 16; ++x) v[x] = __fadd2_rn(v[x], x2[x]);
      }
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const int ch = 4 * q + x;  // 16-byte chunk of the row: box ch / 8, chunk ch % 8 swizzled by row
        *reinterpret_cast<uint4*>(wst + (ch >> 3) * 4096 + lane * 128 + (((ch & 7) ^ (lane & 7)) << 4)) =
            make_uint4(pack_bf16x2(v[4 * x].x, v[4 * x].y), pack_bf16x2(v[4 * x + 1].x, v[4 * x + 1].y),
                       pack_bf16x2(v[4 * x + 2].x, v[4 * x + 2].y), pack_bf16x2(v[4 * x + 3].x, v[4 * x + 3].y));
      }
    }
    fence_async_smem();
    __syncwarp();
    if (lane == 0 && warp_on) {
      tma_store_3d(tm_o, wst, h * 128, qt * 128 + quarter * 32, b);
      tma_store_3d(tm_o, wst + 4096, h * 128 + 64, qt * 128 + quarter * 32, b);
      bulk_commit();
    }
    staged = true;
    if (n_contrib > 0 && lane == 0) {  // the pieces are read: their flags go back to zero for the next launch
      for (int q = 0; q < n_contrib; ++q) p.ready[(size_t(2 * (pair + 1 + q) + rank)) * 4 + quarter] = 0u;
    }
    ++k;
  }
  if (lane == 0) bulk_wait0();
  return true;
}

// ------------------------------------------------------------------ kernel
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
attn_pair_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_mq,
                 const __grid_constant__ CUtensorMap tm_o, const AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                               // [2] Q slots
  uint8_t* sR = smem + 2 * kQTile;                  // [kRing] half tiles
  uint8_t* sStage = sR + kRing * kSlot;             // output staging
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kTilesBytes);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + B_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  float* stats = reinterpret_cast<float*>(smem + kTilesBytes + kBarBytes);  // per warpgroup m[128], l[128]
  float* mchain = stats + 4 * 128;                                          // running max hand-off [2][128]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cta = blockIdx.x;
  const int rank = int(cluster_ctarank());
  const int pair = cta >> 1;
  // (debug build) the pair's segment list lies inside the launch's list
  const bool pair_ok = ARL2_CHECKED(int(gridDim.x) == p.grid && p.grid <= kAttnMaxGrid);
  const unsigned u_begin = pair_ok ? p.seg_first[pair] : 0u, u_end = pair_ok ? p.seg_first[pair + 1] : 0u;
  const bool segs_ok =
      pair_ok && ARL2_CHECKED(u_begin <= u_end && u_end <= unsigned(p.n_segs) && p.n_segs <= kAttnMaxSegs);
  // The same offset in both CTAs (the launch gives both the same dynamic
  // shared memory); a layout that does not fit is refused by both.
  const bool fits = size_t(smem - smem_raw) + kTilesBytes + kBarBytes + kStatsBytes <= size_t(kSmem);

  if (threadIdx.x == 0) {
    for (int i = 0; i < B_COUNT; ++i) {
      uint32_t count = 1;
      if (i >= B_SC && i < B_PF + 2) count = 8;   // the owning warpgroup's 4 warps in each CTA
      if (i == B_ST) count = 8;                    // 8 softmax warps
      if (i == B_STC || i == B_EL) count = 4;      // the epilogue's 4 warps
      if (i == B_EO) count = 8;                    // 4 epilogue warps x 2 CTAs (rank 0's copy)
      mbar_init(&bars[i], count);
    }
    *abort_flag = (fits && segs_ok) ? 0 : 1;
    fence_barrier_init();
  }
  if (warp == 2) tmem_alloc_pair(tmem_holder, 512);
  tc_fence_before();
  __syncthreads();
  cluster_barrier();  // both CTAs' barriers initialised before any remote arrive or load
  tc_fence_after();
  // The set-up above touches only this pair's shared and tensor memory, so it
  // may overlap the kernel before this one on the stream; every global access
  // below follows that kernel's completion.  The next launch of this kernel may
  // then be scheduled on the SMs this grid frees as its CTAs finish.
  grid_dependency_wait();
  allow_dependent_launch();
  if (threadIdx.x == 0 && !fits) record_error(p.err, kDevBadShape);
  if (threadIdx.x == 0 && !segs_ok) record_error(p.err, kDevBounds);
  const uint32_t tmem = *tmem_holder;
  const WaitCtl w{abort_flag, p.err, p.wait_limit_ns};
  const int wg = warp >> 2;
  if (!*abort_flag) {
    if (wg == 0) {
      regs_dec<kCtlRegs>();
      if (warp == 0 && lane == 0) {
        tma_prefetch(&tm_q);
        tma_prefetch(&tm_k);
        tma_prefetch(&tm_v);
        producer(p, bars, sQ, sR, &tm_q, &tm_k, &tm_v, &tm_mq, rank, u_begin, u_end, w);
      } else if (warp == 1 && lane == 0 && rank == 0) {
        s_issuer(p, bars, tmem, smem_u32(sQ), smem_u32(sR), u_begin, u_end, w);
      } else if (warp == 3 && lane == 0 && rank == 0) {
        pv_issuer(p, bars, tmem, smem_u32(sQ), smem_u32(sR), u_begin, u_end, w);
      }
      __syncwarp();
    } else if (wg == 3) {
      regs_dec<kEpiRegs>();
      epilogue_role(p, bars, stats, sStage, sQ, &tm_o, tmem, cta, rank, warp & 3, lane, u_begin, u_end, abort_flag, w);
    } else {
      regs_inc<kSoftmaxRegs>();
      softmax_role(p, bars, stats, mchain, tmem, rank, wg - 1, warp & 3, lane, u_begin, u_end, w);
    }
  }

  // ------------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  // Every MMA issued by rank 0 has completed and every commit it made has
  // arrived in both CTAs once the drain commit (the last one) has arrived:
  // only then may either CTA release its shared and tensor memory.
  if (warp == 1 && lane == 0) {
    if (rank == 0) mma_commit_pair(&bars[B_DRAIN]);
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(&bars[B_DRAIN], 0) && global_timer_ns() - t0 < 10000000ull) {
    }
  }
  if (*abort_flag) {
    // A wait ran out (here or, through a barrier that never completed, in the
    // other CTA): let this CTA's own copies land before its shared memory is
    // released.
    if (warp == 0 && lane == 0) {
      const uint64_t t0 = global_timer_ns();
      while (global_timer_ns() - t0 < 2000000ull) {
      }
    }
    if (wg == 3 && lane == 0) bulk_wait0();
  }
  __syncthreads();
  cluster_barrier();  // neither CTA leaves while the other may still signal its barriers
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

}  // namespace

cudaError_t launch_attn_pair(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             const CUtensorMap& tmq, const CUtensorMap& tmo, const AttnParams& p,
                             cudaStream_t stream) {
  static unsigned done = 0;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(attn_pair_kernel), kSmem, &done);
  if (e != cudaSuccess) return e;
  static int regs = -1;
  if (regs < 0) {
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, attn_pair_kernel);
    if (e != cudaSuccess) return e;
    regs = fa.numRegs;
  }
  if (regs != kLaunchRegs) return cudaErrorInvalidConfiguration;  // the register split needs this count
  if (p.grid < 2 || (p.grid & 1)) return cudaErrorInvalidConfiguration;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmem;
  cfg.stream = stream;
  // Every pair must be resident at once (a finishing pair waits for the
  // pieces of the pairs after it): the grid may not exceed the number of
  // clusters the device can hold.
  static int capacity = -1;
  if (capacity < 0) {
    int n = 0;
    e = cudaOccupancyMaxActiveClusters(&n, attn_pair_kernel, &cfg);
    if (e != cudaSuccess) return e;
    capacity = n;
  }
  if (p.grid / 2 > capacity) return cudaErrorCooperativeLaunchTooLarge;
  // Programmatic stream serialisation: the grid may be scheduled before the
  // kernel ahead of it on the stream has finished (the kernel waits for it
  // before any global access), which hides this launch's set-up.
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, attn_pair_kernel, tq, tk, tv, tmq, tmo, p);
}

int attn_pair_capacity() {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmem;
  static unsigned done = 0;
  if (ensure_smem_attr(reinterpret_cast<const void*>(attn_pair_kernel), kSmem, &done) != cudaSuccess) return 0;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, attn_pair_kernel, &cfg) != cudaSuccess) return 0;
  return n;
}

// Host partition of the (block, key tile) units over the pairs, as explicit
// per-pair segment lists.  Two schedules are costed (a segment costs its key
// tiles plus kSegCost for its start-up, drain and epilogue) and the cheaper
// makespan is taken:
//  * stream-K: the unit sequence cut into equal contiguous ranges (a range is
//    the tail of one block, whole blocks, and the head of another);
//  * whole blocks first: every pair takes floor(NB / pairs) whole blocks
//    (round f: blocks f P .. f P + P - 1, so the blocks of a head run side by
//    side); the NB % pairs remaining blocks are each cut into k near-equal
//    pieces (k pairs per block, at most one piece per pair).  A contributing
//    piece is its pair's first segment, so that it is stored early, or, for
//    key ranges of kLongKeyTiles tiles and more, its last, so that all whole
//    blocks start together (their K/V tiles are then read from DRAM once and
//    shared through L2); the piece holding key tile 0, which merges the
//    others, is its pair's last.
// In both, a split block is finished by the pair holding its key tile 0 and
// continued by the pairs right after it; each pair contributes at most one
// piece (one scratch slot per CTA).
namespace {
constexpr int kSegCost = 2;
// a finishing segment reads its first piece with one bulk copy issued while
// its MMAs run, and every further piece with latency-bound loads at the end
constexpr int kMergeCost = 4;
constexpr int kLongKeyTiles = 32;

struct HostSeg {
  long long bh;
  int blk, j0, j1, n_contrib;
};

bool pack_segments(AttnParams& p, const std::vector<std::vector<HostSeg>>& per_pair) {
  int n = 0;
  for (size_t c = 0; c < per_pair.size(); ++c) {
    p.seg_first[c] = unsigned(n);
    for (const HostSeg& h : per_pair[c]) {
      if (n >= kAttnMaxSegs || h.bh >= (1LL << 28) || h.blk >= 1024 || h.j0 >= 2048 || h.j1 - h.j0 >= 2048 ||
          h.j1 <= h.j0 || h.n_contrib > kMaxContrib)
        return false;
      p.seg[n].x = unsigned(h.bh) | (unsigned(h.n_contrib) << 28);
      p.seg[n].y = unsigned(h.blk) | (unsigned(h.j0) << 10) | (unsigned(h.j1 - h.j0) << 21);
      ++n;
    }
  }
  p.seg_first[per_pair.size()] = unsigned(n);
  p.n_segs = n;
  return true;
}

long long makespan(const std::vector<std::vector<HostSeg>>& per_pair) {
  long long worst = 0;
  for (const auto& v : per_pair) {
    long long c = 0;
    for (const HostSeg& h : v) c += (h.j1 - h.j0) + kSegCost + kMergeCost * std::max(0, h.n_contrib - 1);
    worst = std::max(worst, c);
  }
  return worst;
}

// stream-K over `units` with `pairs` contiguous ranges
std::vector<std::vector<HostSeg>> stream_k(const AttnParams& p, long long units, long long pairs) {
  std::vector<long long> range(static_cast<size_t>(pairs) + 1);
  for (long long c = 0; c <= pairs; ++c) range[size_t(c)] = units * c / pairs;
  std::vector<std::vector<HostSeg>> out(static_cast<size_t>(pairs));
  for (long long c = 0; c < pairs; ++c) {
    long long u = range[size_t(c)];
    while (u < range[size_t(c) + 1]) {
      const long long blk_lin = u / p.nkv;
      HostSeg h;
      h.bh = blk_lin / p.n_blk;
      h.blk = int(blk_lin % p.n_blk);
      h.j0 = int(u % p.nkv);
      h.j1 = int(std::min<long long>(p.nkv, h.j0 + (range[size_t(c) + 1] - u)));
      h.n_contrib = 0;
      if (h.j0 == 0 && h.j1 < p.nkv) {  // the pairs after this one that continue the block
        const long long block_end = (blk_lin + 1) * p.nkv;
        int n = 0;
        while (c + 1 + n < pairs && range[size_t(c + 1 + n)] < block_end) ++n;
        h.n_contrib = n;
      }
      out[size_t(c)].push_back(h);
      u += h.j1 - h.j0;
    }
  }
  return out;
}

std::vector<std::vector<HostSeg>> blocks_first(const AttnParams& p, long long nb, long long pairs, bool pieces_last) {
  std::vector<std::vector<HostSeg>> out(static_cast<size_t>(pairs));
  const long long full = nb / pairs, rem = nb - full * pairs;
  long long k = rem > 0 ? std::min<long long>({pairs / rem, kMaxContrib + 1, p.nkv}) : 0;
  if (rem > 0 && k < 1) k = 1;
  std::vector<HostSeg> first(static_cast<size_t>(pairs), HostSeg{-1, 0, 0, 0, 0});
  std::vector<HostSeg> last(static_cast<size_t>(pairs), HostSeg{-1, 0, 0, 0, 0});
  for (long long r = 0; r < rem; ++r) {
    const long long blk_lin = full * pairs + r;
    for (long long q = 0; q < k; ++q) {
      HostSeg h;
      h.bh = blk_lin / p.n_blk;
      h.blk = int(blk_lin % p.n_blk);
      h.j0 = int(p.nkv * q / k);
      h.j1 = int(p.nkv * (q + 1) / k);
      h.n_contrib = q == 0 ? int(k - 1) : 0;
      const long long c = r * k + q;  // block r's pieces on pairs r k .. r k + k - 1
      (q == 0 ? last : first)[size_t(c)] = h;
    }
  }
  for (long long c = 0; c < pairs; ++c) {
    if (!pieces_last && first[size_t(c)].bh >= 0) out[size_t(c)].push_back(first[size_t(c)]);
    for (long long f = 0; f < full; ++f) {  // round f: blocks f P .. f P + P - 1, the heads' blocks side by side
      const long long blk_lin = f * pairs + c;
      out[size_t(c)].push_back(HostSeg{blk_lin / p.n_blk, int(blk_lin % p.n_blk), 0, p.nkv, 0});
    }
    if (pieces_last && first[size_t(c)].bh >= 0) out[size_t(c)].push_back(first[size_t(c)]);
    if (last[size_t(c)].bh >= 0) out[size_t(c)].push_back(last[size_t(c)]);
  }
  return out;
}
}  // namespace

bool attn_pair_partition(AttnParams& p, int batch, int max_pairs) {
  p.n_qt = (p.q_len + 127) / 128;
  p.n_blk = (p.n_qt + 1) / 2;
  p.nkv = (p.kv_len + 127) / 128;
  if (p.n_qt < 1 || p.nkv < 1) return false;
  const long long bh = (long long)batch * p.heads;
  const long long nb = bh * p.n_blk;
  const long long units = nb * p.nkv;
  if (units >= (1LL << 31)) return false;
  p.total_units = units;
  // Each pair takes at least an eighth of a block, so a block is split across
  // at most nine pairs (the finishing pair reads at most eight pieces).
  const long long u_min = (p.nkv + kMaxContrib - 1) / kMaxContrib;
  long long pairs = units / (u_min > 0 ? u_min : 1);
  if (pairs > max_pairs) pairs = max_pairs;
  if (pairs > kAttnMaxGrid / 2) pairs = kAttnMaxGrid / 2;
  if (pairs < 1) return false;
  std::vector<std::vector<HostSeg>> a = stream_k(p, units, pairs);
  // Long key ranges (KV-cache layers): every pair starts its whole blocks at
  // once, so the pairs on one head's blocks read each K/V tile at about the
  // same time and it crosses DRAM once; the split pieces come last.  Short
  // ones: the cheaper of the two schedules.
  const bool long_keys = p.nkv >= kLongKeyTiles;
  std::vector<std::vector<HostSeg>> b = blocks_first(p, nb, pairs, long_keys);
  std::vector<std::vector<HostSeg>>& best = (long_keys || makespan(b) < makespan(a)) ? b : a;
  while (!best.empty() && best.back().empty()) best.pop_back();  // pairs left without work
  if (best.empty() || !pack_segments(p, best)) return false;
  p.grid = int(2 * best.size());
  return true;
}

}  // namespace arl2
