// Intra-frame softmax attention with the inter-frame read-out fused into its
// epilogue, bf16 operands, fp32 accumulation in tensor memory (sm_100a).
//
//   O = softmax(Q K^T * scale) V  +  Q MqT^T        (MqT = (phi_q S_{N-1})^T)
//
// The first term is the intra-frame branch (ARL2 summary, section 2.1: the
// original bidirectional softmax attention within each frame).  The second is
// the inter-frame read-out O_inter = Q' S_{N-1} = (Q phi_q) S_{N-1}, computed
// as Q (phi_q S_{N-1}): phi_q S is formed once per state write, so a pass
// costs one extra 128 x 128 x 128 MMA per 128 query rows.
//
// Work decomposition.  Query tiles of 128 rows are paired into blocks of 256
// rows (sub-tiles A and B) that share every K/V tile.  The work of a launch is
// the sequence of (block, key tile) units over all (stream, head) pairs.  A
// persistent grid of one CTA per SM takes contiguous, equal ranges of that sequence
// ("stream-K"), so the grid stays full whatever the number of query tiles.  A
// block whose key range is split across CTAs is finished by the CTA holding
// its first key tiles (its last segment): the others (whose first segment
// continues it) store their normalised partial output and softmax statistics
// (m, l) to a scratch slot and raise a ready flag; the finishing CTA combines
// the partials in key order (deterministic) and adds the read-out.  Ready
// flags are reset by their consumer, so every launch leaves them at zero.
//
// Roles (512 threads, four warpgroups):
//   warp 0       TMA producer: per segment, Q of both sub-tiles; K_j, V_j
//                (and MqT for blocks this CTA finishes) through a 4-slot ring;
//   warp 1       tcgen05 issuer (one thread): S = Q K_j^T, O += P V_j,
//                X = Q MqT^T;
//   warp 2       tensor-memory allocator;
//   warps 4..7   softmax of sub-tile A (one query row per thread);
//   warps 8..11  softmax of sub-tile B;
//   warps 12..15 epilogue: reads O (and X) from tensor memory at the end of a
//                segment, hands tensor memory back to the issuer at once, then
//                writes the partial or the combined output (TMA tile store)
//                while the other roles run the next segment.
// Tensor memory (512 columns): S_A [0,128), S_B [128,256) (P written in
// place as bf16 pairs, then X), O_A [256,384), O_B [384,512).
//
// The same kernel without the read-out serves the softmax layers that keep a
// growing KV cache (the K/V tensor maps then cover the cache).

#include "params.h"
#include "sm100.cuh"

namespace arl2 {

constexpr int kAttnThreads = 512;
constexpr int kRing = 4;
constexpr uint32_t kTile = 32768;  // 128 rows x 128 bf16
constexpr uint32_t kHalf = 16384;  // one 64-column box
constexpr uint32_t kTilesBytes = (2 + kRing + 1) * kTile;  // Q x2, ring, output staging
constexpr uint32_t kBarBytes = 256;                         // mbarriers, tensor-memory address, abort flag
constexpr uint32_t kStatsBytes = 2 * 2 * 128 * 4;           // (m, l) of both sub-tiles
constexpr uint32_t kSmallBytes = kBarBytes + kStatsBytes;
// the whole 227 KB a CTA may have: the tiles start at the first 1024-byte
// boundary of the dynamic shared memory, and the kernel checks that the
// padding this costs fits
constexpr int kAttnSmem = 232448;
static_assert(kTilesBytes + kSmallBytes <= uint32_t(kAttnSmem), "shared memory layout too large");
constexpr int kSlotFloats = kAttnSlotFloats;
constexpr int kSlotStats = 128 * 64;  // floats before (m, l) in a slot: 128 x 128 bf16 partial O
constexpr int kMaxContrib = 8;        // partials a finishing CTA may combine
// Register split: the launch gives every thread kLaunchRegs; warpgroup 0
// (producer, issuer, allocator) drops to kCtlRegs, the epilogue warpgroup to
// kEpiRegs, and the two softmax warpgroups rise to kSoftmaxRegs.  The sum
// over the CTA must not exceed 512 * kLaunchRegs, or setmaxnreg.inc would wait
// forever; the launcher refuses to run unless the compiled kernel has exactly
// kLaunchRegs.  80 / 64 / 184 measured fastest on the 1560-token frame (357
// TFLOP/s against 338 with 56 / 72 / 192): the issuer spills less.
// Of every 16 exp2 pairs of a full tile, this many run on the FMA pipe
// (exp2_poly) instead of the MUFU.  Measured on the 1560-token frame: 0 is
// fastest (342 TFLOP/s against 320 with 5), the softmax being bound by issue
// and latency rather than by the MUFU, so the option stays off.
constexpr int kPolyPairs = 0;
constexpr int kLaunchRegs = 128;
constexpr int kCtlRegs = 80;
constexpr int kEpiRegs = 64;
constexpr int kSoftmaxRegs = 184;
static_assert(128 * kCtlRegs + 128 * kEpiRegs + 256 * kSoftmaxRegs <= kAttnThreads * kLaunchRegs,
              "register split too large");

enum {
  B_QF = 0,           // [2] Q sub-tile loaded
  B_QE = 2,           // [2] Q sub-tile free (its last MMA completed)
  B_RF = 4,           // [kRing] ring slot loaded
  B_RE = 4 + kRing,   // [kRing] ring slot free
  B_SF = 4 + 2 * kRing,  // [2] S of the current key tile in tensor memory
  B_PF = B_SF + 2,    // [2] P written (4 softmax warps)
  B_ST = B_PF + 2,    // [2] softmax statistics of the segment in shared memory (4 warps)
  B_SD = B_ST + 2,    // [2] every MMA of the segment completed
  B_ES = B_SD + 2,    // [2] epilogue done with the S columns (X read, or nothing to read) (4 warps)
  B_EO = B_ES + 2,    // [2] epilogue has read O from tensor memory (4 warps)
  B_PRE = B_EO + 2,   // [2] contributors' flags acquired (1 arrival; once per launch)
  B_PD = B_PRE + 2,   // [2] contributors' partials in shared memory (1 arrival + bulk-copy bytes; once per launch)
  B_DRAIN = B_PD + 2,
  B_COUNT
};

// Named barriers (id 0 is __syncthreads).
enum { NB_EPI = 1 };

// ------------------------------------------------------------------ partition
// Units are (block, key tile) pairs in (stream, head, block, key tile) order;
// the host cuts them into equal per-CTA ranges (AttnParams::range).
struct Seg {
  int bh, blk, j0, j1;
};

__device__ __forceinline__ bool next_seg(const AttnParams& p, unsigned& u, unsigned u_end, Seg& s) {
  if (u >= u_end) return false;
  const unsigned per = unsigned(p.n_blk) * unsigned(p.nkv);
  s.bh = int(u / per);
  const unsigned r = u - unsigned(s.bh) * per;
  s.blk = int(r / unsigned(p.nkv));
  s.j0 = int(r - unsigned(s.blk) * unsigned(p.nkv));
  s.j1 = int(min(unsigned(p.nkv), unsigned(s.j0) + (u_end - u)));
  u += unsigned(s.j1 - s.j0);
  return true;
}

__device__ __forceinline__ void named_bar(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_release(unsigned* p, unsigned v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ float bf16_lo(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t x) { return __uint_as_float(x & 0xFFFF0000u); }

// Byte offset of 16-byte chunk c (8 bf16, columns 8c..8c+7) of row r in a
// 128-row x 128-column tile stored as two 64-column boxes in the 128-byte
// swizzle layout (the layout TMA reads and writes for these tensor maps).
__device__ __forceinline__ uint32_t sw128_chunk(int r, int c) {
  return uint32_t(c >> 3) * kHalf + uint32_t(r) * 128 + uint32_t(((c & 7) ^ (r & 7)) << 4);
}

// Number of CTAs after `cta` whose first segment continues block (bh, blk).
// Every CTA's range is non-empty (the host gives each at least a sixth of a
// block), so they are CTAs cta + 1 .. cta + n.  Returns -1 if the block's
// pieces do not end within kMaxContrib contributors (the host rules that out).
__device__ __forceinline__ int contributors(const AttnParams& p, int cta, const Seg& s) {
  const unsigned block_end = (unsigned(s.bh) * unsigned(p.n_blk) + unsigned(s.blk) + 1u) * unsigned(p.nkv);
  int n = 0;
  while (cta + 1 + n < p.grid && p.range[cta + 1 + n] < block_end) ++n;
  return n <= kMaxContrib ? n : -1;
}

// Scratch slot of sub-tile `sub` of CTA c.
__device__ __forceinline__ float* slot_of(const AttnParams& p, int c, int sub) {
  return p.scratch + (size_t(c) * 2 + sub) * kSlotFloats;
}

// Wait (one thread) until a phase of `bar` completes; bounded like mbar_wait.
__device__ __forceinline__ bool wait1(uint64_t* bar, uint32_t parity, const WaitCtl& w) {
  return mbar_wait(bar, parity, w);
}

// ------------------------------------------------------------------ producer
// One thread.  Per segment: the first K/V tiles, Q of both sub-tiles (once the
// previous segment's MMAs have released them), the remaining K/V tiles and,
// for blocks this CTA finishes, MqT -- all through the 4-slot ring in the
// order the issuer consumes them.  The next segment's Q tiles are prefetched
// into L2 as soon as the current segment starts.
__device__ __forceinline__ void producer(const AttnParams& p, uint64_t* bars, uint8_t* sQ, uint8_t* sR,
                                         const CUtensorMap* tm_q, const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                                         const CUtensorMap* tm_mq, const unsigned u_begin, const unsigned u_end,
                                         const WaitCtl& w) {
  uint32_t ring = 0, q_use[2] = {0, 0};
  unsigned u = u_begin;
  Seg s;
  while (next_seg(p, u, u_end, s)) {
    const int b = s.bh / p.heads, h = s.bh % p.heads;
    const bool has_b = s.blk < p.n_pair;
    const int qt_a = has_b ? 2 * s.blk : p.n_qt - 1;
    const bool writer = s.j0 == 0;
    const int n = s.j1 - s.j0;
    const int ntiles = 2 * n + ((writer && p.has_inter) ? 1 : 0);
    const int x0 = h * 128;
    auto prefetch_next_q = [&]() {  // L2 prefetch of the next segment's Q tiles
      unsigned u2 = u;
      Seg s2;
      if (next_seg(p, u2, u_end, s2)) {
        const bool hb2 = s2.blk < p.n_pair;
        const int qt2 = hb2 ? 2 * s2.blk : p.n_qt - 1;
        for (int sub = 0; sub < (hb2 ? 2 : 1); ++sub) {
          tma_prefetch_l2_3d(tm_q, (s2.bh % p.heads) * 128, (qt2 + sub) * 128, s2.bh / p.heads);
          tma_prefetch_l2_3d(tm_q, (s2.bh % p.heads) * 128 + 64, (qt2 + sub) * 128, s2.bh / p.heads);
        }
      }
    };
    auto put = [&](int t) -> bool {
      const uint32_t slot = ring % kRing;
      if (ring >= kRing && !wait1(&bars[B_RE + slot], ((ring / kRing) - 1) & 1, w)) return false;
      uint8_t* dst = sR + slot * kTile;
      mbar_expect_tx(&bars[B_RF + slot], kTile);
      if (t < 2 * n) {
        const int j = s.j0 + (t >> 1);
        const CUtensorMap* m = (t & 1) ? tm_v : tm_k;
        tma_load_3d(dst, m, &bars[B_RF + slot], x0, j * 128, b);
        tma_load_3d(dst + kHalf, m, &bars[B_RF + slot], x0 + 64, j * 128, b);
      } else {
        tma_load_3d(dst, tm_mq, &bars[B_RF + slot], 0, 0, s.bh);
        tma_load_3d(dst + kHalf, tm_mq, &bars[B_RF + slot], 64, 0, s.bh);
      }
      ++ring;
      return true;
    };
    auto load_q = [&](int sub) -> bool {
      if (q_use[sub] > 0 && !wait1(&bars[B_QE + sub], (q_use[sub] - 1) & 1, w)) return false;
      uint8_t* dst = sQ + sub * kTile;
      const int row = (qt_a + sub) * 128;
      mbar_expect_tx(&bars[B_QF + sub], kTile);
      tma_load_3d(dst, tm_q, &bars[B_QF + sub], x0, row, b);
      tma_load_3d(dst + kHalf, tm_q, &bars[B_QF + sub], x0 + 64, row, b);
      ++q_use[sub];
      return true;
    };
    if (q_use[0] == 0) {
      // The launch's first segment: every CTA starts at once and its first
      // tiles come from HBM, so only what the first MMA needs (K_j0 and Q of
      // sub-tile A) is requested until it has landed; V_j0, Q of sub-tile B,
      // the next tiles and the L2 prefetch follow.
      if (!put(0) || !load_q(0)) return;
      if (!wait1(&bars[B_QF + 0], 0, w)) return;
      if (!put(1)) return;
      if (has_b && !load_q(1)) return;
      prefetch_next_q();
      for (int t = 2; t < ntiles; ++t)
        if (!put(t)) return;
      continue;
    }
    prefetch_next_q();
    const int pre = min(2, ntiles);
    for (int t = 0; t < pre; ++t)
      if (!put(t)) return;
    for (int sub = 0; sub < (has_b ? 2 : 1); ++sub)
      if (!load_q(sub)) return;
    for (int t = pre; t < ntiles; ++t)
      if (!put(t)) return;
  }
}

// ------------------------------------------------------------------ MMA issuer
// tcgen05.mma has almost no issue queue: an instruction is accepted about when
// the previous one finishes, so any work between two MMAs of a group stalls
// the tensor pipe.  The groups below are fully unrolled with compile-time
// descriptor offsets.
__device__ __forceinline__ void mma_ss_lo(const uint32_t d, const uint32_t a_lo, const uint32_t b_lo,
                                          const uint32_t hi, const uint32_t idesc, const uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 da, db;\n\t"
      "setp.ne.b32 p, %5, 0;\n\t"
      "mov.b64 da, {%1, %3};\n\t"
      "mov.b64 db, {%2, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %4, p;\n\t}" ::"r"(d),
      "r"(a_lo), "r"(b_lo), "r"(hi), "r"(idesc), "r"(acc));
}

__device__ __forceinline__ void mma_ts_lo(const uint32_t d, const uint32_t a_tmem, const uint32_t b_lo,
                                          const uint32_t hi, const uint32_t idesc, const uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 db;\n\t"
      "setp.ne.b32 p, %5, 0;\n\t"
      "mov.b64 db, {%2, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], db, %4, p;\n\t}" ::"r"(d),
      "r"(a_tmem), "r"(b_lo), "r"(hi), "r"(idesc), "r"(acc));
}

// S (or X) = A B^T over K = 128 (eight 16-deep steps): both operands K-major
// 128 x 128 tiles, given by the low words of their descriptors.
__device__ __forceinline__ void mma_s_group(const uint32_t d, const uint32_t a_lo, const uint32_t b_lo,
                                            const uint32_t hi, const uint32_t idesc) {
  constexpr uint32_t kHalf16 = kHalf >> 4;
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const uint32_t off = (kk >> 2) * kHalf16 + (kk & 3) * 2;
    mma_ss_lo(d, a_lo + off, b_lo + off, hi, idesc, kk > 0);
  }
}

// O (+)= P V_j for nk 16-key steps (8 on every key tile but a ragged last one).
__device__ __forceinline__ void mma_pv_group(const uint32_t d, const uint32_t p_tmem, const uint32_t v_lo,
                                             const uint32_t hi, const uint32_t idesc, const int nk, const bool acc0) {
  if (nk == 8) {
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) mma_ts_lo(d, p_tmem + kk * 8, v_lo + kk * 128, hi, idesc, kk > 0 || acc0);
  } else {
    for (int kk = 0; kk < nk; ++kk) mma_ts_lo(d, p_tmem + kk * 8, v_lo + kk * 128, hi, idesc, kk > 0 || acc0);
  }
}

// One thread.  Order per key tile t, with sub-tile B one tile behind A:
//     S_A(t), PV_B(t-1), S_B(t), PV_A(t)
// so that each softmax warpgroup has two MMA groups' time to produce P.  An S
// MMA is issued right after the PV that reads the P it overwrites: tcgen05.mma
// operations of one thread execute in issue order.  A sub-tile's first S MMA of
// a segment waits until the epilogue is done with its S columns (where X of
// the previous segment may lie), its first PV until the epilogue has read O.
__device__ __forceinline__ void mma_issuer(const AttnParams& p, uint64_t* bars, const uint32_t tmem,
                                           const uint32_t q_addr, const uint32_t r_addr, const unsigned u_begin,
                                           const unsigned u_end, const WaitCtl& w) {
  constexpr uint32_t kTile16 = kTile >> 4;  // descriptor address units
  const uint32_t id_o = idesc_bf16(128, 128, 0, 1);                 // P (TMEM) x V (MN-major)
  const uint32_t id_x = idesc_bf16(128, 128, 0, 0);
  // Every operand descriptor shares its high word (stride, version, swizzle);
  // only the low word (start address, leading offset) differs.
  const uint64_t dq64 = smem_desc_sw128(q_addr, 16, 1024);
  const uint32_t hi = uint32_t(dq64 >> 32);
  const uint32_t dqa = uint32_t(dq64), dqb = dqa + kTile16;
  const uint32_t dr0 = uint32_t(smem_desc_sw128(r_addr, 16, 1024));     // K-major ring tile
  const uint32_t dv0 = uint32_t(smem_desc_sw128(r_addr, kHalf, 1024));  // MN-major ring tile
  const uint32_t tSA = tmem, tSB = tmem + 128, tOA = tmem + 256, tOB = tmem + 384;
  uint32_t ring = 0, qa_use = 0, qb_use = 0, ita = 0, itb = 0, sega = 0, segb = 0;
  unsigned u = u_begin;
  Seg s;
  while (next_seg(p, u, u_end, s)) {
    const bool has_b = s.blk < p.n_pair;
    const int n = s.j1 - s.j0;
    if (!wait1(&bars[B_QF + 0], qa_use & 1, w)) return;
    ++qa_use;
    if (sega > 0 && !wait1(&bars[B_ES + 0], (sega - 1) & 1, w)) return;
    tc_fence_after();
    uint32_t vprev = 0;
    int nk_prev = 0;
    for (int t = 0; t < n; ++t) {
      const int valid = min(128, p.kv_len - (s.j0 + t) * 128);
      const uint32_t id_s = idesc_bf16(128, min(128, (valid + 15) & ~15), 0, 0);
      const int nk = (valid + 15) >> 4;
      const uint32_t kslot = ring & (kRing - 1);
      const uint32_t vslot = (ring + 1) & (kRing - 1);
      const uint32_t dk = dr0 + kslot * kTile16, dvv = dv0 + vslot * kTile16, dvp = dv0 + vprev * kTile16;
      if (!wait1(&bars[B_RF + kslot], (ring / kRing) & 1, w)) return;
      mma_s_group(tSA, dqa, dk, hi, id_s);
      mma_commit(&bars[B_SF + 0]);
      if (has_b) {
        if (t > 0) {
          if (!wait1(&bars[B_PF + 1], itb & 1, w)) return;
          ++itb;
          if (t == 1 && segb > 0 && !wait1(&bars[B_EO + 1], (segb - 1) & 1, w)) return;
          tc_fence_after();
          mma_pv_group(tOB, tSB, dvp, hi, id_o, nk_prev, t > 1);
          mma_commit(&bars[B_RE + vprev]);
        } else {  // sub-tile B's Q, and its tensor memory back from the epilogue
          if (!wait1(&bars[B_QF + 1], qb_use & 1, w)) return;
          ++qb_use;
          if (segb > 0 && !wait1(&bars[B_ES + 1], (segb - 1) & 1, w)) return;
          tc_fence_after();
        }
        mma_s_group(tSB, dqb, dk, hi, id_s);
        mma_commit(&bars[B_SF + 1]);
      }
      mma_commit(&bars[B_RE + kslot]);
      if (!wait1(&bars[B_RF + vslot], ((ring + 1) / kRing) & 1, w)) return;
      ring += 2;
      if (!wait1(&bars[B_PF + 0], ita & 1, w)) return;
      ++ita;
      if (t == 0 && sega > 0 && !wait1(&bars[B_EO + 0], (sega - 1) & 1, w)) return;
      tc_fence_after();
      mma_pv_group(tOA, tSA, dvv, hi, id_o, nk, t > 0);
      if (!has_b) mma_commit(&bars[B_RE + vslot]);
      vprev = vslot;
      nk_prev = nk;
    }
    if (has_b) {
      if (!wait1(&bars[B_PF + 1], itb & 1, w)) return;
      ++itb;
      if (n == 1 && segb > 0 && !wait1(&bars[B_EO + 1], (segb - 1) & 1, w)) return;
      tc_fence_after();
      mma_pv_group(tOB, tSB, dv0 + vprev * kTile16, hi, id_o, nk_prev, n > 1);
      mma_commit(&bars[B_RE + vprev]);
    }
    if (s.j0 == 0 && p.has_inter) {  // X = Q MqT^T for the rows this CTA finishes
      const uint32_t mslot = ring & (kRing - 1);
      if (!wait1(&bars[B_RF + mslot], (ring / kRing) & 1, w)) return;
      ++ring;
      const uint32_t dm = dr0 + mslot * kTile16;
      mma_s_group(tSA, dqa, dm, hi, id_x);
      if (has_b) mma_s_group(tSB, dqb, dm, hi, id_x);
      mma_commit(&bars[B_RE + mslot]);
    }
    mma_commit(&bars[B_SD + 0]);
    mma_commit(&bars[B_QE + 0]);
    if (has_b) {
      mma_commit(&bars[B_SD + 1]);
      mma_commit(&bars[B_QE + 1]);
    }
    ++sega;
    if (has_b) ++segb;
  }
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const WaitCtl& w) {
  bool ok = mbar_wait(bar, parity, w);
  return __all_sync(0xffffffffu, ok);
}

// 16-byte chunk `i` (columns 8i..8i+7) of row `row` of a partial (chunk-major).
__device__ __forceinline__ uint4 partial_chunk(const uint8_t* base, const int i, const int row) {
  return reinterpret_cast<const uint4*>(base)[i * 128 + row];
}

__device__ __forceinline__ void add_chunk(float* v, const uint4 x, const float wgt) {
  const uint32_t x4[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    v[2 * e] = fmaf(bf16_lo(x4[e]), wgt, v[2 * e]);
    v[2 * e + 1] = fmaf(bf16_hi(x4[e]), wgt, v[2 * e + 1]);
  }
}

// Shared-memory place of partial k of sub-tile s of a split block
// (chunk-major, as in the scratch slot): the first one in the staging buffer,
// the others in the K/V ring once the CTA's last MMA has released it.
__device__ __forceinline__ const uint8_t* part_slot(const uint8_t* stage, const uint8_t* ring, int s, int k) {
  return (s == 0 && k == 0) ? stage : ring + (s == 0 ? 0 : 1 + k) * kTile;
}

// The last segment of a CTA whose block continues in the next CTAs (a split
// writer), for one sub-tile, run by that sub-tile's softmax warpgroup once its
// last P is out: O = sum over pieces of (weight x normalised piece) + X, the
// pieces being this CTA's accumulator and the contributors' partials, weighted
// by l * 2^(m - M) / sum(l * 2^(m - M)) with M the largest m.  The output goes
// through the sub-tile's own Q buffer (free: nothing is loaded after the last
// segment) as per-warp 32-row boxes written by TMA tile stores.
__device__ __forceinline__ bool split_epilogue(const AttnParams& p, uint64_t* bars, const uint8_t* stage,
                                               const uint8_t* ring, uint8_t* obox, const CUtensorMap* tm_o,
                                               const uint32_t tmem, const int cta, const int sub, const int quarter,
                                               const int lane, const Seg& s, const int n_contrib, const float m,
                                               const float l, const uint32_t sd_parity, const WaitCtl& w) {
  const int row = quarter * 32 + lane;
  const uint32_t lane_off = uint32_t(quarter * 32) << 16;
  const uint32_t tS = tmem + sub * 128, tO = tmem + 256 + sub * 128;
  const bool has_b = s.blk < p.n_pair;
  const int qt = (has_b ? 2 * s.blk : p.n_qt - 1) + sub;
  const bool row_ok = qt * 128 + row < p.q_len;
  const bool warp_on = qt * 128 + quarter * 32 < p.q_len;  // warp-uniform
  const int b = s.bh / p.heads, h = s.bh % p.heads;
  const bool use_intra = !(p.flags & 2u);
  const bool use_inter = p.has_inter && !(p.flags & 1u);
  const bool in_smem = n_contrib <= 2;
  // The contributors' flags are acquired (by the epilogue warpgroup): their
  // statistics are read from global memory while the last MMAs may still run.
  if (!warp_wait(&bars[B_PRE + sub], 0, w)) return false;
  float a_self = 0.f, wk[kMaxContrib];
#pragma unroll
  for (int k = 0; k < kMaxContrib; ++k) wk[k] = 0.f;
  if (row_ok) {
    float mk[kMaxContrib], lk[kMaxContrib];
#pragma unroll
    for (int k = 0; k < kMaxContrib; ++k) {
      mk[k] = -INFINITY;
      lk[k] = 0.f;
      if (k < n_contrib) {
        const float* st = slot_of(p, cta + 1 + k, sub) + kSlotStats;
        mk[k] = st[row];
        lk[k] = st[128 + row];
      }
    }
    float M = m;
#pragma unroll
    for (int k = 0; k < kMaxContrib; ++k) M = fmaxf(M, mk[k]);
    const float e_self = fast_exp2(m - M);
    float L = l * e_self;
#pragma unroll
    for (int k = 0; k < kMaxContrib; ++k) {
      wk[k] = k < n_contrib ? lk[k] * fast_exp2(mk[k] - M) : 0.f;
      L += wk[k];
    }
    const float inv = 1.f / L;
    a_self = e_self * inv;
#pragma unroll
    for (int k = 0; k < kMaxContrib; ++k) wk[k] *= inv;
  }
  if (!warp_wait(&bars[B_SD + sub], sd_parity, w)) return false;
  if (!warp_wait(&bars[B_PD + sub], 0, w)) return false;
  tc_fence_after();
  uint8_t* wbox = obox + quarter * 8192;
  if (warp_on) {
    const float2 as2 = make_float2(use_intra ? a_self : 0.f, use_intra ? a_self : 0.f);
#pragma unroll 1
    for (int q = 0; q < 4; ++q) {  // 32 columns at a time
      uint32_t ro[32], rx[32];
      tmem_ld32(tO + lane_off + q * 32, ro);
      if (use_inter) tmem_ld32(tS + lane_off + q * 32, rx);
      tmem_wait_ld();
      float2* v = reinterpret_cast<float2*>(ro);
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] = __fmul2_rn(v[i], as2);
      if (use_intra) {
#pragma unroll
        for (int k = 0; k < kMaxContrib; ++k) {
          if (k < n_contrib) {
            const uint8_t* base = in_smem ? part_slot(stage, ring, sub, k)
                                          : reinterpret_cast<const uint8_t*>(slot_of(p, cta + 1 + k, sub));
            const float2 w2 = make_float2(wk[k], wk[k]);
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
              const uint4 x = partial_chunk(base, q * 4 + ch, row);
              const uint32_t x4[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
              for (int e = 0; e < 4; ++e)
                v[4 * ch + e] = __ffma2_rn(make_float2(bf16_lo(x4[e]), bf16_hi(x4[e])), w2, v[4 * ch + e]);
            }
          }
        }
      }
      if (use_inter) {
        const float2* x2 = reinterpret_cast<const float2*>(rx);
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = __fadd2_rn(v[i], x2[i]);
      }
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        const int c16 = q * 4 + ch;  // 16-byte chunk of the row: box c16 / 8, chunk c16 % 8 swizzled by row
        *reinterpret_cast<uint4*>(wbox + (c16 >> 3) * 4096 + lane * 128 + (((c16 & 7) ^ (lane & 7)) << 4)) =
            make_uint4(pack_bf16x2(v[4 * ch + 0].x, v[4 * ch + 0].y), pack_bf16x2(v[4 * ch + 1].x, v[4 * ch + 1].y),
                       pack_bf16x2(v[4 * ch + 2].x, v[4 * ch + 2].y), pack_bf16x2(v[4 * ch + 3].x, v[4 * ch + 3].y));
      }
    }
  }
  tc_fence_before();
  fence_async_smem();
  __syncwarp();
  if (lane == 0) {
    mbar_arrive(&bars[B_ES + sub]);
    mbar_arrive(&bars[B_EO + sub]);
    if (warp_on) {
      tma_store_3d(tm_o, wbox, h * 128, qt * 128 + quarter * 32, b);
      tma_store_3d(tm_o, wbox + 4096, h * 128 + 64, qt * 128 + quarter * 32, b);
      bulk_commit();
      bulk_wait_read0();  // the box is read before the CTA's shared memory goes away
    }
  }
  __syncwarp();
  return true;
}

// ------------------------------------------------------------------ softmax
// One warpgroup per sub-tile, one query row per thread.  Per key tile: the
// whole 128-column row of S from tensor memory; its maximum; lazy rescaling
// (the running max m moves only when the tile's max exceeds it by more than
// 8, a factor 256, so P stays <= 256 and O is rescaled rarely); P =
// 2^(S * scale * log2(e) - m) packed to bf16 pairs over S's first 64 columns;
// the running row sum l.  At the end of a segment, (m, l) go to shared memory
// for the epilogue.
__device__ __forceinline__ void softmax_role(const AttnParams& p, uint64_t* bars, float* stats, const uint8_t* stage,
                                             const uint8_t* ring, uint8_t* qbuf, const CUtensorMap* tm_o,
                                             const uint32_t tmem, const int cta, const int sub, const int quarter,
                                             const int lane, const unsigned u_begin, const unsigned u_end,
                                             const WaitCtl& w) {
  const int row = quarter * 32 + lane;
  const uint32_t lane_off = uint32_t(quarter * 32) << 16;
  const uint32_t tS = tmem + sub * 128, tO = tmem + 256 + sub * 128;
  const float sl2 = p.scale_log2;
  uint32_t it = 0, nseg = 0;
  unsigned u = u_begin;
  Seg s;
  while (next_seg(p, u, u_end, s)) {
    const bool has_b = s.blk < p.n_pair;
    if (sub == 1 && !has_b) continue;
    ++nseg;
    const int qt = (has_b ? 2 * s.blk : p.n_qt - 1) + sub;
    const bool warp_on = qt * 128 + quarter * 32 < p.q_len;  // warp-uniform
    float m = -INFINITY, l = 0.f;
    for (int t = 0; t < s.j1 - s.j0; ++t) {
      if (!warp_wait(&bars[B_SF + sub], it & 1, w)) return;
      tc_fence_after();
      const int valid = min(128, p.kv_len - (s.j0 + t) * 128);
      if (warp_on) {
        uint32_t r[128];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tS + lane_off + c * 32, slice32(r, c));
        tmem_wait_ld();
        if (valid < 128) {
#pragma unroll
          for (int i = 0; i < 128; ++i)
            if (i >= valid) r[i] = __float_as_uint(-INFINITY);
        }
        // row max over four independent chains of three-input maxima
        float m4[4];
#pragma unroll
        for (int k = 0; k < 4; ++k)
          m4[k] = fmax3(__uint_as_float(r[k]), __uint_as_float(r[4 + k]), __uint_as_float(r[8 + k]));
#pragma unroll
        for (int i = 12; i < 124; i += 8)
#pragma unroll
          for (int k = 0; k < 4; ++k) m4[k] = fmax3(m4[k], __uint_as_float(r[i + k]), __uint_as_float(r[i + 4 + k]));
#pragma unroll
        for (int k = 0; k < 4; ++k) m4[k] = fmaxf(m4[k], __uint_as_float(r[124 + k]));
        const float mx = fmaxf(fmax3(m4[0], m4[1], m4[2]), m4[3]) * sl2;
        float f = 1.f;
        bool any_rescale = false;
        if (t == 0) {
          m = mx;
        } else {
          const bool need = mx > m + 8.f;
          any_rescale = __any_sync(0xffffffffu, need);
          if (need) {
            f = fast_exp2(m - mx);
            m = mx;
          }
        }
        // P = exp2(S * scale * log2(e) - m), packed to bf16 pairs over S's first 64
        // columns.  On full tiles kPolyPairs of every 16 pairs take the FMA-pipe
        // exp2 so that the MUFU is not the limit; the masked last tile (columns at
        // -inf) takes the MUFU for all of them.
        const float2 sc = make_float2(sl2, sl2), nm = make_float2(-m, -m);
        float2 s2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        if (valid == 128) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float2 x = __ffma2_rn(
                  make_float2(__uint_as_float(r[c * 32 + 2 * i]), __uint_as_float(r[c * 32 + 2 * i + 1])), sc, nm);
              float2 e;
              if (i >= 16 - kPolyPairs) {  // x <= 8: the lazy max is at most 8 below the row max
                e = make_float2(exp2_poly(x.x), exp2_poly(x.y));
              } else {
                e = make_float2(fast_exp2(x.x), fast_exp2(x.y));
              }
              s2[i & 3] = __fadd2_rn(s2[i & 3], e);
              pk[i] = pack_bf16x2(e.x, e.y);
            }
            tmem_st16(tS + lane_off + c * 16, pk);
          }
        } else {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float2 x = __ffma2_rn(
                  make_float2(__uint_as_float(r[c * 32 + 2 * i]), __uint_as_float(r[c * 32 + 2 * i + 1])), sc, nm);
              const float2 e = make_float2(fast_exp2(x.x), fast_exp2(x.y));
              s2[i & 3] = __fadd2_rn(s2[i & 3], e);
              pk[i] = pack_bf16x2(e.x, e.y);
            }
            tmem_st16(tS + lane_off + c * 16, pk);
          }
        }
        const float2 s01 = __fadd2_rn(s2[0], s2[1]), s23 = __fadd2_rn(s2[2], s2[3]);
        const float2 sa = __fadd2_rn(s01, s23);
        l = fmaf(l, f, sa.x + sa.y);
        tmem_wait_st();
        if (any_rescale) {  // rare: O is rescaled before P is signalled, so PV sees a consistent O
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t o[32];
            tmem_ld32(tO + lane_off + c * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
            tmem_st32(tO + lane_off + c * 32, o);
          }
          tmem_wait_st();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[B_PF + sub]);
      ++it;
    }
    stats[(sub * 2 + 0) * 128 + row] = m;
    stats[(sub * 2 + 1) * 128 + row] = l;
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars[B_ST + sub]);
    if (s.j0 == 0 && s.j1 < p.nkv) {  // a split writer: always this CTA's last segment
      const int n_contrib = contributors(p, cta, s);
      if (n_contrib > 0 && !split_epilogue(p, bars, stage, ring, qbuf + sub * kTile, tm_o, tmem, cta, sub, quarter,
                                           lane, s, n_contrib, m, l, (nseg - 1) & 1, w))
        return;
    }
  }
}

// ------------------------------------------------------------------ epilogue
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// Contributor: this CTA's rows of a block another CTA finishes.  The output
// normalised by its own l goes to this CTA's slot as bf16 in chunk-major order
// (16-byte chunk i of row r at uint4 index i * 128 + r, so a warp's store is
// one contiguous 512-byte span), then (m, l).
__device__ __forceinline__ void store_partial(const AttnParams& p, float* slot, const uint32_t tO,
                                              const uint32_t lane_off, const int row, const bool row_ok,
                                              const bool warp_on, const float m, const float l) {
  uint4* d4 = reinterpret_cast<uint4*>(slot) + row;
  const float inv = row_ok ? 1.f / l : 0.f;
  if (warp_on) {
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      uint32_t r[32];
      tmem_ld32(tO + lane_off + c * 32, r);
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t* q = r + 8 * i;
        d4[(4 * c + i) * 128] = make_uint4(pack_bf16x2(__uint_as_float(q[0]) * inv, __uint_as_float(q[1]) * inv),
                                           pack_bf16x2(__uint_as_float(q[2]) * inv, __uint_as_float(q[3]) * inv),
                                           pack_bf16x2(__uint_as_float(q[4]) * inv, __uint_as_float(q[5]) * inv),
                                           pack_bf16x2(__uint_as_float(q[6]) * inv, __uint_as_float(q[7]) * inv));
      }
    }
  }
  if (row_ok) {
    slot[kSlotStats + row] = m;
    slot[kSlotStats + 128 + row] = l;
  }
}

// One warpgroup, one query row per thread, for both sub-tiles in turn.  At the
// end of a segment (its MMAs done, the softmax statistics in shared memory):
//  * a segment that does not start at key tile 0 (a contributor) stores its
//    partial (store_partial) for both sub-tiles, then raises the slots' ready
//    flags;
//  * a segment holding a whole block writes O / l (+ X) through per-warp
//    staging boxes and TMA tile stores;
//  * a segment that starts a block continued by the next CTAs (always the
//    CTA's last segment) only brings the contributors' partials into shared
//    memory; the softmax warpgroups combine them (split_epilogue).
// Tensor memory is handed back to the issuer as soon as it has been read: the
// S columns (B_ES) at once when they hold no X, the O columns (B_EO) after O.
__device__ __forceinline__ bool epilogue_role(const AttnParams& p, uint64_t* bars, const float* stats, uint8_t* stage,
                                              uint8_t* ring, const CUtensorMap* tm_o, const uint32_t tmem,
                                              const int cta, const int quarter,
                                              const int lane, const unsigned u_begin, const unsigned u_end,
                                              volatile int* abort_flag, const WaitCtl& w) {
  const int row = quarter * 32 + lane;
  const int et = threadIdx.x - 3 * 128;  // 0..127
  const uint32_t lane_off = uint32_t(quarter * 32) << 16;
  const bool use_intra = !(p.flags & 2u);
  const bool use_inter = p.has_inter && !(p.flags & 1u);
  uint32_t segc[2] = {0, 0};
  bool staged = false;  // this warp may have a tile store reading its staging boxes
  unsigned u = u_begin;
  Seg s;
  while (next_seg(p, u, u_end, s)) {
    const bool has_b = s.blk < p.n_pair;
    const int nsub = has_b ? 2 : 1;
    const int b = s.bh / p.heads, h = s.bh % p.heads;
    const bool writer = s.j0 == 0, full = writer && s.j1 == p.nkv;
    int n_contrib = 0;
    if (writer && !full && (n_contrib = contributors(p, cta, s)) < 0) {
      record_error(p.err, kDevBadShape);  // the host partition rules this out
      *abort_flag = 1;
      return false;
    }
    if (n_contrib > 0) {
      // Split block (this CTA's last segment): acquire the contributors' flags
      // (B_PRE: the softmax warpgroups may then read the contributors'
      // statistics), then bring their partials into shared memory with bulk
      // copies for the combine in split_epilogue (B_PD): the first partial of
      // sub-tile A into the staging buffer at once, the others into the K/V
      // ring once the CTA's last MMA has released it.  With more than two
      // contributors the combine reads the partials from global memory.
      const bool in_smem = n_contrib <= 2;
      if (lane == 0 && staged) bulk_wait_read0();  // earlier tile stores have read the staging buffer
      named_bar(NB_EPI, 128);
      if (et == 0) {
        for (int s2 = 0; s2 < nsub; ++s2)
          for (int k = 0; k < n_contrib && !*abort_flag; ++k) {
            const unsigned* f = p.ready + (cta + 1 + k) * 2 + s2;
            const uint64_t t0 = global_timer_ns();
            while (ld_acquire(f) == 0u) {
              if (*abort_flag || global_timer_ns() - t0 > p.wait_limit_ns) {
                *abort_flag = 1;
                record_error(p.err, kDevTimeout);
                break;
              }
            }
          }
        if (!*abort_flag) {
          fence_async_global();
          for (int s2 = 0; s2 < nsub; ++s2) {
            mbar_arrive(&bars[B_PRE + s2]);
            mbar_expect_tx(&bars[B_PD + s2], in_smem ? uint32_t(n_contrib) * kTile : 0u);
          }
          if (in_smem) {
            bulk_load(stage, slot_of(p, cta + 1, 0), kTile, &bars[B_PD + 0]);
            if (n_contrib > 1 || nsub > 1) {
              if (wait1(&bars[B_SD + nsub - 1], segc[nsub - 1] & 1, w)) {  // the ring is idle from here on
                for (int s2 = 0; s2 < nsub; ++s2)
                  for (int k = (s2 == 0 ? 1 : 0); k < n_contrib; ++k)
                    bulk_load(const_cast<uint8_t*>(part_slot(stage, ring, s2, k)), slot_of(p, cta + 1 + k, s2), kTile,
                              &bars[B_PD + s2]);
              }
            }
          }
        }
      }
      __syncwarp();
      if (*abort_flag) return false;
      // once the combine has read the partials (it arrives on B_ES), their flags
      // go back to zero for the next launch
      for (int s2 = 0; s2 < nsub; ++s2)
        if (!warp_wait(&bars[B_ES + s2], segc[s2] & 1, w)) return false;
      if (et == 0)
        for (int s2 = 0; s2 < nsub; ++s2)
          for (int k = 0; k < n_contrib; ++k) p.ready[(cta + 1 + k) * 2 + s2] = 0u;
      continue;  // the last segment: nothing else for this warpgroup
    }
    for (int sub = 0; sub < nsub; ++sub) {
      if (!warp_wait(&bars[B_SD + sub], segc[sub] & 1, w)) return false;
      if (!warp_wait(&bars[B_ST + sub], segc[sub] & 1, w)) return false;
      ++segc[sub];
      tc_fence_after();
      const int qt = (has_b ? 2 * s.blk : p.n_qt - 1) + sub;
      const int q_row = qt * 128 + row;
      const bool row_ok = q_row < p.q_len;
      const bool warp_on = qt * 128 + quarter * 32 < p.q_len;  // warp-uniform
      const float m = stats[(sub * 2 + 0) * 128 + row], l = stats[(sub * 2 + 1) * 128 + row];
      const uint32_t tS = tmem + sub * 128, tO = tmem + 256 + sub * 128;
      if (!writer) {  // ------------------------------------------------ contributor
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[B_ES + sub]);  // the S columns hold nothing for the epilogue
        store_partial(p, slot_of(p, cta, sub), tO, lane_off, row, row_ok, warp_on, m, l);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[B_EO + sub]);
        if (sub == nsub - 1) {  // both partials written: publish them
          __threadfence();
          named_bar(NB_EPI, 128);
          if (et < nsub) st_release(p.ready + cta * 2 + et, 1u);
        }
        continue;
      }
      // ------------------------------------------------------------------ writer
      // A whole block: O / l (+ X).
      const float a_self = row_ok ? 1.f / l : 0.f;
      // Output rows go through this warp's 8 KB of a staging area: two boxes of
      // 32 rows x 64 columns in the 128-byte swizzle layout, written out by two
      // TMA tile stores (rows past the frame are not written).  A split block
      // stages in the idle ring (slot 3): the staging buffer then holds the
      // first contributor's partial.
      uint8_t* wst = stage + quarter * 8192;
      if (lane == 0 && staged) bulk_wait_read0();  // this warp's previous tile store has read its boxes
      __syncwarp();
      if (warp_on) {
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {  // 16 columns at a time
          uint32_t ro[16], rx[16];
          tmem_ld16(tO + lane_off + c * 16, ro);
          if (p.has_inter) tmem_ld16(tS + lane_off + c * 16, rx);
          tmem_wait_ld();
          float* v = reinterpret_cast<float*>(ro);
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] = use_intra ? v[i] * a_self : 0.f;
          if (use_inter) {
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] += __uint_as_float(rx[i]);
          }
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const int ch = 2 * c + i;  // 16-byte chunk of the row: box ch / 8, chunk ch % 8 swizzled by row
            *reinterpret_cast<uint4*>(wst + (ch >> 3) * 4096 + lane * 128 + (((ch & 7) ^ (lane & 7)) << 4)) =
                make_uint4(pack_bf16x2(v[8 * i + 0], v[8 * i + 1]), pack_bf16x2(v[8 * i + 2], v[8 * i + 3]),
                           pack_bf16x2(v[8 * i + 4], v[8 * i + 5]), pack_bf16x2(v[8 * i + 6], v[8 * i + 7]));
          }
        }
      }
      tc_fence_before();
      fence_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bars[B_ES + sub]);
        mbar_arrive(&bars[B_EO + sub]);
        if (warp_on) {
          tma_store_3d(tm_o, wst, h * 128, qt * 128 + quarter * 32, b);
          tma_store_3d(tm_o, wst + 4096, h * 128 + 64, qt * 128 + quarter * 32, b);
          bulk_commit();
        }
      }
      staged = true;
    }
  }
  if (lane == 0) bulk_wait0();
  return true;
}

// ------------------------------------------------------------------ kernel
__global__ void __launch_bounds__(kAttnThreads, 1)
attn_bf16_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_mq,
                 const __grid_constant__ CUtensorMap tm_o, const AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                               // [2] sub-tiles
  uint8_t* sR = smem + 2 * kTile;                   // [kRing] K / V / MqT tiles
  uint8_t* sStage = smem + (2 + kRing) * kTile;     // output tile staging
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kTilesBytes);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + B_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  float* stats = reinterpret_cast<float*>(smem + kTilesBytes + kBarBytes);  // [2 sub][m, l][128]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cta = blockIdx.x;
  const unsigned u_begin = p.range[cta], u_end = p.range[cta + 1];
  if (size_t(smem - smem_raw) + kTilesBytes + kSmallBytes > size_t(kAttnSmem)) {  // uniform over the CTA
    if (threadIdx.x == 0) record_error(p.err, kDevBadShape);
    return;
  }

  if (threadIdx.x == 0) {
    for (int i = 0; i < B_COUNT; ++i) {
      const bool four = (i >= B_PF && i < B_PF + 2) || (i >= B_ST && i < B_ST + 2) || (i >= B_ES && i < B_EO + 2);
      mbar_init(&bars[i], four ? 4u : 1u);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 2) tmem_alloc(tmem_holder, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const WaitCtl w{abort_flag, p.err, p.wait_limit_ns};
  const int wg = warp >> 2;
  if (wg == 0) {
    regs_dec<kCtlRegs>();
    if (warp == 0 && lane == 0) {
      tma_prefetch(&tm_q);
      tma_prefetch(&tm_k);
      tma_prefetch(&tm_v);
      producer(p, bars, sQ, sR, &tm_q, &tm_k, &tm_v, &tm_mq, u_begin, u_end, w);
    } else if (warp == 1 && lane == 0) {
      mma_issuer(p, bars, tmem, smem_u32(sQ), smem_u32(sR), u_begin, u_end, w);
    }
    __syncwarp();
  } else if (wg == 3) {
    regs_dec<kEpiRegs>();
    epilogue_role(p, bars, stats, sStage, sR, &tm_o, tmem, cta, warp & 3, lane, u_begin, u_end, abort_flag, w);
  } else {
    regs_inc<kSoftmaxRegs>();
    softmax_role(p, bars, stats, sStage, sR, sQ, &tm_o, tmem, cta, wg - 1, warp & 3, lane, u_begin, u_end, w);
  }

  // ------------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    // A wait ran out: let this CTA's own asynchronous work land before the
    // shared and tensor memory are released.
    if (warp == 1 && lane == 0) {
      mma_commit(&bars[B_DRAIN]);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(&bars[B_DRAIN], 0) && global_timer_ns() - t0 < 10000000ull) {
      }
    }
    if (warp == 0 && lane == 0) {
      const uint64_t t0 = global_timer_ns();
      while (global_timer_ns() - t0 < 2000000ull) {
      }
    }
    if (wg == 3 && lane == 0) bulk_wait0();
    __syncthreads();
  }
  if (warp == 2) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

cudaError_t launch_attn_bf16(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             const CUtensorMap& tmq, const CUtensorMap& tmo, const AttnParams& p,
                             cudaStream_t stream) {
  static unsigned done = 0;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(attn_bf16_kernel), kAttnSmem, &done);
  if (e != cudaSuccess) return e;
  static int regs = -1;
  if (regs < 0) {
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, attn_bf16_kernel);
    if (e != cudaSuccess) return e;
    regs = fa.numRegs;
  }
  if (regs != kLaunchRegs) return cudaErrorInvalidConfiguration;  // the register split needs this count
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.grid);
  cfg.blockDim = dim3(kAttnThreads);
  cfg.dynamicSmemBytes = kAttnSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;  // every CTA resident: the combine waits on peers
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, attn_bf16_kernel, tq, tk, tv, tmq, tmo, p);
}

bool attn_partition(AttnParams& p, int batch, int sms) {
  p.n_qt = (p.q_len + 127) / 128;
  p.n_pair = p.n_qt / 2;
  p.n_blk = p.n_pair + (p.n_qt & 1);
  p.nkv = (p.kv_len + 127) / 128;
  const long long bh = (long long)batch * p.heads;
  const long long units = bh * p.n_blk * p.nkv;
  if (units >= (1LL << 31)) return false;
  p.total_units = units;
  // Every unit costs about the same: a block of one sub-tile (the frame's last,
  // partial query tile) cannot overlap its softmax with a second sub-tile's
  // MMAs, so its key tile takes as long as a paired one.  Each CTA takes at
  // least a sixth of a block, so a block is split across at most eight CTAs
  // (the finishing CTA reads at most seven partials).
  const long long u_min = (p.nkv + 5) / 6;
  long long g = units / (u_min > 0 ? u_min : 1);
  if (g < 1) g = 1;
  if (g > sms) g = sms;
  if (g > kAttnMaxGrid) g = kAttnMaxGrid;
  p.grid = int(g);
  for (int c = 0; c <= p.grid; ++c) p.range[c] = unsigned(units * c / p.grid);
  return true;
}

}  // namespace arl2
