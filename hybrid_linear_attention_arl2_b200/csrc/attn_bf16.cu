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
// the sequence of (block, key tile) units over all (stream, head) pairs; each
// unit weighs the number of query tiles it covers.  A persistent grid of one
// CTA per SM takes contiguous, equal-weight ranges of that sequence
// ("stream-K"), so the grid stays full whatever the number of query tiles.  A
// block whose key range is split across CTAs is finished by the CTA holding
// its first key tiles: the others store their unnormalised partial output and
// softmax statistics (m, l) to a scratch slot and raise a ready flag; the
// finishing CTA combines the partials in key order (deterministic) and adds
// the read-out.  Ready flags are reset by their consumer, so every launch
// leaves them at zero.
//
// Roles (384 threads):
//   warp 0       TMA producer: per block, Q of both sub-tiles; K_j, V_j (and
//                MqT for blocks this CTA finishes) through a 4-slot ring;
//   warp 1       tcgen05 issuer: S = Q K_j^T, O += P V_j, X = Q MqT^T;
//   warp 2       tensor-memory allocator;
//   warps 4..7   softmax + epilogue of sub-tile A (one row per thread);
//   warps 8..11  softmax + epilogue of sub-tile B.
// Tensor memory (512 columns): S_A [0,128), S_B [128,256) (P written in
// place as bf16 pairs, then X), O_A [256,384), O_B [384,512).
//
// The same kernel without the read-out serves the softmax layers that keep a
// growing KV cache (the K/V tensor maps then cover the cache).

#include "params.h"
#include "sm100.cuh"

namespace arl2 {

constexpr int kAttnThreads = 384;
constexpr int kRing = 4;
constexpr uint32_t kTile = 32768;  // 128 rows x 128 bf16
constexpr uint32_t kHalf = 16384;  // one 64-column box
constexpr int kAttnSmem = (2 + kRing) * kTile + 32768 + 512 + 1024;
constexpr int kSlotFloats = kAttnSlotFloats;
constexpr int kSlotStats = 128 * 64;  // floats before (m, l) in a slot: 128 x 128 bf16 partial O
constexpr int kMaxContrib = 8;        // partials a finishing CTA may combine
constexpr uint32_t kStageBytes = 8 * 4096;  // per softmax warp: 32 rows x 128 B of output
// Register split: the launch gives every thread kLaunchRegs; warpgroup 0
// (producer, MMA issuer, allocator) drops to kCtlRegs and the two softmax
// warpgroups rise to kSoftmaxRegs.  128 * kCtlRegs + 256 * kSoftmaxRegs must
// not exceed 384 * kLaunchRegs, or setmaxnreg.inc would wait forever; the
// launcher refuses to run unless the compiled kernel has exactly kLaunchRegs.
constexpr int kPolyPairs = 5;  // of every 16 exp2 pairs of a full tile, this many run on the FMA pipe
constexpr int kLaunchRegs = 168;
constexpr int kCtlRegs = 72;
constexpr int kSoftmaxRegs = 216;
static_assert(128 * kCtlRegs + 256 * kSoftmaxRegs <= kAttnThreads * kLaunchRegs, "register split too large");

enum {
  B_QF = 0,                       // [2]
  B_QE = 2,                       // [2]
  B_RF = 4,                       // [kRing]
  B_RE = 4 + kRing,               // [kRing]
  B_SF = 4 + 2 * kRing,           // [2]
  B_PF = B_SF + 2,                // [2]
  B_SD = B_PF + 2,                // [2] segment done: every MMA of the segment completed
  B_ED = B_SD + 2,                // [2]
  B_TURN = B_ED + 2,              // [2] exponential-section turn of sub-tile A / B
  B_DRAIN = B_TURN + 2,
  B_COUNT
};

// ------------------------------------------------------------------ partition
// Units are (block, key tile) pairs in (stream, head, block, key tile) order;
// the host cuts them into per-CTA ranges of equal weight (AttnParams::range).
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

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const WaitCtl& w) {
  bool ok = mbar_wait(bar, parity, w);
  return __all_sync(0xffffffffu, ok);
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

// Stages 32 rows x 64 columns (bf16, one 128-byte half row per lane) through
// this warp's 4 KB of shared memory and writes them out four rows per store
// instruction (whole 128-byte row segments: coalesced).
__device__ __forceinline__ void store_rows_half(const AttnParams& p, uint8_t* stage, const int lane, const int b,
                                                const int h, const int row0, const int half, const uint32_t (&pk)[32]) {
  // write: chunk c of this lane's row at 16-byte column c ^ (lane & 7) (bank-conflict free)
  uint4* st = reinterpret_cast<uint4*>(stage);
#pragma unroll
  for (int c = 0; c < 8; ++c)
    st[lane * 8 + (c ^ (lane & 7))] = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
  __syncwarp();
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int r = 4 * it + (lane >> 3), c = lane & 7;
    const uint4 v = st[r * 8 + (c ^ (r & 7))];
    const int q_row = row0 + r;
    if (q_row < p.q_len) {
      __nv_bfloat16* dst = p.o + ((size_t(b) * p.q_len + q_row) * p.heads + h) * 128 + half * 64 + c * 8;
      *reinterpret_cast<uint4*>(dst) = v;
    }
  }
  __syncwarp();
}

__device__ __forceinline__ float bf16_lo(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t x) { return __uint_as_float(x & 0xFFFF0000u); }

// End of one segment for one sub-tile (a warpgroup, one row per thread).
//  * a segment that does not start at key tile 0 stores its unnormalised O
//    rows (bf16, chunk-major) and (m, l) to this CTA's slot and raises the
//    slot's ready flag;
//  * a segment that starts at key tile 0 writes the final rows: its own
//    accumulator, combined with the partials of the CTAs that hold the rest of
//    the block's keys (in key order), normalised, plus the read-out X.
// Arrives on `ed_bar` once the tensor-memory reads are done.  Returns false if
// a wait gave up.
__device__ __forceinline__ bool segment_epilogue(const AttnParams& p, const Seg s, const int cta,
                                              const int sub, const int lane, const int row, const uint32_t lane_off,
                                              const uint32_t tS, const uint32_t tO, const bool warp_on,
                                              const bool row_ok, const int q_row, const float m, const float l,
                                              uint64_t* ed_bar, volatile int* abort_flag, uint8_t* stage) {
  const int wg_thread = threadIdx.x - 128 - sub * 128;  // 0..127 within the warpgroup
  const bool writer = s.j0 == 0, full = writer && s.j1 == p.nkv;
  const bool use_intra = !(p.flags & 2u);
  const bool use_inter = p.has_inter && !(p.flags & 1u);
  if (!writer) {
    float* slot = p.scratch + (size_t(cta) * 2 + sub) * kSlotFloats;
    if (warp_on) {
      uint32_t r[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tO + lane_off + c * 32, slice32(r, c));
      tmem_wait_ld();
      if (row_ok) {
        // bf16, chunk-major: 16-byte chunk i of row r at uint4 index i * 128 + r, so the
        // 32 rows of a warp write one contiguous 512-byte span per instruction
        uint4* d4 = reinterpret_cast<uint4*>(slot) + row;
#pragma unroll
        for (int i = 0; i < 16; ++i)
          d4[i * 128] = make_uint4(
              pack_bf16x2(__uint_as_float(r[8 * i]), __uint_as_float(r[8 * i + 1])),
              pack_bf16x2(__uint_as_float(r[8 * i + 2]), __uint_as_float(r[8 * i + 3])),
              pack_bf16x2(__uint_as_float(r[8 * i + 4]), __uint_as_float(r[8 * i + 5])),
              pack_bf16x2(__uint_as_float(r[8 * i + 6]), __uint_as_float(r[8 * i + 7])));
        slot[kSlotStats + row] = m;
        slot[kSlotStats + 128 + row] = l;
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(ed_bar);
    __threadfence();
    named_bar(1 + sub, 128);
    if (wg_thread == 0) st_release(p.ready + cta * 2 + sub, 1u);
    return true;
  }
  // Contributors: the CTAs after this one whose first segment continues this
  // block (empty ranges skipped), as a bit mask over cta + 1 + i.
  uint32_t cmask = 0;
  int n_contrib = 0;
  bool ok = true;
  if (!full) {
    bool complete = false;
    for (int c2 = cta + 1; c2 < p.grid && c2 <= cta + 32 && n_contrib < kMaxContrib; ++c2) {
      const unsigned a0 = p.range[c2], a1 = p.range[c2 + 1];
      if (a0 == a1) continue;
      unsigned uu = a0;
      Seg s2;
      next_seg(p, uu, a1, s2);
      if (s2.bh != s.bh || s2.blk != s.blk) break;
      cmask |= 1u << (c2 - cta - 1);
      ++n_contrib;
      if (s2.j1 == p.nkv) {
        complete = true;
        break;
      }
    }
    if (!complete) {  // the host partition bounds a block to kMaxContrib + 1 pieces; never expected
      record_error(p.err, kDevBadShape);
      *abort_flag = 1;
    }
    if (wg_thread == 0) {  // wait until every contributor's partial is visible
      for (uint32_t mm = cmask; mm && !*abort_flag; mm &= mm - 1) {
        const unsigned* f = p.ready + (cta + 1 + __ffs(mm) - 1) * 2 + sub;
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
    // thread 0's acquire and this barrier order every thread's reads of the partials
    named_bar(1 + sub, 128);
    ok = !*abort_flag;
  }
  // slot of the k-th contributor (k < n_contrib)
  auto slot_of = [&](int k) -> const float* {
    uint32_t mm = cmask;
    for (int i = 0; i < k; ++i) mm &= mm - 1;
    return p.scratch + (size_t(cta + __ffs(mm)) * 2 + sub) * kSlotFloats;
  };
  // combined statistics, all contributors' (m, l) loaded in one batch
  float M = m, a_self = 0.f;
  float mk[kMaxContrib], lk[kMaxContrib];
#pragma unroll
  for (int k = 0; k < kMaxContrib; ++k) {
    mk[k] = -INFINITY;
    lk[k] = 0.f;
    if (ok && row_ok && k < n_contrib) {
      const float* sl = slot_of(k);
      mk[k] = sl[kSlotStats + row];
      lk[k] = sl[kSlotStats + 128 + row];
    }
  }
  if (ok && row_ok) {
#pragma unroll
    for (int k = 0; k < kMaxContrib; ++k) M = fmaxf(M, mk[k]);
    float Lsum = l * fast_exp2(m - M);
#pragma unroll
    for (int k = 0; k < kMaxContrib; ++k) {
      mk[k] = fast_exp2(mk[k] - M);  // now the contributor's weight
      Lsum = fmaf(lk[k], mk[k], Lsum);
    }
    const float inv_l = 1.f / Lsum;
    a_self = fast_exp2(m - M) * inv_l;
#pragma unroll
    for (int k = 0; k < kMaxContrib; ++k) mk[k] *= inv_l;
  }
  if (ok && warp_on) {
    const int b = s.bh / p.heads, h = s.bh % p.heads;
    const int row0 = (q_row - row) + (row & ~31);  // first query row of this warp
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      // this half row of the first contributor, fetched before the tensor-memory reads
      uint4 xh[8];
      if (row_ok && n_contrib > 0) {
        const uint4* s4 = reinterpret_cast<const uint4*>(slot_of(0)) + half * 8 * 128 + row;
#pragma unroll
        for (int i = 0; i < 8; ++i) xh[i] = s4[i * 128];
      }
      uint32_t pk[32];
#pragma unroll
      for (int qq = 0; qq < 2; ++qq) {
        const int col = half * 64 + qq * 32;
        uint32_t ro[32], rx[32];
        tmem_ld32(tO + lane_off + col, ro);
        if (p.has_inter) tmem_ld32(tS + lane_off + col, rx);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) ro[i] = __float_as_uint(__uint_as_float(ro[i]) * a_self);
#pragma unroll
        for (int k = 0; k < kMaxContrib; ++k) {
          if (row_ok && k < n_contrib) {
            uint4 x[4];
            if (k == 0) {
#pragma unroll
              for (int i = 0; i < 4; ++i) x[i] = xh[qq * 4 + i];
            } else {
              const uint4* s4 = reinterpret_cast<const uint4*>(slot_of(k)) + (col / 8) * 128 + row;
#pragma unroll
              for (int i = 0; i < 4; ++i) x[i] = s4[i * 128];
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const uint32_t w4[4] = {x[i].x, x[i].y, x[i].z, x[i].w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                ro[8 * i + 2 * e] = __float_as_uint(fmaf(bf16_lo(w4[e]), mk[k], __uint_as_float(ro[8 * i + 2 * e])));
                ro[8 * i + 2 * e + 1] =
                    __float_as_uint(fmaf(bf16_hi(w4[e]), mk[k], __uint_as_float(ro[8 * i + 2 * e + 1])));
              }
            }
          }
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float v0 = use_intra ? __uint_as_float(ro[2 * i]) : 0.f;
          float v1 = use_intra ? __uint_as_float(ro[2 * i + 1]) : 0.f;
          if (use_inter) {
            v0 += __uint_as_float(rx[2 * i]);
            v1 += __uint_as_float(rx[2 * i + 1]);
          }
          pk[qq * 16 + i] = pack_bf16x2(v0, v1);
        }
      }
      if (half == 1) {  // every tensor-memory read of this segment is done
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(ed_bar);
      }
      store_rows_half(p, stage, lane, b, h, row0, half, pk);
    }
  } else {
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(ed_bar);
  }
  if (!full) {
    named_bar(1 + sub, 128);  // every row has read the partials
    if (wg_thread == 0)
      for (uint32_t mm = cmask; mm; mm &= mm - 1) p.ready[(cta + __ffs(mm)) * 2 + sub] = 0u;
  }
  return ok;
}

// The tcgen05 issuer (one warp: every lane runs the loop and waits, so all
// operands are warp-uniform; the elected lane issues).  Order per key tile t,
// with sub-tile B one
// tile behind A:   S_A(t), PV_B(t-1), S_B(t), PV_A(t)
// so that each softmax warpgroup has two MMA groups' time to produce P.  An S
// MMA is issued right after the PV that reads the P it overwrites: tcgen05.mma
// operations of one thread execute in issue order.  All state is in scalars
// (no arrays indexed at run time) so the issue loop stays in registers.
__device__ __forceinline__ void mma_issuer(const AttnParams& p, uint64_t* bars, const uint32_t tmem,
                                           const uint32_t q_addr, const uint32_t r_addr, const unsigned u_begin,
                                           const unsigned u_end, const WaitCtl& w) {
  const bool leader = elect_one();
  constexpr uint32_t kTile16 = kTile >> 4, kHalf16 = kHalf >> 4;  // descriptor address units
  const uint32_t id_o = idesc_bf16(128, 128, 0, 1);                 // P (TMEM) x V (MN-major)
  const uint32_t id_x = idesc_bf16(128, 128, 0, 0);
  const uint64_t dqa = smem_desc_sw128(q_addr, 16, 1024), dqb = dqa + kTile16;
  const uint64_t dr0 = smem_desc_sw128(r_addr, 16, 1024);     // K-major ring tile
  const uint64_t dv0 = smem_desc_sw128(r_addr, kHalf, 1024);  // MN-major ring tile
  const uint32_t tSA = tmem, tSB = tmem + 128, tOA = tmem + 256, tOB = tmem + 384;
  uint32_t ring = 0, qa_use = 0, qb_use = 0, ita = 0, itb = 0, sega = 0, segb = 0;
  unsigned u = u_begin;
  Seg s;
  while (next_seg(p, u, u_end, s)) {
    const bool has_b = s.blk < p.n_pair;
    const int n = s.j1 - s.j0;
    if (!warp_wait(&bars[B_QF + 0], qa_use & 1, w)) return;
    ++qa_use;
    if (sega > 0 && !warp_wait(&bars[B_ED + 0], (sega - 1) & 1, w)) return;
    if (has_b) {
      if (!warp_wait(&bars[B_QF + 1], qb_use & 1, w)) return;
      ++qb_use;
      if (segb > 0 && !warp_wait(&bars[B_ED + 1], (segb - 1) & 1, w)) return;
    }
    uint32_t vprev = 0;
    int nk_prev = 0;
    for (int t = 0; t < n; ++t) {
      const int j = s.j0 + t;
      const int valid = min(128, p.kv_len - j * 128);
      const uint32_t id_s = idesc_bf16(128, min(128, (valid + 15) & ~15), 0, 0);
      const int nk = (valid + 15) >> 4;
      // K_j
      const uint32_t kslot = ring & (kRing - 1);
      if (!warp_wait(&bars[B_RF + kslot], (ring / kRing) & 1, w)) return;
      ++ring;
      tc_fence_after();
      const uint64_t dk = dr0 + kslot * kTile16;
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * kHalf16 + (kk & 3) * 2;
          mma_ss(tSA, dqa + off, dk + off, id_s, kk > 0);
        }
        mma_commit(&bars[B_SF + 0]);
      }
      __syncwarp();
      if (has_b) {
        if (t > 0) {
          if (!warp_wait(&bars[B_PF + 1], itb & 1, w)) return;
          ++itb;
          tc_fence_after();
          const uint64_t dvp = dv0 + vprev * kTile16;
          if (leader) {
            for (int kk = 0; kk < nk_prev; ++kk) mma_ts(tOB, tSB + kk * 8, dvp + kk * 128, id_o, (t > 1 || kk > 0));
            mma_commit(&bars[B_RE + vprev]);
          }
          __syncwarp();
        }
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * kHalf16 + (kk & 3) * 2;
            mma_ss(tSB, dqb + off, dk + off, id_s, kk > 0);
          }
          mma_commit(&bars[B_SF + 1]);
        }
        __syncwarp();
      }
      if (leader) mma_commit(&bars[B_RE + kslot]);
      __syncwarp();
      // V_j
      const uint32_t vslot = ring & (kRing - 1);
      if (!warp_wait(&bars[B_RF + vslot], (ring / kRing) & 1, w)) return;
      ++ring;
      if (!warp_wait(&bars[B_PF + 0], ita & 1, w)) return;
      ++ita;
      tc_fence_after();
      const uint64_t dvv = dv0 + vslot * kTile16;
      if (leader) {
        for (int kk = 0; kk < nk; ++kk) mma_ts(tOA, tSA + kk * 8, dvv + kk * 128, id_o, (t > 0 || kk > 0));
        if (!has_b) mma_commit(&bars[B_RE + vslot]);
      }
      __syncwarp();
      vprev = vslot;
      nk_prev = nk;
    }
    if (has_b && n > 0) {
      if (!warp_wait(&bars[B_PF + 1], itb & 1, w)) return;
      ++itb;
      tc_fence_after();
      const uint64_t dvp = dv0 + vprev * kTile16;
      if (leader) {
        for (int kk = 0; kk < nk_prev; ++kk) mma_ts(tOB, tSB + kk * 8, dvp + kk * 128, id_o, (n > 1 || kk > 0));
        mma_commit(&bars[B_RE + vprev]);
      }
      __syncwarp();
    }
    if (s.j0 == 0 && p.has_inter) {  // X = Q MqT^T for the rows this CTA finishes
      const uint32_t mslot = ring & (kRing - 1);
      if (!warp_wait(&bars[B_RF + mslot], (ring / kRing) & 1, w)) return;
      ++ring;
      tc_fence_after();
      const uint64_t dm = dr0 + mslot * kTile16;
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * kHalf16 + (kk & 3) * 2;
          mma_ss(tSA, dqa + off, dm + off, id_x, kk > 0);
        }
        if (has_b) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * kHalf16 + (kk & 3) * 2;
            mma_ss(tSB, dqb + off, dm + off, id_x, kk > 0);
          }
        }
        mma_commit(&bars[B_RE + mslot]);
      }
      __syncwarp();
    }
    if (leader) {
      mma_commit(&bars[B_SD + 0]);
      mma_commit(&bars[B_QE + 0]);
      if (has_b) {
        mma_commit(&bars[B_SD + 1]);
        mma_commit(&bars[B_QE + 1]);
      }
    }
    __syncwarp();
    ++sega;
    if (has_b) ++segb;
  }
}

__global__ void __launch_bounds__(kAttnThreads, 1)
attn_bf16_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_mq,
                 const AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                   // [2] sub-tiles
  uint8_t* sR = smem + 2 * kTile;       // [kRing] K / V / MqT tiles
  uint8_t* sStage = smem + (2 + kRing) * kTile;  // [8 softmax warps][4 KB] output staging
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (2 + kRing) * kTile + kStageBytes);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + B_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cta = blockIdx.x;
  const unsigned u_begin = p.range[cta], u_end = p.range[cta + 1];

  if (threadIdx.x == 0) {
    for (int i = 0; i < B_COUNT; ++i) mbar_init(&bars[i], (i == B_PF || i == B_PF + 1 || i == B_ED || i == B_ED + 1 || i == B_TURN || i == B_TURN + 1) ? 4u : 1u);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 2) tmem_alloc(tmem_holder, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const WaitCtl w{abort_flag, p.err, p.wait_limit_ns};
  if (warp < 4) {
    regs_dec<kCtlRegs>();
  if (warp == 0) {
    {
      // ---------------------------------------------------------------- producer (whole warp,
      // the elected lane issues the copies)
      const bool leader = elect_one();
      if (leader) {
        tma_prefetch(&tm_q);
        tma_prefetch(&tm_k);
        tma_prefetch(&tm_v);
      }
      uint32_t ring = 0, qa_use = 0, qb_use = 0;
      bool ok = true;
      unsigned u = u_begin;
      Seg s;
      while (ok && next_seg(p, u, u_end, s)) {
        const int b = s.bh / p.heads, h = s.bh % p.heads;
        const bool has_b = s.blk < p.n_pair;
        const int qt_a = has_b ? 2 * s.blk : p.n_qt - 1;
        const bool writer = s.j0 == 0;
        const int n = s.j1 - s.j0;
        const int ntiles = 2 * n + ((writer && p.has_inter) ? 1 : 0);
        const int x0 = h * 128;
        auto put = [&](int t) -> bool {
          const uint32_t slot = ring % kRing;
          if (ring >= kRing && !warp_wait(&bars[B_RE + slot], ((ring / kRing) - 1) & 1, w)) return false;
          uint8_t* dst = sR + slot * kTile;
          if (leader) {
            mbar_expect_tx(&bars[B_RF + slot], kTile);
            if (t < 2 * n) {
              const int j = s.j0 + (t >> 1);
              const CUtensorMap* m = (t & 1) ? &tm_v : &tm_k;
              tma_load_3d(dst, m, &bars[B_RF + slot], x0, j * 128, b);
              tma_load_3d(dst + kHalf, m, &bars[B_RF + slot], x0 + 64, j * 128, b);
            } else {
              tma_load_3d(dst, &tm_mq, &bars[B_RF + slot], 0, 0, s.bh);
              tma_load_3d(dst + kHalf, &tm_mq, &bars[B_RF + slot], 64, 0, s.bh);
            }
          }
          __syncwarp();
          ++ring;
          return true;
        };
        const int pre = min(2, ntiles);
        for (int t = 0; ok && t < pre; ++t) ok = put(t);
        for (int sub = 0; ok && sub < (has_b ? 2 : 1); ++sub) {
          const uint32_t used = sub ? qb_use : qa_use;
          if (used > 0 && !(ok = warp_wait(&bars[B_QE + sub], (used - 1) & 1, w))) break;
          uint8_t* dst = sQ + sub * kTile;
          const int row = (qt_a + sub) * 128;
          if (leader) {
            mbar_expect_tx(&bars[B_QF + sub], kTile);
            tma_load_3d(dst, &tm_q, &bars[B_QF + sub], x0, row, b);
            tma_load_3d(dst + kHalf, &tm_q, &bars[B_QF + sub], x0 + 64, row, b);
          }
          __syncwarp();
          if (sub) ++qb_use; else ++qa_use;
        }
        for (int t = pre; ok && t < ntiles; ++t) ok = put(t);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer (whole warp)
    mma_issuer(p, bars, tmem, smem_u32(sQ), smem_u32(sR), u_begin, u_end, w);
  }
  } else {
    regs_inc<kSoftmaxRegs>();
    // ------------------------------------------------------------------ softmax + epilogue
    const int sub = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = uint32_t(quarter * 32) << 16;
    const uint32_t tS = tmem + sub * 128, tO = tmem + 256 + sub * 128;
    const float sl2 = p.scale_log2;
    uint32_t it = 0, segs_done = 0, turns = 0;
    bool ok = true;
    unsigned u = u_begin;
    Seg s;
    while (ok && next_seg(p, u, u_end, s)) {
      const bool has_b = s.blk < p.n_pair;
      if (sub == 1 && !has_b) continue;
      const int b = s.bh / p.heads, h = s.bh % p.heads;
      const int qt = (has_b ? 2 * s.blk : p.n_qt - 1) + sub;
      const int q_row = qt * 128 + row;
      const bool row_ok = q_row < p.q_len;
      const bool warp_on = qt * 128 + quarter * 32 < p.q_len;  // warp-uniform
      const bool writer = s.j0 == 0, full = writer && s.j1 == p.nkv;
      float m = -INFINITY, l = 0.f;
      for (int t = 0; t < s.j1 - s.j0; ++t) {
        if (!(ok = warp_wait(&bars[B_SF + sub], it & 1, w))) break;
        tc_fence_after();
        const int j = s.j0 + t;
        const int valid = min(128, p.kv_len - j * 128);
        // The two warpgroups take turns for the exponentials (when the block
        // has both sub-tiles), so each runs its section with the SMSPs' issue
        // slots and MUFU to itself.
        const bool take_turn = has_b && !(sub == 0 && turns == 0);
        const uint32_t turn_parity = sub == 0 ? (turns - 1) & 1 : turns & 1;
        if (warp_on) {
          // the whole 128-column row of S in one round trip
          uint32_t r[128];
#pragma unroll
          for (int c = 0; c < 4; ++c) tmem_ld32(tS + lane_off + c * 32, slice32(r, c));
          tmem_wait_ld();
          if (valid < 128) {
#pragma unroll
            for (int i = 0; i < 128; ++i)
              if (i >= valid) r[i] = __float_as_uint(-INFINITY);
          }
          // row max: a two-input max tree over 8 independent chains
          float m8[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) m8[k] = __uint_as_float(r[k]);
#pragma unroll
          for (int i = 8; i < 128; i += 8)
#pragma unroll
            for (int k = 0; k < 8; ++k) m8[k] = fmaxf(m8[k], __uint_as_float(r[i + k]));
          const float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                                 fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7]))) * sl2;
          // Lazy rescaling: the running max moves only when it grows by more
          // than 8 (a factor 256), so P stays <= 256 and O is touched rarely.
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
          if (take_turn && !(ok = warp_wait(&bars[B_TURN + sub], turn_parity, w))) break;
          // P = exp2(S * scale * log2(e) - m), packed to bf16 pairs over S's first 64
          // columns.  On full tiles kPolyPairs of every 16 pairs take the FMA-pipe
          // exp2 so that the MUFU is not the limit; the masked last tile (columns
          // at -inf) takes the MUFU for all of them.
          const float nm = -m;
          float l8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
          if (valid == 128) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              uint32_t pk[16];
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const float x0 = fmaf(__uint_as_float(r[c * 32 + 2 * i]), sl2, nm);
                const float x1 = fmaf(__uint_as_float(r[c * 32 + 2 * i + 1]), sl2, nm);
                float p0, p1;
                if (i >= 16 - kPolyPairs) {  // x <= 8: the lazy max is at most 8 below the row max
                  p0 = exp2_poly(x0);
                  p1 = exp2_poly(x1);
                } else {
                  p0 = fast_exp2(x0);
                  p1 = fast_exp2(x1);
                }
                l8[(2 * i) & 7] += p0;
                l8[(2 * i + 1) & 7] += p1;
                pk[i] = pack_bf16x2(p0, p1);
              }
              tmem_st16(tS + lane_off + c * 16, pk);
            }
          } else {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              uint32_t pk[16];
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const float p0 = fast_exp2(fmaf(__uint_as_float(r[c * 32 + 2 * i]), sl2, nm));
                const float p1 = fast_exp2(fmaf(__uint_as_float(r[c * 32 + 2 * i + 1]), sl2, nm));
                l8[(2 * i) & 7] += p0;
                l8[(2 * i + 1) & 7] += p1;
                pk[i] = pack_bf16x2(p0, p1);
              }
              tmem_st16(tS + lane_off + c * 16, pk);
            }
          }
          if (has_b) {
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[B_TURN + (sub ^ 1)]);
          }
          l = fmaf(l, f, ((l8[0] + l8[1]) + (l8[2] + l8[3])) + ((l8[4] + l8[5]) + (l8[6] + l8[7])));
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
        } else if (has_b) {  // a warp with no valid rows still passes the turn on
          if (take_turn && !(ok = warp_wait(&bars[B_TURN + sub], turn_parity, w))) break;
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars[B_TURN + (sub ^ 1)]);
        }
        if (has_b) ++turns;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[B_PF + sub]);
        ++it;
      }
      if (!ok) break;
      if (!(ok = warp_wait(&bars[B_SD + sub], segs_done & 1, w))) break;
      ++segs_done;
      tc_fence_after();
      if (!segment_epilogue(p, s, cta, sub, lane, row, lane_off, tS, tO, warp_on, row_ok, q_row, m, l,
                            &bars[B_ED + sub], abort_flag, sStage + (warp - 4) * 4096))
        ok = false;
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
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(&bars[B_DRAIN], 0) && global_timer_ns() - t0 < 10000000ull) {
      }
    }
    if (warp == 0 && lane == 0) {
      const uint64_t t0 = global_timer_ns();
      while (global_timer_ns() - t0 < 2000000ull) {
      }
    }
    __syncthreads();
  }
  if (warp == 2) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

cudaError_t launch_attn_bf16(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             const CUtensorMap& tmq, const AttnParams& p, cudaStream_t stream) {
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
  return cudaLaunchKernelEx(&cfg, attn_bf16_kernel, tq, tk, tv, tmq, p);
}

bool attn_partition(AttnParams& p, int batch, int sms) {
  p.n_qt = (p.q_len + 127) / 128;
  p.n_pair = p.n_qt / 2;
  p.n_blk = p.n_pair + (p.n_qt & 1);
  p.nkv = (p.kv_len + 127) / 128;
  const long long bh = (long long)batch * p.heads;
  const long long units = bh * p.n_blk * p.nkv;
  if (units >= (1LL << 31)) return false;
  p.total_weight = bh * p.n_qt * p.nkv;
  // Each CTA takes at least a sixth of a two-tile block, so a block is split
  // across at most eight CTAs (the finishing CTA reads at most seven partials).
  const long long w_min = (2LL * p.nkv + 5) / 6;
  long long g = p.total_weight / (w_min > 0 ? w_min : 1);
  if (g < 1) g = 1;
  if (g > sms) g = sms;
  if (g > kAttnMaxGrid) g = kAttnMaxGrid;
  p.grid = int(g);
  // CTA c starts at the first unit whose start weight is >= W * c / grid.
  const long long wbh = (long long)p.n_qt * p.nkv;
  const long long pair_w = (long long)p.n_pair * 2 * p.nkv;
  auto units_before = [&](long long w) {
    const long long b_h = w / wbh, r = w - b_h * wbh;
    long long u = b_h * (long long)p.n_blk * p.nkv;
    u += r <= pair_w ? (r + 1) / 2 : (long long)p.n_pair * p.nkv + (r - pair_w);
    return u;
  };
  for (int c = 0; c <= p.grid; ++c) p.range[c] = unsigned(units_before(p.total_weight * c / p.grid));
  return true;
}

}  // namespace arl2
