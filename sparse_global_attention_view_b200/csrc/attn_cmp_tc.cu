// Attention in the pooled sequence fused with the S_guide streaming top-K
// (Speed3R technical summary 2.1: compression branch and selection branch;
// 2.2: a streaming top-K inside the attention loop, no score matrix in memory).
//
// One CTA = one 128-row tile of compressed queries of one head, 12 warps:
//   warp 0      TMA producer: the fp32 pooled query tile once, then a 2-stage
//               ring of 128-entry fp32 pooled-K tiles, each stage refilled as
//               soon as the QK^T product that read it is complete;
//   warp 3      TMA producer of the 2-stage ring of bf16 pooled-V tiles, each
//               stage refilled once its PV product is complete;
//   warp 1      MMA issuer: S = Qc Kc^T with kind::tf32 from the fp32 means
//               (the top-K ranking needs better than bf16 scores), into one of
//               three TMEM score buffers, then O += P Vc (bf16, P from TMEM);
//   warp 2      TMEM allocation (S at columns 0/128/256, O at 384, P at 448);
//   warps 4-7   softmax, one thread per query row;
//   warps 8-11  streaming top-K, one thread per query row.
// S(j+1) is computed while both warpgroups work on S(j): the softmax writes
// P(j) to its own TMEM columns (one buffer, rewritten once the P V product of
// the tile before is complete), so the raw scores stay readable until the
// top-K warpgroup is done with them; with three score buffers the top-K
// warpgroup may trail the softmax by a tile without stalling the tensor core.
// The softmax already forms the maxima of the tile's sixteen 8-column groups;
// it compares them with each row's current K-th best score (published in
// shared memory by the top-K thread) and hands the top-K warp a 16-bit mask
// of the groups that may hold a candidate.  The top-K warp reads from TMEM
// only the groups flagged for any of its 32 rows and releases the score
// buffer after its last read.  Candidates (columns that beat the row's K-th
// best) go to a per-row buffer in shared memory without branches (every
// column is written to the next free slot, which is kept only for a
// candidate); when a row's buffer could not take the next group, the warp
// inserts buffered candidates in lockstep (one round of insertions serves
// every row, each row taking its newest) into the rows' heaps of K best
// (score, block id) pairs until no row holds more than kKeep; special entries
// are never ranked.  Once every heap of the warp is full, a round is one
// predicated three-level replacement of the root per lane (lanes without a
// candidate walk it without moving), with the next round's candidate loaded
// during the current one: no lane diverges.  Only a strictly larger key
// displaces the root, and a key orders by score, then by the lower id, so
// the heaps hold the K largest keys whatever the order of insertion.  The
// softmax keeps independent max and sum chains (three-input maxima, paired
// fp32 arithmetic): one warp per sub-partition runs it and shares the
// sub-partition's issue slots with a top-K warp.  A second instantiation
// (kDump) also writes the logits of requested rows for debugging.
#include <math_constants.h>

#include "internal.h"
#include "tc_common.cuh"

namespace gsa {
namespace {

using namespace tc;

constexpr int TQ = kCmpTileRows;
constexpr int TK = 128;
constexpr int ST = 2;
constexpr int kThreads = 384;
constexpr int kMaxK = kFusedTopK;  // heap capacity per row
constexpr int kBuf = 32;         // candidate buffer entries per row
constexpr int kKeep = 20;        // candidates a row may keep buffered after a flush (<= kBuf - 8)
constexpr uint32_t kSub = 128 * 128;    // one [128][32] fp32 (or [128][64] bf16) tile: 16 KB

constexpr uint32_t OFF_Q = 0;                        // 2 sub-tiles (d 0-31, 32-63)
constexpr uint32_t OFF_K = OFF_Q + 2 * kSub;         // ST x 2 sub-tiles
constexpr uint32_t OFF_V = OFF_K + ST * 2 * kSub;    // ST x bf16 tile
constexpr uint32_t OFF_HS = OFF_V + ST * kSub;       // heap keys [kMaxK][128] (8 bytes)
constexpr uint32_t OFF_CS = OFF_HS + kMaxK * TQ * 8; // candidate scores [kBuf][128]
constexpr uint32_t OFF_CC = OFF_CS + kBuf * TQ * 4;  // candidate entry indices
constexpr uint32_t OFF_BAR = OFF_CC + kBuf * TQ * 4;
constexpr int kCandGap = (int)((OFF_CC - OFF_CS) / 4);  // floats from a candidate's score to its index
constexpr uint32_t OFF_TAU = OFF_BAR + 256;          // each row's K-th best score [128]
constexpr int NS = 3;                                // TMEM score buffers
constexpr uint32_t OFF_MASK = OFF_TAU + TQ * 4;      // candidate-group masks [NS][128] bytes
constexpr uint32_t OFF_MISC = OFF_MASK + NS * TQ * 2;
constexpr uint32_t kSmemBytes = OFF_MISC + 64 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory per block");

// KE / VE: a K / V stage is free again (the QK^T resp. PV product that read it
// is complete); MR: the softmax has published the candidate-group masks of
// score buffer b.
constexpr int B_Q = 0, B_KF = 1, B_VF = B_KF + ST, B_KE = B_VF + ST, B_VE = B_KE + ST,
              B_SF = B_VE + ST, B_PF = B_SF + NS, B_SR = B_PF + 1, B_MR = B_SR + NS, B_OD = B_MR + NS,
              B_OF = B_OD + 1, B_DRAIN = B_OF + 1, B_COUNT = B_DRAIN + 1;
static_assert(B_COUNT * 8 <= 256, "barrier area");
constexpr uint32_t kCols = 512;
// Register split: the block is launched with kLaunchRegs per thread; the
// producer/MMA warpgroup gives registers to the softmax and top-K warpgroups.
// 128 * kRegsLow + 256 * kRegsHigh must not exceed 384 * kLaunchRegs, or the
// increase would wait forever, so the host refuses to launch unless the
// compiled kernel uses exactly kLaunchRegs registers per thread.
constexpr int kLaunchRegs = 168, kRegsLow = 56, kRegsHigh = 224;
static_assert(128 * kRegsLow + 256 * kRegsHigh <= kThreads * kLaunchRegs, "register split");

// The K best (score, block id) pairs of one row: a 4-ary min-heap in shared
// memory of packed 64-bit keys, [slot][row] layout so the 128 rows hit
// distinct banks.  key = (order-preserving bits of the score) << 32 |
// (0x7fffffff - id): a larger key is a better pair (higher score, or equal
// score and lower id), so the root holds the worst pair.  Four children per
// node keep a sift to 3 levels of 4 independent loads.
__device__ __forceinline__ uint32_t order_bits(float s) {
  const uint32_t u = __float_as_uint(s);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float order_value(uint32_t o) {
  return __uint_as_float((o & 0x80000000u) ? (o & 0x7fffffffu) : ~o);
}
__device__ __forceinline__ unsigned long long pair_key(float s, int id) {
  return ((unsigned long long)order_bits(s) << 32) | (uint32_t)(0x7fffffff - id);
}
struct Heap {
  unsigned long long* hk;
  int r, K, cnt;
  float tau;  // score of the worst pair kept (-inf until the heap is full)
  unsigned long long rootkey;  // key of the worst pair kept (0 until the heap is full)

  __device__ __forceinline__ unsigned long long at(int i) const { return hk[i * TQ + r]; }
  __device__ __forceinline__ void put(int i, unsigned long long k) { hk[i * TQ + r] = k; }
  __device__ __forceinline__ void sift(int p, unsigned long long key) {
    while (true) {
      const int c0 = 4 * p + 1;
      if (c0 >= K) break;
      unsigned long long m = at(c0);
      int mc = c0;
#pragma unroll
      for (int t = 1; t < 4; ++t) {
        if (c0 + t < K) {
          const unsigned long long x = at(c0 + t);
          if (x < m) m = x, mc = c0 + t;
        }
      }
      if (m >= key) break;
      put(p, m);
      p = mc;
    }
    put(p, key);
  }
  // Replace the root (the worst pair) of a full heap by `key` and restore the
  // heap order: a fixed three levels (K <= 64 pairs fit in 1 + 4 + 16 + 64
  // slots), the four children of a level loaded together and the descent
  // predicated rather than branched, so every lane of the warp takes the same
  // path; the new root is tracked in a register.
  __device__ __forceinline__ void replace_root(unsigned long long key, bool take = true) {
    if (!take) key = 0ull;  // a lane without a candidate walks the levels without moving
    int p = 0;
    bool go = take;
    unsigned long long root = key;
#pragma unroll
    for (int lvl = 0; lvl < 3; ++lvl) {
      const int c0 = 4 * p + 1;
      unsigned long long x[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) x[t] = (go && c0 + t < K) ? at(c0 + t) : ~0ull;
      unsigned long long m = x[0];
      int mc = c0;
#pragma unroll
      for (int t = 1; t < 4; ++t)
        if (x[t] < m) m = x[t], mc = c0 + t;
      const bool move = go && m < key;
      if (move) put(p, m);
      if (lvl == 0 && move) root = m;
      p = move ? mc : p;
      go = move;
    }
    if (take) {
      put(p, key);
      rootkey = root;
      tau = order_value((uint32_t)(root >> 32));
    }
  }
  __device__ __forceinline__ void push(unsigned long long key) {
    if (cnt < K) {
      put(cnt, key);
      if (++cnt == K) {
        for (int p = (K - 2) / 4; p >= 0; --p) sift(p, at(p));
        rootkey = at(0);
        tau = order_value((uint32_t)(rootkey >> 32));
      }
      return;
    }
    replace_root(key);
  }
  __device__ __forceinline__ int id_of(int i) const { return 0x7fffffff - (int)(uint32_t)at(i); }
  __device__ __forceinline__ float score_of(int i) const { return order_value((uint32_t)(at(i) >> 32)); }
};

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}
// Wait for this thread's TMEM loads; the registers are passed through so that
// no use of them can be scheduled before the wait.
__device__ __forceinline__ void tmem_wait_ld16(uint32_t (&r)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;\n"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                 "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
                 "+r"(r[14]), "+r"(r[15])
               :
               : "memory");
}

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld8(uint32_t (&r)[8]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;\n"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7])
               :
               : "memory");
}

// kDump: the debug instantiation that also writes the requested rows'
// logits (CmpPass::dump); the production one has no dump code at all.
template <bool kDump>
__global__ void __launch_bounds__(kThreads, 1)
    attn_cmp_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                       const __grid_constant__ CUtensorMap tv, const Dims d, float* __restrict__ oc,
                       float* __restrict__ cand_s, int* __restrict__ cand_i, int* __restrict__ sel,
                       unsigned* err, const CmpPass cp) {
  extern __shared__ __align__(1024) uint8_t cmp_smem_raw[];
  const uint32_t raw = smem_u32(cmp_smem_raw);
  const uint32_t sb = (raw + 1023u) & ~1023u;
  uint8_t* sp = cmp_smem_raw + (sb - raw);
  const uint32_t sQ = sb + OFF_Q, sK = sb + OFF_K, sV = sb + OFF_V;
  auto bar = [&](int i) -> uint32_t { return sb + OFF_BAR + 8u * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sp + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sp + OFF_MISC + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.y;
  const long long m0 = (long long)(blockIdx.x + cp.tile0) * TQ;
  const long long n_k = d.Tc;
  const int nt = (int)((n_k + TK - 1) / TK);

  if (tid == 0) {
    mbar_init(bar(B_Q), 1);
    for (int s = 0; s < ST; ++s) {
      mbar_init(bar(B_KF + s), 1);
      mbar_init(bar(B_VF + s), 1);
      mbar_init(bar(B_KE + s), 1);
      mbar_init(bar(B_VE + s), 1);
    }
    for (int b = 0; b < NS; ++b) {
      mbar_init(bar(B_SF + b), 1);
      mbar_init(bar(B_SR + b), TQ);  // top-K warpgroup is done with S buffer b
      mbar_init(bar(B_MR + b), TQ);
    }
    mbar_init(bar(B_PF), TQ);
    mbar_init(bar(B_OD), 1);
    mbar_init(bar(B_OF), 1);
    mbar_init(bar(B_DRAIN), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  volatile float* tau_s = reinterpret_cast<volatile float*>(sp + OFF_TAU);
  volatile uint16_t* mask_s = reinterpret_cast<volatile uint16_t*>(sp + OFF_MASK);
  if (tid < TQ) tau_s[tid] = -CUDART_INF_F;
  if (warp == 2) {
    tmem_alloc(smem_u32(tmem_slot), kCols);
    tmem_relinquish();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tbase = *tmem_slot;

  if (warp < 4) {
    regs_dec<kRegsLow>();
  }
  if (warp == 0) {
    // TMA producer of the query tile and the K ring: a K stage is refilled as
    // soon as the QK^T product that read it is complete
    if (lane == 0) {
      prefetch_tmap(&tq);
      prefetch_tmap(&tk);
      mbar_expect_tx(bar(B_Q), 2 * kSub);
      for (int half = 0; half < 2; ++half)
        tma_load_3d(sQ + half * kSub, &tq, bar(B_Q), 32 * half, h, (int)m0);
      int issued = 0;
      for (int j = 0; j < nt; ++j) {
        const int s = j % ST;
        if (j >= ST && !mbar_wait(bar(B_KE + s), ((j / ST) - 1) & 1, abort_flag, err, d.wait_cycles)) break;
        mbar_expect_tx(bar(B_KF + s), 2 * kSub);
        for (int half = 0; half < 2; ++half)
          tma_load_3d(sK + (2 * s + half) * kSub, &tk, bar(B_KF + s), 32 * half, h, j * TK);
        issued = j + 1;
      }
      if (*abort_flag) {
        volatile int never = 0;
        mbar_wait(bar(B_Q), 0, &never, err);
        for (int j = issued - 1; j >= 0 && j >= issued - ST; --j)
          mbar_wait(bar(B_KF + j % ST), (j / ST) & 1, &never, err);
      }
    }
  } else if (warp == 3) {
    // TMA producer of the V ring: a V stage is refilled once its PV product is complete
    if (lane == 0 && !cp.scores_only) {
      prefetch_tmap(&tv);
      int issued = 0;
      for (int j = 0; j < nt; ++j) {
        const int s = j % ST;
        if (j >= ST && !mbar_wait(bar(B_VE + s), ((j / ST) - 1) & 1, abort_flag, err, d.wait_cycles)) break;
        mbar_expect_tx(bar(B_VF + s), kSub);
        tma_load_3d(sV + s * kSub, &tv, bar(B_VF + s), 0, h, j * TK);
        issued = j + 1;
      }
      if (*abort_flag) {
        volatile int never = 0;
        for (int j = issued - 1; j >= 0 && j >= issued - ST; --j)
          mbar_wait(bar(B_VF + j % ST), (j / ST) & 1, &never, err);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id_qk = idesc(128, 128, kFmtTF32, 0, 0);
      const uint32_t id_pv = idesc(128, 64, kFmtBF16, 0, 1);
      auto issue_s = [&](int s, int b) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * kSub + (kk & 3) * 32;
          mma_tf32_ss(tbase + b * 128, sdesc_k(sQ + off), sdesc_k(sK + 2 * s * kSub + off), id_qk, kk > 0);
        }
        mma_commit(bar(B_SF + b));
        mma_commit(bar(B_KE + s));
      };
      bool ok = mbar_wait(bar(B_Q), 0, abort_flag, err, d.wait_cycles) && mbar_wait(bar(B_KF), 0, abort_flag, err, d.wait_cycles);
      if (ok) {
        fence_after_sync();
        issue_s(0, 0);
      }
      for (int j = 0; ok && j < nt; ++j) {
        const int s = j % ST;
        if (j + 1 < nt) {
          const int s1 = (j + 1) % ST, b1 = (j + 1) % NS;
          ok = mbar_wait(bar(B_KF + s1), ((j + 1) / ST) & 1, abort_flag, err, d.wait_cycles);
          // S(j+1) reuses the buffer of S(j+1-NS): the top-K warpgroup must
          // have read it (the softmax has: PV(j-1) waited for its P)
          if (ok && j + 1 >= NS)
            ok = mbar_wait(bar(B_SR + b1), (((j + 1) / NS) - 1) & 1, abort_flag, err, d.wait_cycles);
          if (!ok) break;
          fence_after_sync();
          issue_s(s1, b1);
        }
        if (cp.scores_only) continue;
        // P(j) is in TMEM once the softmax has arrived on PF
        ok = mbar_wait(bar(B_VF + s), (j / ST) & 1, abort_flag, err, d.wait_cycles) &&
             mbar_wait(bar(B_PF), j & 1, abort_flag, err, d.wait_cycles);
        if (!ok) break;
        fence_after_sync();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ts(tbase + 384, tbase + 448 + kk * 8, sdesc_mn(sV + s * kSub + kk * 2048), id_pv,
                      (j > 0 || kk > 0) ? 1u : 0u);
        mma_commit(bar(B_OD));
        mma_commit(bar(B_VE + s));
      }
      if (ok) {
        mma_commit(bar(B_OF));
      } else {
        volatile int never = 0;
        mma_commit(bar(B_DRAIN));
        mbar_wait(bar(B_DRAIN), 0, &never, err);
      }
    }
  } else if (warp >= 4 && warp < 8) {
    regs_inc<kRegsHigh>();
    // ---------------- softmax ----------------
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const uint32_t o_addr = tbase + lane_off + 384;
    const float c2 = d.scale_log2;
    float m_used = -CUDART_INF_F, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nt; ++j) {
      const int b = j % NS;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(B_SF + b), (j / NS) & 1, abort_flag, err, d.wait_cycles))) {
        ok = false;
        break;
      }
      fence_after_sync();
      const uint32_t s_addr = tbase + lane_off + b * 128;
      const uint32_t p_addr = tbase + lane_off + 448;
      const long long rem = n_k - (long long)j * TK;
      if constexpr (kDump) {
        // debug: this row's unscaled logits of the tile, as ranked, re-read
        // from TMEM 16 columns at a time (a short loop, off the hot path)
        const long long row = m0 + r;
        const bool mine = row >= cp.dump_row0 && row < cp.dump_row0 + cp.dump_rows && row < d.Tc;
        float* o = cp.dump + ((long long)h * cp.dump_rows + (row - cp.dump_row0)) * n_k + (long long)j * TK;
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          uint32_t t[16];
          tmem_ld16(s_addr + 16 * c, t);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i)
            if (mine && 16 * c + i < rem) o[16 * c + i] = __uint_as_float(t[i]);
        }
      }
      // all 128 scores in one round of TMEM loads: the softmax is bound by
      // TMEM load latency, so a second round would cost as much as the first
      uint32_t sv[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(s_addr + 32 * c, sv[c]);
      tmem_wait_ld();
      if (rem < TK) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (32 * c + i >= rem) sv[c][i] = __float_as_uint(-CUDART_INF_F);
      }
      // the maxima of the sixteen 8-column groups: sixteen independent chains
      // keep the single softmax warp of each sub-partition from stalling on one
      // 128-long dependency chain
      float mq[16];
      {
        // three-input maxima: four instructions per group of eight
        auto e = [&](int q, int i) -> float { return __uint_as_float(sv[q >> 2][(q & 3) * 8 + i]); };
#pragma unroll
        for (int q = 0; q < 16; ++q)
          mq[q] = fmaxf(fmax3(fmax3(e(q, 0), e(q, 1), e(q, 2)), fmax3(e(q, 3), e(q, 4), e(q, 5)), e(q, 6)), e(q, 7));
      }
      {
        // tell the top-K warp which groups may hold a candidate for this row:
        // those whose maximum beats the row's K-th best so far (a stale, lower
        // threshold only flags more groups)
        const float tau = tau_s[r];
        uint32_t msk = 0;
#pragma unroll
        for (int q = 0; q < 16; ++q) msk |= (mq[q] >= tau ? 1u : 0u) << q;
        if (m0 + r >= d.Tc) msk = 0u;  // rows past the sequence never rank
        mask_s[b * TQ + r] = (uint16_t)msk;
        mbar_arrive(bar(B_MR + b));
      }
      if (cp.scores_only) {
        // ranking pass: no attention (the top-K warpgroup's release of the
        // buffer also says this warpgroup has read it: it follows MR)
        continue;
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) mq[q] = fmaxf(mq[q], mq[q + 8]);
      const float mx = fmaxf(fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3])),
                             fmaxf(fmaxf(mq[4], mq[5]), fmaxf(mq[6], mq[7])));
      const float mxs = mx * c2;
      const bool need = mxs > m_used + 8.f;
      if (__any_sync(0xffffffffu, need)) {
        const float corr = need ? exp2f(m_used - mxs) : 1.f;
        if (j > 0) {
          // the previous P V product must be complete before O is rescaled
          if (!__all_sync(0xffffffffu, mbar_wait(bar(B_OD), (j - 1) & 1, abort_flag, err, d.wait_cycles))) {
            ok = false;
            break;
          }
          fence_after_sync();
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t ov[16];
            tmem_ld16(o_addr + 16 * c, ov);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * corr);
            tmem_st16(o_addr + 16 * c, ov);
          }
          tmem_wait_st();
        }
        if (need) {
          l *= corr;
          m_used = mxs;
        }
      }
      // P has one TMEM buffer: the P V product of the previous tile must be
      // complete before it is overwritten
      if (j > 0 && !__all_sync(0xffffffffu, mbar_wait(bar(B_OD), (j - 1) & 1, abort_flag, err, d.wait_cycles))) {
        ok = false;
        break;
      }
      // scaled, shifted scores two at a time (paired fp32 instructions, each
      // half rounded as the scalar form); four paired sum chains
      const uint64_t c2p = f2_pack(c2, c2), nmp = f2_pack(-m_used, -m_used);
      uint64_t ps2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float x0, x1;
          f2_unpack(f2_fma(f2_pack(__uint_as_float(sv[c][2 * i]), __uint_as_float(sv[c][2 * i + 1])), c2p, nmp), x0, x1);
          const float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
          ps2[i & 3] = f2_add(ps2[i & 3], f2_pack(p0, p1));
          pk[i] = pack_bf16x2(p0, p1);
        }
        tmem_st16(p_addr + 16 * c, pk);
      }
      tmem_wait_st();
      {
        float lo, hi;
        f2_unpack(f2_add(f2_add(ps2[0], ps2[1]), f2_add(ps2[2], ps2[3])), lo, hi);
        l += lo + hi;
      }
      fence_before_sync();
      mbar_arrive(bar(B_PF));
    }
    if (ok && !cp.scores_only) ok = __all_sync(0xffffffffu, mbar_wait(bar(B_OF), 0, abort_flag, err, d.wait_cycles));
    if (ok && !cp.scores_only) {
      fence_after_sync();
      const long long row = m0 + r;
      const bool store = row < d.Tc;
      const float inv = 1.f / l;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t ov[16];
        tmem_ld16(o_addr + 16 * c, ov);
        tmem_wait_ld();
        if (!store) continue;
        float4* dst = reinterpret_cast<float4*>(oc + (row * d.H + h) * kHeadDim + 16 * c);
#pragma unroll
        for (int i = 0; i < 4; ++i)
          dst[i] = make_float4(__uint_as_float(ov[4 * i]) * inv, __uint_as_float(ov[4 * i + 1]) * inv,
                               __uint_as_float(ov[4 * i + 2]) * inv, __uint_as_float(ov[4 * i + 3]) * inv);
      }
    }
  } else if (warp >= 8) {
    regs_inc<kRegsHigh>();
    // ---------------- streaming top-K over S_guide ----------------
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    float* cb_s = reinterpret_cast<float*>(sp + OFF_CS);
    int* cb_e = reinterpret_cast<int*>(sp + OFF_CC);
    Heap top{reinterpret_cast<unsigned long long*>(sp + OFF_HS), r, d.K, 0, -CUDART_INF_F, 0ull};
    const int E = d.E, S = d.S, Bf = d.Bf, B0 = (int)d.B0;
    const int ntok = (int)n_k;
    const long long my_row = m0 + r;
    // rows past the sequence (zero-filled queries, all scores equal) never rank
    const bool row_in = my_row < d.Tc;
    // a second ranking pass keeps only pairs strictly below the first pass's
    // K-th best (score, id) key of the row
    const unsigned long long ub =
        (cp.ub != nullptr && my_row < d.Tc) ? cp.ub[(long long)h * d.Tc + my_row] : ~0ull;
    int nb = 0;  // candidates waiting in this row's buffer
    // Insert the buffered candidates.  All lanes run this together, so one
    // round of insertions serves every row of the warp at once.
    // entry e -> frame f = e / E, position i = e - f E on the integer pipe
    // (a float quotient would queue its conversions behind the softmax's
    // exponentials): with m = floor((2^32 - 1) / E), hi32(e m) is e / E or
    // one less for every e < 2^31
    const uint32_t e_magic = 0xffffffffu / (uint32_t)E;
    auto decode = [&](int e, int& f, int& i) {
      f = (int)__umulhi((uint32_t)e, e_magic);
      i = e - f * E;
      if (i >= E) i -= E, ++f;
    };
    auto flush = [&](int keep) {
      if (__all_sync(0xffffffffu, !row_in || top.cnt == d.K)) {
        // every heap of the warp is full: one predicated replacement per
        // round, each row taking its newest candidate, until no row holds
        // more than `keep` (the order of insertion does not change the K
        // largest keys, and a row that keeps a few candidates keeps its lane
        // busy in the next flush's rounds)
        const int rounds = max(0, (int)__reduce_max_sync(0xffffffffu, (unsigned)nb) - keep);
        float v_next = nb > 0 ? cb_s[(nb - 1) * TQ + r] : -CUDART_INF_F;
        int e_next = nb > 0 ? cb_e[(nb - 1) * TQ + r] : 0;
        for (int n = 0; n < rounds; ++n) {
          const bool have = nb > 0;
          const float v = v_next;
          const int e = e_next;
          nb -= have ? 1 : 0;
          // the next round's candidate is read while this one is inserted
          v_next = nb > 0 ? cb_s[(nb - 1) * TQ + r] : -CUDART_INF_F;
          e_next = nb > 0 ? cb_e[(nb - 1) * TQ + r] : 0;
          int f, i;
          decode(e, f, i);
          const int id = f * Bf + (i - S);
          const unsigned long long key = pair_key(v, id);
          const bool take = have && key > top.rootkey && i >= S && id >= B0 && key < ub;
          top.replace_root(key, take);
        }
        tau_s[r] = top.tau;
        return;
      }
      for (int n = 0; n < nb; ++n) {
        const float v = cb_s[n * TQ + r];
        if (v < top.tau) continue;
        int f, i;
        decode(cb_e[n * TQ + r], f, i);
        // special entries are never ranked, nor blocks below B0 (frame 0 when
        // it is kept whole); once the heap is full only a larger key enters
        if (i >= S && f * Bf + (i - S) >= B0) {
          const unsigned long long key = pair_key(v, f * Bf + (i - S));
          if (key < ub && (top.cnt < top.K || key > top.rootkey)) top.push(key);
        }
      }
      nb = 0;
      tau_s[r] = top.tau;
    };
    // One 16-column group of the score tile: candidates are the columns that
    // beat the row's K-th best; the warp only scans groups where some of its
    // rows has one.
    auto group = [&](const uint32_t (&g)[8], int q, int e0, int lim) {
      // branch-free appends: every column is written to the row's next free
      // slot and the slot is kept only when the column is a candidate (the
      // buffer has room for 16 more, so the writes stay inside it)
      const float tau = top.tau;
      const int n_in = lim - 8 * q;  // columns of the group inside the sequence
      const int cbase = e0 + 8 * q;
      float* ps = cb_s + nb * TQ + r;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float v = __uint_as_float(g[i]);
        const bool c = row_in && v >= tau && i < n_in;
        ps[0] = v;
        ps[kCandGap] = __int_as_float(cbase + i);
        ps += c ? TQ : 0;
        nb += c ? 1 : 0;
      }
      if (__any_sync(0xffffffffu, nb > kBuf - 8)) flush(kKeep);
    };
    bool ok = true;
    for (int j = 0; j < nt; ++j) {
      const int b = j % NS;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(B_MR + b), (j / NS) & 1, abort_flag, err, d.wait_cycles))) {
        ok = false;
        break;
      }
      fence_after_sync();
      const uint32_t s_addr = tbase + lane_off + b * 128;
      const int e0 = j * TK;
      const int lim = ntok - e0;
      // the groups flagged by the softmax for any of the warp's 32 rows
      uint32_t G = __reduce_or_sync(0xffffffffu, (uint32_t)mask_s[b * TQ + r]);
      bool released = false;
      while (G != 0) {
        const int q = __ffs(G) - 1;
        G &= G - 1;
        uint32_t g[8];
        tmem_ld8(s_addr + 8 * q, g);
        tmem_wait_ld8(g);
        if (G == 0) {
          fence_before_sync();
          mbar_arrive(bar(B_SR + b));  // the tensor core may overwrite this buffer now
          released = true;
        }
        group(g, q, e0, lim);
      }
      if (!released) {
        fence_before_sync();
        mbar_arrive(bar(B_SR + b));
      }
    }
    if (__all_sync(0xffffffffu, ok)) flush(0);
    const long long row = m0 + r;
    if (ok && row < d.Tc && cp.root != nullptr)
      cp.root[(long long)h * d.Tc + row] = top.cnt == d.K ? top.at(0) : 0ull;
    if (ok && row < d.Tc && cp.best != nullptr) {
      // the row's best pair: the largest key of its heap (-1 when it is empty)
      unsigned long long bk = 0ull;
      int bi = -1;
      for (int k = 0; k < top.cnt; ++k)
        if (top.at(k) > bk) bk = top.at(k), bi = k;
      cp.best[(long long)h * d.Tc + row] = bi >= 0 ? top.id_of(bi) : -1;
    }
    if (ok && row < d.Tc) {
      const long long cb = ((long long)h * d.Tc + row) * d.K;
      if (cand_s != nullptr) {
        for (int k = 0; k < d.K; ++k) {
          const bool have = k < top.cnt;
          cand_s[cb + k] = have ? top.score_of(k) * d.scale : -CUDART_INF_F;
          cand_i[cb + k] = have ? top.id_of(k) : -1;
        }
      }
      if (sel != nullptr) {
        // the heap holds exactly this row's top-K: write its ids in ascending
        // order (rank of each id among the row's distinct ids), then -1 padding
        for (int k = 0; k < top.cnt; ++k) {
          const int me = top.id_of(k);
          int rank = 0;
          for (int k2 = 0; k2 < top.cnt; ++k2) rank += top.id_of(k2) < me;
          sel[cb + rank] = me;
        }
        for (int k = top.cnt; k < d.K; ++k) sel[cb + k] = -1;
      }
    }
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 2) {
    fence_after_sync();
    tmem_dealloc(tbase, kCols);
  }
}

}  // namespace

bool compressed_tc_supported(const Dims& d) { return d.K <= kMaxK; }

cudaError_t launch_compressed_tc(const Dims& d, const float* qc32, const float* kc32, const bf16* vc,
                                 float* oc, float* cand_score, int* cand_idx, int* sel, unsigned* err,
                                 cudaStream_t st, const CmpPass& cp) {
  if (!compressed_tc_supported(d)) return cudaErrorInvalidValue;
  const unsigned long long H = (unsigned long long)d.H, Tc = (unsigned long long)d.Tc;
  CUtensorMap mq, mk, mv;
  bool ok = make_tmap_3d(&mq, true, qc32, 64, H, Tc, 256, H * 256, 32, 1, 128) &&
            make_tmap_3d(&mk, true, kc32, 64, H, Tc, 256, H * 256, 32, 1, 128) &&
            make_tmap_3d(&mv, false, vc, 64, H, Tc, 128, H * 128, 64, 1, 128);
  if (!ok) return cudaErrorInvalidValue;
  auto kernel = cp.dump != nullptr ? attn_cmp_tc_kernel<true> : attn_cmp_tc_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, kernel);
  if (e != cudaSuccess) return e;
  if (fa.numRegs != kLaunchRegs) return cudaErrorInvalidConfiguration;
  const long long all_tiles = (d.Tc + TQ - 1) / TQ;
  if (cp.tile0 < 0 || cp.tiles < 0 || cp.tile0 + cp.tiles > all_tiles) return cudaErrorInvalidValue;
  dim3 grid((unsigned)(cp.tiles > 0 ? cp.tiles : all_tiles - cp.tile0), (unsigned)d.H);
  kernel<<<grid, kThreads, kSmemBytes, st>>>(mq, mk, mv, d, oc, cand_score, cand_idx, sel, err, cp);
  return cudaGetLastError();
}

}  // namespace gsa
