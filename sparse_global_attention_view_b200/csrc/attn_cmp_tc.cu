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
//               two TMEM score buffers, then O += P Vc and l += P 1 (bf16, P
//               from TMEM; the row sums of P come from the tensor core as the
//               product with a block of ones, so they sum exactly the bf16
//               weights the numerator uses);
//   warp 2      TMEM allocation (S at columns 0/128, O at 256, P at 320/384,
//               l at 448);
//   warps 4-7   softmax, one thread per query row;
//   warps 8-11  streaming top-K, one thread per query row.
// S(j+1) is computed while both warpgroups work on S(j): the softmax writes
// P(j) to its own TMEM columns, so the raw scores stay readable until the
// top-K warpgroup is done with them.  The softmax forms exp2 two at a time
// (packed f32x2 scaling, bf16x2 exp2: P is bf16 for the PV product anyway).
// It also forms the maxima of the tile's eight 16-column groups, compares them
// with each row's current K-th best score (published in shared memory by the
// top-K thread) and hands the top-K warp an 8-bit mask of the groups that may
// hold a candidate.  The top-K warp reads from TMEM only the groups flagged
// for any of its 32 rows and releases the score buffer after its last read.
// Candidates (columns that beat the row's K-th best, special entries and
// blocks below B0 excluded) are appended to a per-row buffer in shared
// memory.  When a row's buffer cannot take the next group, the whole warp
// merges it into the row's list of best pairs: the buffer is sorted across the
// 32 lanes by a bitonic network, combined with the sorted list (two entries
// per lane) by the max of opposite ends, and the result put in order by a
// bitonic merge -- a few hundred instructions for up to 28 candidates,
// instead of a heap insertion per candidate.  Pairs are packed 64-bit keys
// (score bits, then the complement of the entry index), so a larger key is a
// better pair and equal scores keep the lower entry, i.e. the lower block id.
// Columns arrive in ascending entry order, so a column whose score equals
// the K-th best comes after it and is rightly not a candidate.
#include <math_constants.h>

#include "internal.h"
#include "tc_common.cuh"

namespace gsa {
namespace {

using namespace tc;

// Of every 8 pairs of attention weights, this many are computed on the FMA
// pipe (exp2_bf16x2_poly) and the rest on the special-function unit.
#ifndef GSA_CMP_POLY_OF_8
#define GSA_CMP_POLY_OF_8 0
#endif

constexpr int TQ = 128;
constexpr int TK = 128;
constexpr int ST = 2;
constexpr int kThreads = 384;
constexpr int kMaxK = kFusedTopK;  // list capacity per row (two entries per lane)
constexpr int kBuf = 28;           // candidate buffer slots per row
constexpr uint32_t kSub = 128 * 128;    // one [128][32] fp32 (or [128][64] bf16) tile: 16 KB

constexpr uint32_t OFF_Q = 0;                          // 2 sub-tiles (d 0-31, 32-63)
constexpr uint32_t OFF_K = OFF_Q + 2 * kSub;           // ST x 2 sub-tiles
constexpr uint32_t OFF_V = OFF_K + ST * 2 * kSub;      // ST x bf16 tile
constexpr uint32_t OFF_ONES = OFF_V + ST * kSub;       // [16][128] bf16 ones: B of the row-sum product
constexpr uint32_t OFF_LST = OFF_ONES + 4096;          // [128 rows][64] keys, sorted descending
constexpr uint32_t OFF_BUF = OFF_LST + TQ * kMaxK * 8; // [kBuf slots][128 rows] keys (row ^ slot)
constexpr uint32_t OFF_BAR = OFF_BUF + kBuf * TQ * 8;
constexpr uint32_t OFF_TAU = OFF_BAR + 256;            // each row's K-th best score [128]
constexpr uint32_t OFF_MASK = OFF_TAU + TQ * 4;        // candidate-group masks [2][128] bytes
constexpr uint32_t OFF_MISC = OFF_MASK + 2 * TQ;
constexpr uint32_t kSmemBytes = OFF_MISC + 64 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory per block");
static_assert(OFF_ONES % 1024 == 0, "ones tile alignment");

// TMEM columns: S at 0 / 128, O at 256, P at 320 / 384 (bf16 pairs), l at 448
constexpr uint32_t TM_S = 0, TM_O = 256, TM_P = 320, TM_L = 448;

// KE / VE: a K / V stage is free again (the QK^T resp. PV product that read it
// is complete); MR: the softmax has published the candidate-group masks of
// score buffer b.
constexpr int B_Q = 0, B_KF = 1, B_VF = B_KF + ST, B_KE = B_VF + ST, B_VE = B_KE + ST,
              B_SF = B_VE + ST, B_PF = B_SF + 2, B_SR = B_PF + 2, B_MR = B_SR + 2, B_OD = B_MR + 2,
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

// A pair's key: the order-preserving bits of the score, then the complement
// of the compressed entry index (the map entry -> block id is increasing, so
// ordering by entry is ordering by block id).  0 is below every real key and
// marks an empty list slot.
__device__ __forceinline__ uint32_t order_bits(float s) {
  const uint32_t u = __float_as_uint(s);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float order_value(uint32_t o) {
  return __uint_as_float((o & 0x80000000u) ? (o & 0x7fffffffu) : ~o);
}
__device__ __forceinline__ unsigned long long u64max(unsigned long long a, unsigned long long b) {
  return a > b ? a : b;
}
// Compare-exchange with the lane `delta` away (xor): keep the larger key when
// `keep_max`, else the smaller.
__device__ __forceinline__ unsigned long long cmpx(unsigned long long x, int delta, bool keep_max) {
  const unsigned long long o = __shfl_xor_sync(0xffffffffu, x, delta);
  return (keep_max == (x > o)) ? x : o;
}
__device__ __forceinline__ void sts_u64(uint32_t addr, unsigned long long v) {
  asm volatile("st.shared.u64 [%0], %1;\n" ::"r"(addr), "l"(v) : "memory");
}
__device__ __forceinline__ unsigned long long lds_u64(uint32_t addr) {
  unsigned long long v;
  asm volatile("ld.shared.u64 %0, [%1];\n" : "=l"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ void tmem_wait_ld16(uint32_t (&r)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;\n"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                 "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
                 "+r"(r[14]), "+r"(r[15])
               :
               : "memory");
}

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
  const long long m0 = (long long)blockIdx.x * TQ;
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
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(B_SF + b), 1);
      mbar_init(bar(B_PF + b), TQ);
      mbar_init(bar(B_SR + b), TQ);  // top-K warpgroup is done with S buffer b
      mbar_init(bar(B_MR + b), TQ);
    }
    mbar_init(bar(B_OD), 1);
    mbar_init(bar(B_OF), 1);
    mbar_init(bar(B_DRAIN), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  volatile float* tau_s = reinterpret_cast<volatile float*>(sp + OFF_TAU);
  volatile uint8_t* mask_s = sp + OFF_MASK;
  if (tid < TQ) tau_s[tid] = -CUDART_INF_F;
  {
    // the B operand of the row-sum product: 16 x 128 bf16 ones (layout-free)
    fill_ones(sp + OFF_ONES, kOnesBytes, tid, kThreads);
    // empty lists: key 0 is below every real pair
    uint4* lst = reinterpret_cast<uint4*>(sp + OFF_LST);
    for (int i = tid; i < TQ * kMaxK * 8 / 16; i += kThreads) lst[i] = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
  }
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
      const uint32_t id_l = idesc(128, 16, kFmtBF16, 0, 0);
      const uint32_t sOnes = sb + OFF_ONES;
      auto issue_s = [&](int s, int b) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * kSub + (kk & 3) * 32;
          mma_tf32_ss(tbase + TM_S + b * 128, sdesc_k(sQ + off), sdesc_k(sK + 2 * s * kSub + off), id_qk, kk > 0);
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
        const int s = j % ST, b = j & 1;
        if (j + 1 < nt) {
          const int s1 = (j + 1) % ST;
          ok = mbar_wait(bar(B_KF + s1), ((j + 1) / ST) & 1, abort_flag, err, d.wait_cycles);
          // S(j+1) reuses the buffer of S(j-1): the top-K warpgroup must have read it
          if (ok && j >= 1) ok = mbar_wait(bar(B_SR + (b ^ 1)), (((j + 1) >> 1) - 1) & 1, abort_flag, err, d.wait_cycles);
          if (!ok) break;
          fence_after_sync();
          issue_s(s1, b ^ 1);
        }
        // (the softmax's arrival on PF(b) also says it has read S(j) from buffer b)
        ok = (cp.scores_only || mbar_wait(bar(B_VF + s), (j / ST) & 1, abort_flag, err, d.wait_cycles)) &&
             mbar_wait(bar(B_PF + b), (j >> 1) & 1, abort_flag, err, d.wait_cycles);
        if (!ok) break;
        fence_after_sync();
        if (cp.scores_only) continue;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ts(tbase + TM_O, tbase + TM_P + b * 64 + kk * 8, sdesc_mn(sV + s * kSub + kk * 2048), id_pv,
                      (j > 0 || kk > 0) ? 1u : 0u);
        // l += P 1: every column of the 16-wide result holds the row sum
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ts(tbase + TM_L, tbase + TM_P + b * 64 + kk * 8,
                      sdesc_k(sOnes + (kk >> 2) * 2048 + (kk & 3) * 32), id_l, (j > 0 || kk > 0) ? 1u : 0u);
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
    const uint32_t o_addr = tbase + lane_off + TM_O;
    const uint32_t l_addr = tbase + lane_off + TM_L;
    const float c2 = d.scale_log2;
    const unsigned long long c2x2 = pack_f32x2(c2, c2);
    float m_used = -CUDART_INF_F;
    bool ok = true;
    for (int j = 0; j < nt; ++j) {
      const int b = j & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(B_SF + b), (j >> 1) & 1, abort_flag, err, d.wait_cycles))) {
        ok = false;
        break;
      }
      fence_after_sync();
      const uint32_t s_addr = tbase + lane_off + TM_S + b * 128;
      const uint32_t p_addr = tbase + lane_off + TM_P + b * 64;
      const long long rem = n_k - (long long)j * TK;
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
      // the maxima of the eight 16-column groups, three values per max
      // instruction and eight independent chains
      float mq[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const uint32_t* g = &sv[q >> 1][(q & 1) * 16];
        float m = fmax3(__uint_as_float(g[0]), __uint_as_float(g[1]), __uint_as_float(g[2]));
#pragma unroll
        for (int i = 3; i < 15; i += 2) m = fmax3(m, __uint_as_float(g[i]), __uint_as_float(g[i + 1]));
        mq[q] = fmaxf(m, __uint_as_float(g[15]));
      }
      {
        // tell the top-K warp which groups may hold a candidate for this row:
        // those whose maximum beats the row's K-th best so far (a stale, lower
        // threshold only flags more groups)
        const float tau = tau_s[r];
        uint32_t msk = 0;
#pragma unroll
        for (int q = 0; q < 8; ++q) msk |= (mq[q] > tau ? 1u : 0u) << q;
        mask_s[b * TQ + r] = (uint8_t)msk;
        mbar_arrive(bar(B_MR + b));
      }
      if (cp.scores_only) {
        // ranking pass: no attention; S(j) has been read
        fence_before_sync();
        mbar_arrive(bar(B_PF + b));
        continue;
      }
      const float mx = fmax3(fmax3(mq[0], mq[1], mq[2]), fmax3(mq[3], mq[4], mq[5]), fmaxf(mq[6], mq[7]));
      const float mxs = mx * c2;
      const bool need = mxs > m_used + 8.f;
      if (__any_sync(0xffffffffu, need)) {
        const float corr = need ? exp2f(m_used - mxs) : 1.f;
        if (j > 0) {
          // the previous P V and P 1 products must be complete before O and l
          // are rescaled
          if (!__all_sync(0xffffffffu, mbar_wait(bar(B_OD), (j - 1) & 1, abort_flag, err, d.wait_cycles))) {
            ok = false;
            break;
          }
          fence_after_sync();
#pragma unroll
          for (int c = 0; c < 5; ++c) {
            const uint32_t addr = c < 4 ? o_addr + 16 * c : l_addr;
            uint32_t ov[16];
            tmem_ld16(addr, ov);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * corr);
            tmem_st16(addr, ov);
          }
          tmem_wait_st();
        }
        if (need) m_used = mxs;
      }
      const unsigned long long n2 = pack_f32x2(-m_used, -m_used);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[i] = (i & 7) < GSA_CMP_POLY_OF_8 ? exp2_bf16x2_poly(sv[c][2 * i], sv[c][2 * i + 1], c2x2, n2)
                                              : exp2_bf16x2_fma(sv[c][2 * i], sv[c][2 * i + 1], c2x2, n2);
        tmem_st16(p_addr + 16 * c, pk);
      }
      tmem_wait_st();
      fence_before_sync();
      mbar_arrive(bar(B_PF + b));
    }
    if (ok && !cp.scores_only) ok = __all_sync(0xffffffffu, mbar_wait(bar(B_OF), 0, abort_flag, err, d.wait_cycles));
    if (ok && !cp.scores_only) {
      fence_after_sync();
      const long long row = m0 + r;
      const bool store = row < d.Tc;
      uint32_t lv[16];
      tmem_ld16(l_addr, lv);
      tmem_wait_ld();
      const float inv = 1.f / __uint_as_float(lv[0]);
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
    constexpr unsigned FULL = 0xffffffffu;
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    ulonglong2* lst2 = reinterpret_cast<ulonglong2*>(sp + OFF_LST);  // [row][32]: entries 2i, 2i+1
    const uint32_t buf_s = sb + OFF_BUF;
    const int K = d.K;
    const int E = d.E, S = d.S;
    const int e_min = d.B0 > 0 ? E : 0;  // frame 0's entries are not candidates when it is kept whole
    const bool all_cols = S == 0 && e_min == 0;
    const int ntok = (int)n_k;
    const long long my_row = m0 + r;
    const float inv_e = 1.f / (float)E;
    // a second ranking pass keeps only pairs strictly below the first pass's
    // K-th best key of the row
    const unsigned long long ub =
        (cp.ub != nullptr && my_row < d.Tc) ? cp.ub[(long long)h * d.Tc + my_row] : ~0ull;
    const bool has_ub = cp.ub != nullptr;
    const float ub_score = ub == ~0ull ? CUDART_INF_F : order_value((uint32_t)(ub >> 32));
    float tau = -CUDART_INF_F;  // score a candidate must beat (-inf until the list holds K pairs)
    int nb = 0;                 // candidates in this row's buffer
    int cnt = 0;                // pairs in this row's list (at most kMaxK)

    // Merge the buffers of the rows whose lanes are set in `rows` into their
    // lists, the whole warp working on one row at a time.
    auto merge_rows = [&](unsigned rows) {
      __syncwarp();
      while (rows != 0) {
        const int rl = __ffs(rows) - 1;
        rows &= rows - 1;
        const int rr = q4 * 32 + rl;
        const int nbr = __shfl_sync(FULL, nb, rl);
        const int cntr = __shfl_sync(FULL, cnt, rl);
        unsigned long long bk = lane < nbr ? lds_u64(buf_s + (uint32_t)(lane * TQ + (rr ^ lane)) * 8u) : 0ull;
        // sort the buffer descending across the lanes (bitonic)
#pragma unroll
        for (int k = 2; k <= 32; k <<= 1)
#pragma unroll
          for (int jj = k >> 1; jj > 0; jj >>= 1) bk = cmpx(bk, jj, ((lane & jj) == 0) == ((lane & k) == 0));
        // the 64 largest of list (descending) and buffer (descending, padded
        // with zeros to 64): max of entry i and buffer entry 63 - i, a bitonic
        // sequence
        ulonglong2 a2 = lst2[rr * 32 + lane];
        const unsigned long long x0 = __shfl_sync(FULL, bk, (63 - 2 * lane) & 31);
        const unsigned long long x1 = __shfl_sync(FULL, bk, (62 - 2 * lane) & 31);
        if (lane >= 16) {
          a2.x = u64max(a2.x, x0);
          a2.y = u64max(a2.y, x1);
        }
        // bitonic merge into descending order (element distance 2 jj, then 1)
#pragma unroll
        for (int jj = 16; jj > 0; jj >>= 1) {
          const bool lower = (lane & jj) == 0;
          a2.x = cmpx(a2.x, jj, lower);
          a2.y = cmpx(a2.y, jj, lower);
        }
        if (a2.y > a2.x) {
          const unsigned long long t = a2.x;
          a2.x = a2.y;
          a2.y = t;
        }
        lst2[rr * 32 + lane] = a2;
        const int nc = min(cntr + nbr, kMaxK);
        const unsigned long long kth = __shfl_sync(FULL, ((K - 1) & 1) ? a2.y : a2.x, (K - 1) >> 1);
        if (lane == rl) {
          cnt = nc;
          nb = 0;
          tau = nc >= K ? order_value((uint32_t)(kth >> 32)) : -CUDART_INF_F;
          tau_s[r] = tau;
        }
      }
      __syncwarp();
    };

    bool ok = true;
    for (int j = 0; j < nt; ++j) {
      const int b = j & 1;
      if (!__all_sync(FULL, mbar_wait(bar(B_MR + b), (j >> 1) & 1, abort_flag, err, d.wait_cycles))) {
        ok = false;
        break;
      }
      fence_after_sync();
      const uint32_t s_addr = tbase + lane_off + TM_S + b * 128;
      const int e0 = j * TK;
      const int lim = ntok - e0;
      // the groups flagged by the softmax for any of the warp's 32 rows
      uint32_t G = __reduce_or_sync(FULL, (uint32_t)mask_s[b * TQ + r]);
      // which of the tile's 128 columns may be ranked at all (the same for
      // every row): inside the sequence, not a special entry, not below B0
      uint32_t cv[4];
      if (G != 0) {
        if (all_cols && lim >= TK) {
          cv[0] = cv[1] = cv[2] = cv[3] = FULL;
        } else {
          const int i0 = (e0 + lane) % E;
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            const int c = 32 * w + lane;
            // (i0 + 32 w) mod E; the float quotient of a small number is off by at most one
            const int x = i0 + 32 * w;
            int f = (int)((float)x * inv_e);
            int i = x - f * E;
            if (i < 0) i += E;
            if (i >= E) i -= E;
            cv[w] = __ballot_sync(FULL, c < lim && e0 + c >= e_min && i >= S);
          }
        }
      }
      bool released = false;
      while (G != 0) {
        const int q = __ffs(G) - 1;
        G &= G - 1;
        uint32_t g[16];
        tmem_ld16(s_addr + 16 * q, g);
        tmem_wait_ld16(g);
        if (G == 0) {
          fence_before_sync();
          mbar_arrive(bar(B_SR + b));  // the tensor core may overwrite this buffer now
          released = true;
        }
        uint32_t cm = 0;
        if (has_ub) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float v = __uint_as_float(g[i]);
            cm |= (v > tau && v <= ub_score ? 1u : 0u) << i;
          }
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) cm |= (__uint_as_float(g[i]) > tau ? 1u : 0u) << i;
        }
        cm &= (cv[q >> 1] >> ((q & 1) * 16)) & 0xffffu;
        // the columns where any row of the warp has a candidate: usually one
        // or two, so the append below skips the others with a uniform branch
        const uint32_t cu = __reduce_or_sync(FULL, cm);
        if (cu == 0) continue;
        const unsigned over = __ballot_sync(FULL, nb + __popc(cm) > kBuf);
        if (over != 0) merge_rows(over);
        const uint32_t lo0 = 0x7fffffffu - (uint32_t)(e0 + 16 * q);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          if (cu & (1u << i)) {
            if (cm & (1u << i)) {
              const unsigned long long key =
                  ((unsigned long long)order_bits(__uint_as_float(g[i])) << 32) | (lo0 - (uint32_t)i);
              if (key < ub) {
                sts_u64(buf_s + (uint32_t)(nb * TQ + (r ^ nb)) * 8u, key);
                ++nb;
              }
            }
          }
        }
      }
      if (!released) {
        fence_before_sync();
        mbar_arrive(bar(B_SR + b));
      }
    }
    ok = __all_sync(FULL, ok);
    if (ok) merge_rows(__ballot_sync(FULL, nb > 0));
    if (ok) {
      // write each row's result, the warp working on one row at a time: the
      // list's first min(cnt, K) pairs are the row's top-K
      for (int rl = 0; rl < 32; ++rl) {
        const int rr = q4 * 32 + rl;
        const long long row = m0 + rr;
        if (row >= d.Tc) break;
        const int kk = min(__shfl_sync(FULL, cnt, rl), K);
        const ulonglong2 a2 = lst2[rr * 32 + lane];
        const long long cb = ((long long)h * d.Tc + row) * d.K;
        if (cp.root != nullptr && lane == ((K - 1) >> 1))
          cp.root[(long long)h * d.Tc + row] = kk == K ? (((K - 1) & 1) ? a2.y : a2.x) : 0ull;
        int id[2];
        bool have[2];
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          const unsigned long long key = t ? a2.y : a2.x;
          const int e = (int)(0x7fffffffu - (uint32_t)key);
          const int f = e / E;
          id[t] = f * d.Bf + (e - f * E - S);
          have[t] = 2 * lane + t < kk;
        }
        if (cp.best != nullptr && lane == 0) cp.best[(long long)h * d.Tc + row] = kk > 0 ? id[0] : -1;
        if (cand_s != nullptr) {
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            const int k = 2 * lane + t;
            if (k < K) {
              const unsigned long long key = t ? a2.y : a2.x;
              cand_s[cb + k] = have[t] ? order_value((uint32_t)(key >> 32)) * d.scale : -CUDART_INF_F;
              cand_i[cb + k] = have[t] ? id[t] : -1;
            }
          }
        }
        if (sel != nullptr) {
          // ascending ids: each pair's rank among the row's kk distinct ids
          int rank[2] = {0, 0};
          for (int m = 0; m < 32; ++m) {
            const int o0 = __shfl_sync(FULL, id[0], m), o1 = __shfl_sync(FULL, id[1], m);
            const bool h0 = 2 * m < kk, h1 = 2 * m + 1 < kk;
#pragma unroll
            for (int t = 0; t < 2; ++t) rank[t] += (h0 && o0 < id[t]) + (h1 && o1 < id[t]);
          }
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            const int k = 2 * lane + t;
            if (have[t]) sel[cb + rank[t]] = id[t];
            else if (k < K) sel[cb + k] = -1;
          }
        }
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
  cudaError_t e = cudaFuncSetAttribute(attn_cmp_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, attn_cmp_tc_kernel);
  if (e != cudaSuccess) return e;
  if (fa.numRegs != kLaunchRegs) return cudaErrorInvalidConfiguration;
  dim3 grid((unsigned)((d.Tc + TQ - 1) / TQ), (unsigned)d.H);
  attn_cmp_tc_kernel<<<grid, kThreads, kSmemBytes, st>>>(mq, mk, mv, d, oc, cand_score, cand_idx, sel,
                                                         err, cp);
  return cudaGetLastError();
}

}  // namespace gsa
