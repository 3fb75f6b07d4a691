// Step 5 (and, fused, step 6) on the 5th-generation tensor cores: the
// selection branch (Speed3R technical summary 2.1, selection branch: fine
// attention over the selected regions only; 2.2, Speed3R-VGGT: the reference
// frame / camera tokens are always kept).
//
// The <= 16 fine queries of one compressed entry (query block) share one key
// set, so the products run transposed, with the keys on the 128-row M side and
// the entry's queries as N = 16:
//   S^T  = K_sel Q^T               M = 128 keys, K = 64
//   O^T += [V_sel | 1]^T P^T       M = 128: the 64 value dims, then 64 rows of
//                                  ones whose results are the sums of P per query
// so P never leaves the softmax thread's lane except as the B operand, and the
// row sums come out of the tensor core with exactly the bf16 weights of the
// numerator.  The keys of a pair are the valid tokens of its selected blocks
// packed into consecutive slots (a block at the right or bottom edge holds 4
// or 1 of its 16 patches, and those are the blocks S_guide tends to rank
// first: their means keep more of the tokens' noise, so their scores spread
// wider), so a pair needs ceil(valid tokens / 128) tiles rather than K / 8.
// The gather warp copies each slot's 128 bytes with cp.async straight into
// the 128-byte-swizzled operand layout; the entry's queries are one TMA box of
// 4 x 4 patches over a per-frame view of the token grid.
//
// One CTA per SM works through (head, entry) pairs; 12 warps:
//   warp 0      builder: per entry its queries (one TMA box) and its packed
//               token list (from the selection, loaded one entry ahead) into
//               one of two list buffers;
//   warp 3      gather warp: per entry, once its list is handed over, the K
//               and V rows of every 128-key tile by cp.async into a 5-stage
//               ring; when the always-kept tokens are not supplied as a
//               finished softmax state, their head-major copies are streamed
//               first as plain 128-key TMA tiles;
//   warp 1      MMA issuer (one thread): S^T(t+1) is issued before O^T(t)
//               when tile t+1's keys have landed, so the tensor core works
//               while the softmax handles a tile; otherwise O^T(t) goes first,
//               so that an entry's epilogue never waits for the next gathers;
//   warp 2      TMEM allocation (S^T at columns 0/16, O^T at 32 + 16 e for
//               the four entry slots e);
//   warps 4-7   softmax, one thread per key lane (16 queries per thread);
//   warps 8-11  epilogue of the previous entry (merge with the always-kept
//               segment, one reciprocal denominator per query, gate, store)
//               while the softmax works on the next one.
// The softmax shifts every query by a fixed reference: the always-kept
// segment's log-sum-exp when it is supplied (so that segment's normalised
// output enters with weight 1), else the first tile's maximum.  A tile whose
// scores exceed the reference by 2^8 raises it for its queries and rescales
// their partial sums (rare; one barrier with an OR reduction per tile decides
// it for all 128 key lanes).  Every mbarrier wait is bounded as in the other
// tensor-core kernels.
#include <math_constants.h>
#include <stddef.h>

#include "internal.h"
#include "tc_common.cuh"

namespace gsa {
namespace {

using namespace tc;

constexpr int NQ = 16;           // query slots per entry (P * P <= 16)
constexpr int TKEYS = 128;       // keys per tile
constexpr int ST = 5;            // K/V ring stages: the gathers of 5 tiles in flight
constexpr int NE = 4;            // entry slots (queries, selection, O^T buffer)
constexpr int kThreads = 384;
constexpr uint32_t kKV = 16384;  // one [128][64] bf16 tile
constexpr uint32_t kQ = 2048;    // one [16][64] bf16 query tile
constexpr uint32_t kPT = 4096;   // one [16][128] bf16 P^T tile (two 64-key atoms)

struct Entry {
  int h, a;
  int n_tiles, n_kept;  // tiles in all; the first n_kept stream the always-kept keys
  int n_keys;           // valid tokens of the selected blocks (key slots 0 .. n_keys - 1)
  uint32_t qmask;       // query slots that hold a token
  int tok[NQ];          // token of each query slot
  float m0[NQ];         // initial reference (log2 units of the scaled logit)
  float mf[NQ], wf[NQ]; // final reference and weight of the always-kept segment
};

constexpr uint32_t OFF_K = 0;
constexpr uint32_t OFF_V = OFF_K + ST * kKV;
constexpr uint32_t OFF_ONES = OFF_V + ST * kKV;
constexpr uint32_t OFF_Q = OFF_ONES + kKV;
constexpr uint32_t OFF_PT = OFF_Q + NE * kQ;
constexpr uint32_t OFF_ENT = OFF_PT + 2 * kPT;
constexpr uint32_t kEntBytes = (sizeof(Entry) + 127) / 128 * 128;
constexpr int kTokList = kMaxTopK * NQ;                  // key slots of one entry at most
constexpr uint32_t OFF_TOK = OFF_ENT + NE * kEntBytes;   // two token lists (builder -> gather warp)
constexpr uint32_t OFF_RED = OFF_TOK + 2 * kTokList * 4;  // [4 warps][16] per-query partial maxima
constexpr uint32_t OFF_LS = OFF_RED + 4 * NQ * 4;        // [16] reciprocal denominators (epilogue)
constexpr uint32_t OFF_GATE = OFF_LS + NQ * 4;           // [2] gate partial dot products
constexpr uint32_t OFF_BAR = (OFF_GATE + 16 + 255) / 256 * 256;
constexpr uint32_t OFF_MISC = OFF_BAR + 512;
constexpr uint32_t kSmemBytes = OFF_MISC + 64 + 1024;
static_assert(OFF_Q % 1024 == 0 && OFF_PT % 1024 == 0 && OFF_ONES % 1024 == 0, "operand alignment");
static_assert(kSmemBytes <= 232448, "shared memory per block");

// barriers
constexpr int B_EF = 0, B_EE = B_EF + NE, B_EM = B_EE + NE, B_KF = B_EM + NE, B_VF = B_KF + ST,
              B_KE = B_VF + ST, B_VE = B_KE + ST, B_SF = B_VE + ST, B_PF = B_SF + 2, B_PE = B_PF + 2,
              B_OF = B_PE + 2, B_OD = B_OF + NE, B_DRAIN = B_OD + 1, B_TF = B_DRAIN + 1, B_TE = B_TF + 2,
              B_COUNT = B_TE + 2;
static_assert(B_COUNT * 8 <= 512, "barrier area");

constexpr uint32_t kCols = 128;  // TMEM: S^T at 0 / 16, O^T at 32 + 16 e (e < NE)
constexpr uint32_t TM_S = 0, TM_O = 32;
static_assert(TM_O + 16 * NE <= kCols, "TMEM columns");

__device__ __forceinline__ uint32_t pt_addr(uint32_t base, int q, int k) {
  // [16 queries][128 keys] bf16, K-major, 128-byte swizzle: keys 0-63 and
  // 64-127 in two 2 KB atoms of 16 rows
  const int kk = k & 63;
  return base + (uint32_t)((k >> 6) * 2048 + (q >> 3) * 1024 + (q & 7) * 128 +
                           ((((kk >> 3) ^ (q & 7))) << 4) + (kk & 7) * 2);
}
__device__ __forceinline__ void sts_u16(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.u16 [%0], %1;\n" ::"r"(addr), "h"((unsigned short)v) : "memory");
}
// Barrier over the 128 threads of one warpgroup (named barrier `id`) that also
// returns whether `pred` held for any of them.
__device__ __forceinline__ bool bar_or(int id, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.or.pred q, %2, 128, p;\n"
      " selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void bar_sync128(int id) {
  asm volatile("bar.sync %0, 128;\n" ::"r"(id) : "memory");
}

// Top-left patch (column, row within the frame grid) and frame of block beta,
// and how many of its P x P patches exist in each direction.
struct Blk {
  int f, c0, r0, nr, nc;
};
__device__ __forceinline__ Blk block_of(const Dims& d, int beta) {
  Blk b;
  b.f = udiv31(beta, d.Bf, d.mBf);
  const int j = beta - b.f * d.Bf;
  const int br = udiv31(j, d.Bw, d.mBw), bc = j - br * d.Bw;
  b.r0 = br * d.P;
  b.c0 = bc * d.P;
  b.nr = min(d.P, d.Hp - b.r0);
  b.nc = min(d.P, d.Wp - b.c0);
  return b;
}

struct Maps {
  CUtensorMap q5;          // per-frame grid view of Q, box 4 x 4 patches of one head
  CUtensorMap q3;          // [T][H][64], box one token of one head (special entries)
  CUtensorMap ks, vs;      // [H][NK][64] kept copies, box 128 keys (kept keys streamed inline)
};

__global__ void __launch_bounds__(kThreads, 1)
    selected_tc_kernel(const __grid_constant__ Maps mp, const Dims d, const bf16* __restrict__ kg,
                       const bf16* __restrict__ vg, const int* __restrict__ sel,
                       const int* __restrict__ order, const float* __restrict__ qc32,
                       const float* __restrict__ w, const float* __restrict__ oc, bf16* __restrict__ out,
                       float* __restrict__ lse, const float* __restrict__ o_spec,
                       const float* __restrict__ lse_spec, unsigned* err, int kept_inline) {
  extern __shared__ __align__(1024) uint8_t st_smem_raw[];
  const uint32_t raw = smem_u32(st_smem_raw);
  const uint32_t sb = (raw + 1023u) & ~1023u;
  uint8_t* sp = st_smem_raw + (sb - raw);
  auto bar = [&](int i) -> uint32_t { return sb + OFF_BAR + 8u * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sp + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sp + OFF_MISC + 4);
  auto ent = [&](int s) -> Entry& { return *reinterpret_cast<Entry*>(sp + OFF_ENT + s * kEntBytes); };

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long n_items = (long long)d.H * d.Tc;
  const int n_kept_tiles = kept_inline ? (int)((d.NK + TKEYS - 1) / TKEYS) : 0;

  if (tid == 0) {
    for (int s = 0; s < NE; ++s) {
      mbar_init(bar(B_EF + s), 1);
      mbar_init(bar(B_EE + s), 128);
      mbar_init(bar(B_EM + s), 1);
      mbar_init(bar(B_OF + s), 1);
    }
    for (int s = 0; s < ST; ++s) {
      mbar_init(bar(B_KF + s), 32);  // one arrival per producer lane
      mbar_init(bar(B_VF + s), 32);
      mbar_init(bar(B_KE + s), 1);
      mbar_init(bar(B_VE + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(B_SF + b), 1);
      mbar_init(bar(B_PF + b), 128);
      mbar_init(bar(B_PE + b), 1);
    }
    mbar_init(bar(B_OD), 1);
    mbar_init(bar(B_DRAIN), 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(B_TF + b), 32);  // token list b written (every builder lane)
      mbar_init(bar(B_TE + b), 32);  // token list b read (every gather lane)
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  {
    // the ones rows of the value operand, and zeroed query tiles (slots a
    // special entry leaves unused must hold finite values)
    uint4* ones = reinterpret_cast<uint4*>(sp + OFF_ONES);
    for (int i = tid; i < (int)(kKV / 16); i += kThreads)
      ones[i] = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
    uint4* qz = reinterpret_cast<uint4*>(sp + OFF_Q);
    for (int i = tid; i < (int)(NE * kQ / 16); i += kThreads) qz[i] = make_uint4(0u, 0u, 0u, 0u);
    // the K/V ring: gathered tiles copy only their valid key slots, so the
    // rest must start finite
    uint4* kvz = reinterpret_cast<uint4*>(sp + OFF_K);
    for (int i = tid; i < (int)(2 * ST * kKV / 16); i += kThreads) kvz[i] = make_uint4(0u, 0u, 0u, 0u);
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

  if (warp == 0) {
    // ---------------- TMA producer (the whole warp) ----------------
    if (lane == 0) {
      prefetch_tmap(&mp.q5);
      prefetch_tmap(&mp.q3);
    }
    const int KU = (d.K + 31) / 32;  // ids per lane
    // the selection and the pair of an entry are loaded one entry ahead, so
    // their latency overlaps the gathers of the entry before
    auto pair_of = [&](long long item) -> long long {
      return item < n_items ? (order != nullptr ? (long long)order[item] : item) : -1;
    };
    // The query slot `lane` (< 16) of a pair: its token (or -1), and the
    // always-kept segment's log-sum-exp for it, in log2 units (-inf without).
    struct QSlot {
      long long t;
      float m0;
    };
    auto query_slot = [&](long long pair) -> QSlot {
      QSlot r{-1, -CUDART_INF_F};
      if (pair < 0 || lane >= NQ) return r;
      const int h = pair < 0x7fffffffLL ? udiv31((int)pair, (int)d.Tc, d.mTc) : (int)(pair / d.Tc);
      const int a = (int)(pair - (long long)h * d.Tc);
      const int f = udiv31(a, d.E, d.mE), j = a - f * d.E;
      if (j < d.S) {
        if (lane == 0) r.t = (long long)f * d.L + j;
      } else {
        const Blk qb = block_of(d, f * d.Bf + (j - d.S));
        const int pr = lane >> 2, pc = lane & 3;
        if (pr < qb.nr && pc < qb.nc) r.t = (long long)f * d.L + d.S + (long long)(qb.r0 + pr) * d.Wp + qb.c0 + pc;
      }
      if (r.t >= 0 && lse_spec != nullptr) r.m0 = lse_spec[r.t * d.H + h] * 1.4426950408889634f;
      return r;
    };
    long long pair_cur = pair_of(blockIdx.x);
    long long pair_nxt = pair_of(blockIdx.x + (long long)gridDim.x);
    int ids_cur[kMaxTopK / 32];
#pragma unroll
    for (int u = 0; u < kMaxTopK / 32; ++u) {
      const int k = lane + 32 * u;
      ids_cur[u] = (u < KU && k < d.K && pair_cur >= 0) ? sel[pair_cur * d.K + k] : -1;
    }
    QSlot qs_cur = query_slot(pair_cur);
    int ne = 0;  // entries built
    bool ok = true;
    for (long long it = blockIdx.x; ok && it < n_items; it += gridDim.x, ++ne) {
      const int es = ne % NE;
      // prefetch: the next entry's selection and query slots, the pair after it
      int ids_nxt[kMaxTopK / 32];
#pragma unroll
      for (int u = 0; u < kMaxTopK / 32; ++u) {
        const int k = lane + 32 * u;
        ids_nxt[u] = (u < KU && k < d.K && pair_nxt >= 0) ? sel[pair_nxt * d.K + k] : -1;
      }
      const QSlot qs_nxt = query_slot(pair_nxt);
      const long long pair_nn = pair_of(it + 2LL * gridDim.x);
      // the entry slot is free once the epilogue is done with it; the token
      // list buffer once the gather warp has read it
      const int lb = ne & 1;
      if ((ne >= NE && !__all_sync(0xffffffffu, mbar_wait(bar(B_EE + es), ((ne / NE) - 1) & 1, abort_flag, err, d.wait_cycles))) ||
          (ne >= 2 && !__all_sync(0xffffffffu, mbar_wait(bar(B_TE + lb), ((ne >> 1) - 1) & 1, abort_flag, err, d.wait_cycles)))) {
        ok = false;
        break;
      }
      int* tok_list = reinterpret_cast<int*>(sp + OFF_TOK) + lb * kTokList;
      const long long pair = pair_cur;
      const int h = pair < 0x7fffffffLL ? udiv31((int)pair, (int)d.Tc, d.mTc) : (int)(pair / d.Tc);
      const int a = (int)(pair - (long long)h * d.Tc);
      Entry& E = ent(es);
      // the selection: ascending ids, -1 padded; an id outside [0, NB) ends the
      // list and raises the device-check bit instead of being dereferenced
      int nsel = d.K;
#pragma unroll
      for (int u = 0; u < kMaxTopK / 32; ++u) {
        if (u >= KU) break;
        const int k = lane + 32 * u;
        const bool in = k < d.K;
        const unsigned bad = __ballot_sync(0xffffffffu, in && (ids_cur[u] < 0 || ids_cur[u] >= d.NB));
        const unsigned oob = __ballot_sync(0xffffffffu, in && ids_cur[u] >= d.NB);
        if (oob != 0 && lane == 0) atomicOr(err, kErrDeviceCheck);
        if (bad != 0 && nsel == d.K) nsel = 32 * u + __ffs(bad) - 1;
      }
      // the valid tokens of the selected blocks, in selection order, packed
      // into consecutive key slots: a prefix sum of the blocks' token counts;
      // a block's valid patches are its first nr rows and nc columns
      int carry = 0;
#pragma unroll
      for (int u = 0; u < kMaxTopK / 32; ++u) {
        if (u >= KU || 32 * u >= nsel) break;
        const int k = lane + 32 * u;
        Blk kb{0, 0, 0, 0, 0};
        int cnt = 0;
        if (k < nsel) {
          kb = block_of(d, ids_cur[u]);
          cnt = kb.nr * kb.nc;
        }
        int incl = cnt;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, off);
          if (lane >= off) incl += y;
        }
        int pos = carry + incl - cnt;
        const long long t0 = (long long)kb.f * d.L + d.S + (long long)kb.r0 * d.Wp + kb.c0;
#pragma unroll
        for (int pr = 0; pr < kMaxPool; ++pr) {
#pragma unroll
          for (int pc = 0; pc < kMaxPool; ++pc) {
            if (pr < kb.nr && pc < kb.nc) {
              tok_list[pos] = (int)(t0 + (long long)pr * d.Wp + pc);
              ++pos;
            }
          }
        }
        carry += __shfl_sync(0xffffffffu, incl, 31);
      }
      const int n_keys = carry;
      const int n_tiles = n_kept_tiles + (n_keys + TKEYS - 1) / TKEYS;
      // the entry's queries (tokens and references prefetched with the selection)
      const int f = udiv31(a, d.E, d.mE), j = a - f * d.E;
      const bool special = j < d.S;
      Blk qb{0, 0, 0, 0, 0};
      if (!special) qb = block_of(d, f * d.Bf + (j - d.S));
      if (lane < NQ) {
        E.tok[lane] = (int)qs_cur.t;
        E.m0[lane] = qs_cur.m0;
      }
      const unsigned qm = __ballot_sync(0xffffffffu, lane < NQ && qs_cur.t >= 0);
      if (lane == 0) {
        E.h = h;
        E.a = a;
        E.n_keys = n_keys;
        E.n_kept = n_kept_tiles;
        E.n_tiles = n_tiles;
        E.qmask = qm & 0xffffu;
      }
      __syncwarp();  // the entry info and the token list are written
      if (lane == 0) {
        // the one arrival on the entry's barrier (arrive.expect_tx, release: it
        // also publishes the info the warp wrote above); the phase completes
        // once the query box has landed
        const uint32_t dq = sb + OFF_Q + es * kQ;
        if (special) {
          mbar_expect_tx(bar(B_EF + es), 128);
          tma_load_3d(dq, &mp.q3, bar(B_EF + es), 0, h, f * d.L + j);
        } else {
          mbar_expect_tx(bar(B_EF + es), kQ);
          tma_load_5d(dq, &mp.q5, bar(B_EF + es), 0, h, qb.c0, qb.r0, f);
        }
      }
      // hand the token list to the gather warp (every lane arrives: release
      // of its own writes)
      mbar_arrive(bar(B_TF + lb));
#pragma unroll
      for (int u = 0; u < kMaxTopK / 32; ++u) ids_cur[u] = ids_nxt[u];
      qs_cur = qs_nxt;
      pair_cur = pair_nxt;
      pair_nxt = pair_nn;
    }
    if (*abort_flag && lane == 0) {
      // let this CTA's query boxes land before its shared memory goes away
      volatile int never = 0;
      for (int e = ne - 1; e >= 0 && e >= ne - NE; --e) mbar_wait(bar(B_EF + e % NE), (e / NE) & 1, &never, err);
    }
  } else if (warp == 3) {
    // ---------------- gather warp ----------------
    // per entry, once its token list is handed over: the key tiles into the
    // K/V ring; every lane arrives once on the tile's K and V barriers (count
    // 32): through the TMA transaction count for the always-kept tiles,
    // through cp.async completion for the gathered ones
    int gt = 0;  // tiles loaded
    int ne = 0;  // entries taken
    bool ok = true;
    const long long row = (long long)d.H * kHeadDim;
    for (long long it = blockIdx.x; ok && it < n_items; it += gridDim.x, ++ne) {
      const int es = ne % NE, lb = ne & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(B_TF + lb), (ne >> 1) & 1, abort_flag, err, d.wait_cycles))) {
        ok = false;
        break;
      }
      const int* tl = reinterpret_cast<const int*>(sp + OFF_TOK) + lb * kTokList;
      const Entry& E = ent(es);
      const int n_tiles = E.n_tiles, n_kept = E.n_kept, n_keys = E.n_keys, h = E.h;
      const long long hoff = (long long)h * kHeadDim;
      for (int i = 0; ok && i < n_tiles; ++i, ++gt) {
        const int s = gt % ST;
        if (gt >= ST) {
          const uint32_t ph = ((gt / ST) - 1) & 1;
          if (!__all_sync(0xffffffffu, mbar_wait(bar(B_KE + s), ph, abort_flag, err, d.wait_cycles) &&
                                          mbar_wait(bar(B_VE + s), ph, abort_flag, err, d.wait_cycles))) {
            ok = false;
            break;
          }
        }
        const uint32_t dk = sb + OFF_K + s * kKV, dv = sb + OFF_V + s * kKV;
        if (i < n_kept) {
          if (lane == 0) {
            mbar_expect_tx(bar(B_KF + s), kKV);
            mbar_expect_tx(bar(B_VF + s), kKV);
            tma_load_3d(dk, &mp.ks, bar(B_KF + s), 0, i * TKEYS, h);
            tma_load_3d(dv, &mp.vs, bar(B_VF + s), 0, i * TKEYS, h);
          } else {
            mbar_arrive(bar(B_KF + s));
            mbar_arrive(bar(B_VF + s));
          }
        } else {
          // key slot c of the tile = packed slot 128 i' + c; row c of the
          // operand tile is that token's 128 bytes, its 16-byte chunks in the
          // 128-byte swizzle.  Only the valid slots are copied: the rest keep
          // finite data (zeroed at start, or an earlier tile's rows) that the
          // softmax masks to weight 0.  A lane copies chunk lane % 8 of keys
          // lane / 8 + 4 m.
          const int g0 = (i - n_kept) * TKEYS;
          const int nv = min(TKEYS, n_keys - g0);
          const int ch = lane & 7;
          const bf16* kh = kg + hoff + ch * 8;
          const bf16* vh = vg + hoff + ch * 8;
#pragma unroll 4
          for (int c = lane >> 3; c < nv; c += 4)
            cp_async16(dk + (uint32_t)(c * 128 + ((ch ^ (c & 7)) << 4)), kh + (long long)tl[g0 + c] * row, true);
          cp_async_mbar_arrive_noinc(bar(B_KF + s));
#pragma unroll 4
          for (int c = lane >> 3; c < nv; c += 4)
            cp_async16(dv + (uint32_t)(c * 128 + ((ch ^ (c & 7)) << 4)), vh + (long long)tl[g0 + c] * row, true);
          cp_async_mbar_arrive_noinc(bar(B_VF + s));
        }
      }
      // the token list may be rebuilt (its reads are done)
      mbar_arrive(bar(B_TE + lb));
    }
    cp_async_wait<0>();  // this lane's gathers have landed
    if (*abort_flag && lane == 0) {
      // let this CTA's own copies land before its shared memory goes away
      volatile int never = 0;
      for (int g = gt - 1; g >= 0 && g >= gt - ST; --g) {
        mbar_wait(bar(B_KF + g % ST), (g / ST) & 1, &never, err);
        mbar_wait(bar(B_VF + g % ST), (g / ST) & 1, &never, err);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t id_s = idesc(128, 16, kFmtBF16, 0, 0);
      const uint32_t id_o = idesc(128, 16, kFmtBF16, 1, 0);
      int gt = 0, ne = 0;
      bool ok = true;
      // the tile whose O^T product is still to be issued
      bool pend = false;
      int p_g = 0, p_s = 0, p_b = 0, p_es = 0;  // the pending tile: global index, stage, buffer, entry slot
      bool p_first = false, p_last = false;
      auto finish = [&]() -> bool {
        const int g = p_g;
        if (!mbar_wait(bar(B_VF + p_s), (g / ST) & 1, abort_flag, err, d.wait_cycles) ||
            !mbar_wait(bar(B_PF + p_b), (g >> 1) & 1, abort_flag, err, d.wait_cycles))
          return false;
        fence_after_sync();
        fence_proxy_async_smem();
        const uint32_t sv = sb + OFF_V + p_s * kKV;
        const uint32_t lbo = (sb + OFF_ONES) - sv;  // value dims, then the ones rows
        const uint32_t spt = sb + OFF_PT + p_b * kPT;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ss(tbase + TM_O + p_es * 16, sdesc(sv + kk * 2048, lbo, 1024),
                      sdesc_k(spt + (kk >> 2) * 2048 + (kk & 3) * 32), id_o, (!p_first || kk > 0) ? 1u : 0u);
        mma_commit(bar(B_VE + p_s));
        mma_commit(bar(B_PE + p_b));
        mma_commit(bar(B_OD));
        if (p_last) mma_commit(bar(B_OF + p_es));
        pend = false;
        return true;
      };
      for (long long it = blockIdx.x; ok && it < n_items; it += gridDim.x, ++ne) {
        const int es = ne % NE;
        if (!mbar_wait(bar(B_EF + es), (ne / NE) & 1, abort_flag, err, d.wait_cycles)) {
          ok = false;
          break;
        }
        const int n = ent(es).n_tiles;
        if (n == 0) {
          if (pend && !(ok = finish())) break;
          mma_commit(bar(B_OF + es));  // nothing to add: the epilogue may start
          continue;
        }
        const uint32_t sq = sb + OFF_Q + es * kQ;
        for (int i = 0; i < n; ++i) {
          const int s = gt % ST, b = gt & 1;
          // S^T(t+1) goes first when its keys have landed (the tensor core
          // then works while the softmax finishes tile t); otherwise O^T(t)
          // is issued at once, so that its entry's epilogue is not held up by
          // the next tile's gathers
          if (pend && !mbar_peek(bar(B_KF + s), (gt / ST) & 1) && !(ok = finish())) break;
          if (!mbar_wait(bar(B_KF + s), (gt / ST) & 1, abort_flag, err, d.wait_cycles)) {
            ok = false;
            break;
          }
          fence_after_sync();
          fence_proxy_async_smem();  // the gathered rows were written by cp.async (generic proxy)
          const uint32_t sk = sb + OFF_K + s * kKV;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ss(tbase + TM_S + b * 16, sdesc_k(sk + kk * 32), sdesc_k(sq + kk * 32), id_s, kk > 0);
          mma_commit(bar(B_SF + b));
          mma_commit(bar(B_KE + s));
          if (pend && !(ok = finish())) break;
          pend = true;
          p_g = gt++;
          p_s = s;
          p_b = b;
          p_es = es;
          p_first = i == 0;
          p_last = i == n - 1;
        }
      }
      if (ok && pend) ok = finish();
      if (!ok) {
        volatile int never = 0;
        mma_commit(bar(B_DRAIN));
        mbar_wait(bar(B_DRAIN), 0, &never, err);
      }
    }
  } else if (warp >= 4 && warp < 8) {
    // ---------------- softmax, one thread per key lane ----------------
    const int q4 = warp & 3;
    const int k = q4 * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const float c2 = d.scale_log2;
    float* red = reinterpret_cast<float*>(sp + OFF_RED);
    int gt = 0, ne = 0;
    bool ok = true;
    for (long long it = blockIdx.x; ok && it < n_items; it += gridDim.x, ++ne) {
      const int es = ne % NE;
      // every wait's outcome is agreed on by the whole warpgroup (bar.red), so
      // the 128 threads always reach the same named barriers
      if (bar_or(1, !mbar_wait(bar(B_EF + es), (ne / NE) & 1, abort_flag, err, d.wait_cycles))) {
        ok = false;
        break;
      }
      const Entry& E = ent(es);
      const int n = E.n_tiles, nk = E.n_kept, n_keys = E.n_keys;
      const uint32_t qmask = E.qmask;
      // reference per query; the weight of the always-kept segment (1 when
      // its normalised state is supplied, scaled down with every raise of the
      // reference) is kept in the entry by one thread
      float m[NQ];
#pragma unroll
      for (int q = 0; q < NQ; ++q) m[q] = E.m0[q];
      Entry& Ew = ent(es);
      if (tid == 128) {
#pragma unroll
        for (int q = 0; q < NQ; ++q) Ew.wf[q] = (lse_spec != nullptr && ((qmask >> q) & 1u)) ? 1.f : 0.f;
      }
      for (int i = 0; i < n; ++i, ++gt) {
        const int b = gt & 1;
        // is this lane's key a real key of the tile?
        const bool kvalid = i < nk ? (long long)i * TKEYS + k < d.NK : (i - nk) * TKEYS + k < n_keys;
        // P^T buffer b is free once the O^T product of tile gt - 2 is complete;
        // S^T(gt) is in TMEM once its product is.  Both waits and the test for
        // a raise of the references are decided together by one OR barrier in
        // the common case.
        bool waited = gt < 2 || mbar_wait(bar(B_PE + b), ((gt >> 1) - 1) & 1, abort_flag, err, d.wait_cycles);
        waited = waited && mbar_wait(bar(B_SF + b), (gt >> 1) & 1, abort_flag, err, d.wait_cycles);
        waited = __all_sync(0xffffffffu, waited);  // tcgen05.ld below is warp-collective
        fence_after_sync();
        uint32_t sv[NQ];
        float x[NQ];
        float xmax = -CUDART_INF_F;
        if (waited) {
          tmem_ld16(tbase + lane_off + TM_S + b * 16, sv);
          tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < NQ; ++q) {
            const bool use = kvalid && ((qmask >> q) & 1u);
            x[q] = use ? fmaf(__uint_as_float(sv[q]), c2, -m[q]) : -CUDART_INF_F;
            xmax = fmaxf(xmax, x[q]);
          }
        }
        // a score above its query's reference by 2^8 (or a query without one
        // yet): raise the references of this tile's queries to their maxima
        if (bar_or(1, !waited || xmax > 8.f)) {
          if (bar_or(1, !waited)) {
            ok = false;
            break;
          }
          float tm[NQ];
#pragma unroll
          for (int q = 0; q < NQ; ++q) {
            float v = (kvalid && ((qmask >> q) & 1u)) ? __uint_as_float(sv[q]) * c2 : -CUDART_INF_F;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
            tm[q] = v;
          }
          if (lane < NQ) {
            float v = tm[0];
#pragma unroll
            for (int q = 1; q < NQ; ++q)
              if (lane == q) v = tm[q];
            red[q4 * NQ + lane] = v;
          }
          bar_sync128(1);
          float corr[NQ];
#pragma unroll
          for (int q = 0; q < NQ; ++q) {
            const float t = fmaxf(fmaxf(red[q], red[NQ + q]), fmaxf(red[2 * NQ + q], red[3 * NQ + q]));
            const float mn = fmaxf(m[q], t);
            corr[q] = mn == -CUDART_INF_F ? 1.f : exp2f(m[q] - mn);
            m[q] = mn;
            if (tid == 128) Ew.wf[q] *= corr[q];
          }
          bar_sync128(1);  // red is reused by the next tile
          if (i > 0) {
            // this entry's partial O^T (and sums) must be complete, then rescaled
            if (bar_or(1, !mbar_wait(bar(B_OD), (gt - 1) & 1, abort_flag, err, d.wait_cycles))) {
              ok = false;
              break;
            }
            fence_after_sync();
            uint32_t ov[NQ];
            tmem_ld16(tbase + lane_off + TM_O + es * 16, ov);
            tmem_wait_ld();
#pragma unroll
            for (int q = 0; q < NQ; ++q) ov[q] = __float_as_uint(__uint_as_float(ov[q]) * corr[q]);
            tmem_st16(tbase + lane_off + TM_O + es * 16, ov);
            tmem_wait_st();
          }
#pragma unroll
          for (int q = 0; q < NQ; ++q) {
            const bool use = kvalid && ((qmask >> q) & 1u);
            x[q] = use ? fmaf(__uint_as_float(sv[q]), c2, -m[q]) : -CUDART_INF_F;
          }
        }
        uint32_t pk[NQ / 2];
#pragma unroll
        for (int u = 0; u < NQ / 2; ++u) pk[u] = exp2_bf16x2(x[2 * u], x[2 * u + 1]);
        const uint32_t spt = sb + OFF_PT + b * kPT;
#pragma unroll
        for (int u = 0; u < NQ / 2; ++u) {
          sts_u16(pt_addr(spt, 2 * u, k), pk[u] & 0xffffu);
          sts_u16(pt_addr(spt, 2 * u + 1, k), pk[u] >> 16);
        }
        fence_proxy_async_smem();
        fence_before_sync();
        mbar_arrive(bar(B_PF + b));
      }
      if (!ok) break;
      if (tid == 128) {
#pragma unroll
        for (int q = 0; q < NQ; ++q) Ew.mf[q] = m[q];
        mbar_arrive(bar(B_EM + es));
      }
    }
  } else if (warp >= 8) {
    // ---------------- epilogue, one thread per TMEM lane ----------------
    const int q4 = warp & 3;
    const int dlane = q4 * 32 + lane;  // lanes 0-63: value dims; 64-127: sums of P
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    float* ls = reinterpret_cast<float*>(sp + OFF_LS);  // [16] reciprocal denominators
    float* gz = reinterpret_cast<float*>(sp + OFF_GATE);
    const long long row = (long long)d.H * kHeadDim;
    int ne = 0;
    bool ok = true;
    for (long long it = blockIdx.x; ok && it < n_items; it += gridDim.x, ++ne) {
      const int es = ne % NE;
      const uint32_t ph = (ne / NE) & 1;
      // the entry is known once its info has landed: its global loads (the
      // always-kept segment's outputs, the compressed output, the gate's
      // inputs) are issued now, all at once, so that their latency overlaps
      // the entry's products instead of following them one by one
      if (bar_or(2, !mbar_wait(bar(B_EF + es), ph, abort_flag, err, d.wait_cycles))) {  // agreed on by all four warps
        ok = false;
        break;
      }
      const Entry& E = ent(es);
      const int h = E.h, a = E.a;
      const uint32_t qmask = E.qmask;
      float osv[NQ];
      float cmp = 0.f, zpart = 0.f;
      if (dlane < 64) {
#pragma unroll
        for (int q = 0; q < NQ; ++q)
          osv[q] = (o_spec != nullptr && ((qmask >> q) & 1u))
                       ? o_spec[((long long)E.tok[q] * d.H + h) * kHeadDim + dlane] : 0.f;
        if (w != nullptr) {
          cmp = oc[((long long)a * d.H + h) * kHeadDim + dlane];
          zpart = qc32[((long long)a * d.H + h) * kHeadDim + dlane] * w[(long long)h * kHeadDim + dlane];
        }
      }
      const bool got = mbar_wait(bar(B_EM + es), ph, abort_flag, err, d.wait_cycles) &&
                       mbar_wait(bar(B_OF + es), ph, abort_flag, err, d.wait_cycles);
      if (bar_or(2, !got)) {
        ok = false;
        break;
      }
      fence_after_sync();
      uint32_t ov[NQ];
      if (E.n_tiles > 0) {
        tmem_ld16(tbase + lane_off + TM_O + es * 16, ov);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int q = 0; q < NQ; ++q) ov[q] = 0u;
      }
      if (dlane >= 64 && dlane < 64 + NQ) {
        // rows 64-127 of O^T all hold the sums of P: thread 64 + q forms
        // query q's denominator (the always-kept segment's weight plus the
        // sum), its reciprocal for the value threads, and the log-sum-exp
        const int q = dlane - 64;
        float sq = 0.f;
#pragma unroll
        for (int u = 0; u < NQ; ++u)
          if (u == q) sq = __uint_as_float(ov[u]);
        const float den = E.wf[q] + sq;
        ls[q] = 1.f / den;
        if (w == nullptr && lse != nullptr && ((qmask >> q) & 1u))
          lse[(long long)E.tok[q] * d.H + h] = (E.mf[q] + log2f(den)) * 0.6931471805599453f;
      }
      if (w != nullptr && dlane < 64) {
        float z = zpart;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
        if (lane == 0) gz[q4] = z;
      }
      bar_sync128(2);
      if (dlane < 64) {
        const float g = w != nullptr ? 1.f / (1.f + expf(-(gz[0] + gz[1]))) : 0.f;
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
          if (!((qmask >> q) & 1u)) continue;
          const long long t = E.tok[q];
          const float o = fmaf(E.wf[q], osv[q], __uint_as_float(ov[q])) * ls[q];
          const long long ob = t * row + (long long)h * kHeadDim + dlane;
          out[ob] = __float2bfloat16_rn(w != nullptr ? g * cmp + (1.f - g) * o : o);
        }
      }
      bar_sync128(2);  // ls / gz are reused by the next entry
      fence_before_sync();
      mbar_arrive(bar(B_EE + es));
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

cudaError_t launch_selected_tc(const Dims& d, const bf16* q, const bf16* k, const bf16* v,
                               const bf16* ks, const bf16* vs, const int* sel, const int* order,
                               const float* qc32, const float* w, const float* oc, bf16* out,
                               float* lse, const float* o_spec, const float* lse_spec, unsigned* err,
                               cudaStream_t st) {
  const unsigned long long H = (unsigned long long)d.H;
  const unsigned long long rowb = H * 128;  // bytes per token row
  Maps mp;
  // per-frame grid view of [T][H][64] starting at the first patch of frame 0:
  // (value, head, column, row, frame) with strides (2, 128, rowb, Wp rowb, L rowb)
  const unsigned long long dims5[5] = {64, H, (unsigned long long)d.Wp, (unsigned long long)d.Hp,
                                       (unsigned long long)d.N};
  const unsigned long long str5[4] = {128, rowb, (unsigned long long)d.Wp * rowb, (unsigned long long)d.L * rowb};
  const unsigned box5[5] = {64, 1, 4, 4, 1};
  const long long off = (long long)d.S * d.H * kHeadDim;
  bool ok = make_tmap(&mp.q5, q + off, 5, dims5, str5, box5);
  const unsigned long long dims3[3] = {64, H, (unsigned long long)d.T};
  const unsigned long long str3[2] = {128, rowb};
  const unsigned box3[3] = {64, 1, 1};
  ok = ok && make_tmap(&mp.q3, q, 3, dims3, str3, box3);
  const int kept_inline = (o_spec == nullptr && d.NK > 0) ? 1 : 0;
  if (kept_inline) {
    const unsigned long long dk[3] = {64, (unsigned long long)d.NK, H};
    const unsigned long long sk[2] = {128, (unsigned long long)d.NK * 128};
    const unsigned bk[3] = {64, 128, 1};
    ok = ok && make_tmap(&mp.ks, ks, 3, dk, sk, bk) && make_tmap(&mp.vs, vs, 3, dk, sk, bk);
  } else {
    mp.ks = mp.q3;
    mp.vs = mp.q3;
  }
  if (!ok) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(selected_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long items = (long long)d.H * d.Tc;
  const long long grid = items < (long long)sms ? items : (long long)sms;
  if (grid <= 0) return cudaSuccess;
  selected_tc_kernel<<<(unsigned)grid, kThreads, kSmemBytes, st>>>(mp, d, k, v, sel, order, qc32, w, oc, out, lse,
                                                                  o_spec, lse_spec, err, kept_inline);
  return cudaGetLastError();
}

}  // namespace gsa
