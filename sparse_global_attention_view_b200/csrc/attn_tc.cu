// Exact attention on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// Used for the dense global attention (Speed3R technical summary 1), the
// always-kept segment of the selection branch (2.1, 2.2), frame attention
// (keys restricted to the query's own frame: per-frame key segments; AVGGT
// 2.2) and the kept keys of subsampled global attention (AVGGT 2.2).
//
// One CTA = two 128-row query tiles of one head (TMEM lanes = rows) and 12 warps:
//   warp 0      TMA producer: Q tiles once, then a 4-stage ring of 128-key K/V
//               tiles (128-byte swizzle, out-of-range rows zero-filled);
//   warp 1      MMA issuer (one thread): S_t = Q_t K^T (bf16, fp32 in TMEM),
//               then O_t += P_t V with P_t read from TMEM;
//   warp 2      TMEM allocation (512 columns: S_0, S_1, O_0, O_1);
//   warps 4-11  softmax, one warpgroup per query tile, one thread per row.
// The MMA thread interleaves the two tiles so one tile's softmax overlaps the
// other tile's matrix products.  The softmax keeps eight independent max and
// sum chains and takes a quarter of its exponentials on the FMA pipe.  The softmax keeps a stale maximum until a
// tile's maximum exceeds it by 2^8 and only then rescales O (in TMEM), so the
// common case never waits for the tensor core.  Every mbarrier wait is
// bounded: on timeout the CTA records kErrTimeout, raises its abort flag, drains
// its own TMA loads and MMAs, frees TMEM and returns.
#include <math_constants.h>

#include <mutex>

#include "internal.h"
#include "tc_common.cuh"

namespace gsa {
namespace {

using namespace tc;

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}
// 2^x on the FMA pipe, for a quarter of the softmax's exponentials so that the
// special-function unit is not the only bound: Cody-Waite range reduction
// x = j + f, j = round(x) (added to the exponent bits), f in [-1/2, 1/2], and a
// cubic fitted to 2^f on that interval by iteratively reweighted least squares
// on Chebyshev nodes (max relative error 7.5e-5 in fp32, below the bf16
// rounding of P).  x is clamped at -125 (the result is then ~2^-125, i.e. 0 for
// the softmax).  Both halves of a pair are computed with the paired forms of
// the additions and multiply-adds.
__device__ __forceinline__ uint64_t exp2_fma2(uint64_t x2) {
  float x0, x1;
  f2_unpack(x2, x0, x1);
  const uint64_t x = f2_pack(fmaxf(x0, -125.f), fmaxf(x1, -125.f));
  const uint64_t big = f2_pack(12582912.f, 12582912.f);
  const uint64_t t = f2_add(x, big);
  float t0, t1;
  f2_unpack(t, t0, t1);
  const uint64_t f = f2_sub(x, f2_sub(t, big));
  uint64_t p = f2_fma(f2_pack(0.055171769f, 0.055171769f), f, f2_pack(0.24261113f, 0.24261113f));
  p = f2_fma(p, f, f2_pack(0.69326097f, 0.69326097f));
  p = f2_fma(p, f, f2_pack(0.99992806f, 0.99992806f));
  float p0, p1;
  f2_unpack(p, p0, p1);
  return f2_pack(__int_as_float(__float_as_int(p0) + ((__float_as_int(t0) - 0x4B400000) << 23)),
                 __int_as_float(__float_as_int(p1) + ((__float_as_int(t1) - 0x4B400000) << 23)));
}


constexpr int kPolyOf8 = 2;        // exponential pairs of every eight taken on the FMA pipe
constexpr int TQ = 128;            // rows per query tile
constexpr int NQT = 2;             // query tiles per CTA
constexpr int TK = 128;            // keys per key tile
constexpr int ST = 4;              // K/V ring stages
constexpr int kThreads = 384;
constexpr uint32_t kTile = 128 * 128;  // bytes of one [128][64] bf16 tile

constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_K = OFF_Q + NQT * kTile;
constexpr uint32_t OFF_V = OFF_K + ST * kTile;
constexpr uint32_t OFF_BAR = OFF_V + ST * kTile;
constexpr uint32_t OFF_MISC = OFF_BAR + 256;
constexpr uint32_t kSmemBytes = OFF_MISC + 64 + 1024;  // + alignment slack

// barrier indices
constexpr int B_Q = 0, B_KF = 1, B_VF = B_KF + ST, B_KVE = B_VF + ST, B_SF = B_KVE + ST,
              B_PF = B_SF + NQT, B_OF = B_PF + NQT, B_DRAIN = B_OF + NQT, B_COUNT = B_DRAIN + 1;
static_assert(B_COUNT * 8 <= 256, "barrier area");

constexpr uint32_t kCols = 512;  // TMEM columns: S_t at 128 t, O_t at 256 + 64 t
// Register split between the producer/MMA warpgroup and the two softmax
// warpgroups; it must not exceed the launch allocation, or the increase would
// wait forever (the host checks the compiled register count before launching).
constexpr int kLaunchRegs = 168, kRegsLow = 72, kRegsHigh = 216;
static_assert(128 * kRegsLow + 256 * kRegsHigh <= kThreads * kLaunchRegs, "register split");

__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                   const __grid_constant__ CUtensorMap tv, const AttnTcArgs a) {
  extern __shared__ __align__(1024) uint8_t tc_smem_raw[];
  const uint32_t raw = smem_u32(tc_smem_raw);
  const uint32_t sb = (raw + 1023u) & ~1023u;
  uint8_t* sp = tc_smem_raw + (sb - raw);
  const uint32_t sQ = sb + OFF_Q, sK = sb + OFF_K, sV = sb + OFF_V;
  auto bar = [&](int i) -> uint32_t { return sb + OFF_BAR + 8u * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sp + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sp + OFF_MISC + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.y;
  // Segments: with seg_len > 0 the rows and keys are cut into consecutive
  // segments of seg_len tokens (frames) and every query attends only to the
  // keys of its own segment; seg_ctas CTAs cover one segment's queries.
  long long m0, key0, n_keys, q_end;
  if (a.seg_len > 0) {
    const long long f = blockIdx.x / a.seg_ctas, cx = blockIdx.x % a.seg_ctas;
    key0 = f * a.seg_len;
    m0 = key0 + cx * (NQT * TQ);
    n_keys = a.seg_len;
    q_end = min(key0 + a.seg_len, a.n_q);
  } else {
    key0 = 0;
    m0 = (long long)blockIdx.x * (NQT * TQ);
    n_keys = a.n_k;
    q_end = a.n_q;
  }
  const int nt = (int)((n_keys + TK - 1) / TK);

  if (tid == 0) {
    mbar_init(bar(B_Q), 1);
    for (int s = 0; s < ST; ++s) {
      mbar_init(bar(B_KF + s), 1);
      mbar_init(bar(B_VF + s), 1);
      mbar_init(bar(B_KVE + s), 1);
    }
    for (int t = 0; t < NQT; ++t) {
      mbar_init(bar(B_SF + t), 1);
      mbar_init(bar(B_PF + t), TQ);
      mbar_init(bar(B_OF + t), 1);
    }
    mbar_init(bar(B_DRAIN), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(smem_u32(tmem_slot), kCols);
    tmem_relinquish();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tbase = *tmem_slot;

  if (warp < 4) regs_dec<kRegsLow>();
  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      prefetch_tmap(&tq);
      prefetch_tmap(&tk);
      prefetch_tmap(&tv);
      mbar_expect_tx(bar(B_Q), NQT * kTile);
      for (int t = 0; t < NQT; ++t) tma_load_3d(sQ + t * kTile, &tq, bar(B_Q), 0, h, (int)(m0 + t * TQ));
      int issued = 0;
      for (int j = 0; j < nt; ++j) {
        const int s = j % ST;
        if (j >= ST && !mbar_wait(bar(B_KVE + s), ((j / ST) - 1) & 1, abort_flag, a.err, a.wait_cycles)) break;
        const int kj = (int)(key0 + (long long)j * TK);
        const int c1 = a.kv_head_major ? kj : h;
        const int c2 = a.kv_head_major ? h : kj;
        mbar_expect_tx(bar(B_KF + s), kTile);
        tma_load_3d(sK + s * kTile, &tk, bar(B_KF + s), 0, c1, c2);
        mbar_expect_tx(bar(B_VF + s), kTile);
        tma_load_3d(sV + s * kTile, &tv, bar(B_VF + s), 0, c1, c2);
        issued = j + 1;
      }
      if (*abort_flag) {
        // let this CTA's own copies land before its shared memory goes away
        volatile int never = 0;
        mbar_wait(bar(B_Q), 0, &never, a.err);
        for (int j = issued - 1; j >= 0 && j >= issued - ST; --j) {
          mbar_wait(bar(B_KF + j % ST), (j / ST) & 1, &never, a.err);
          mbar_wait(bar(B_VF + j % ST), (j / ST) & 1, &never, a.err);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t id_qk = idesc(128, 128, kFmtBF16, 0, 0);
      const uint32_t id_pv = idesc(128, 64, kFmtBF16, 0, 1);
      auto issue_s = [&](int t, int s) {
        const uint32_t d = tbase + t * 128;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16_ss(d, sdesc_k(sQ + t * kTile + kk * 32), sdesc_k(sK + s * kTile + kk * 32), id_qk,
                      kk > 0);
        mma_commit(bar(B_SF + t));
      };
      bool ok = mbar_wait(bar(B_Q), 0, abort_flag, a.err, a.wait_cycles) && mbar_wait(bar(B_KF), 0, abort_flag, a.err, a.wait_cycles);
      if (ok) {
        fence_after_sync();
        for (int t = 0; t < NQT; ++t) issue_s(t, 0);
      }
      for (int j = 0; ok && j < nt; ++j) {
        const int s = j % ST;
        ok = mbar_wait(bar(B_VF + s), (j / ST) & 1, abort_flag, a.err, a.wait_cycles);
        for (int t = 0; ok && t < NQT; ++t) {
          ok = mbar_wait(bar(B_PF + t), j & 1, abort_flag, a.err, a.wait_cycles);
          if (!ok) break;
          fence_after_sync();
          const uint32_t d = tbase + 256 + t * 64;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16_ts(d, tbase + t * 128 + kk * 8, sdesc_mn(sV + s * kTile + kk * 2048), id_pv,
                        (j > 0 || kk > 0) ? 1u : 0u);
          if (j + 1 < nt) {
            const int s1 = (j + 1) % ST;
            if (t == 0) {
              ok = mbar_wait(bar(B_KF + s1), ((j + 1) / ST) & 1, abort_flag, a.err, a.wait_cycles);
              if (!ok) break;
              fence_after_sync();
            }
            issue_s(t, s1);
          }
        }
        if (ok) mma_commit(bar(B_KVE + s));
      }
      if (ok) {
        for (int t = 0; t < NQT; ++t) mma_commit(bar(B_OF + t));
      } else {
        // wait for the products already issued before TMEM is released
        volatile int never = 0;
        mma_commit(bar(B_DRAIN));
        mbar_wait(bar(B_DRAIN), 0, &never, a.err);
      }
    }
  } else if (warp >= 4) {
    regs_inc<kRegsHigh>();
    // ---------------- softmax, one thread per row ----------------
    const int t = (warp - 4) >> 2;
    const int q4 = warp & 3;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const uint32_t s_addr = tbase + lane_off + t * 128;
    const uint32_t o_addr = tbase + lane_off + 256 + t * 64;
    const float c2 = a.c2;
    float m_used = -CUDART_INF_F, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nt; ++j) {
      // the whole warp leaves together: tcgen05.ld/st below are warp-collective
      if (!__all_sync(0xffffffffu, mbar_wait(bar(B_SF + t), j & 1, abort_flag, a.err, a.wait_cycles))) {
        ok = false;
        break;
      }
      fence_after_sync();
      uint32_t sv[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(s_addr + 32 * c, sv[c]);
      tmem_wait_ld();
      const long long rem = n_keys - (long long)j * TK;
      if (rem < TK) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (32 * c + i >= rem) sv[c][i] = __float_as_uint(-CUDART_INF_F);
      }
      // eight independent max / sum chains: each softmax warp owns whole rows,
      // so a single 128-long dependency chain would leave it stalled; a
      // three-input maximum takes two columns per instruction
      auto sval = [&](int k) -> float { return __uint_as_float(sv[k >> 5][k & 31]); };
      float mq[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) mq[u] = fmaxf(sval(u), sval(u + 8));
#pragma unroll
      for (int k = 16; k < 128; k += 16)
#pragma unroll
        for (int u = 0; u < 8; ++u) mq[u] = fmax3(mq[u], sval(k + u), sval(k + 8 + u));
      const float mx = fmaxf(fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3])),
                             fmaxf(fmaxf(mq[4], mq[5]), fmaxf(mq[6], mq[7])));
      const float mxs = mx * c2;
      const bool need = mxs > m_used + 8.f;
      // tcgen05.ld/st are warp-collective: the warp rescales together, with
      // factor 1 for the rows that keep their maximum
      if (__any_sync(0xffffffffu, need)) {
        const float corr = need ? exp2f(m_used - mxs) : 1.f;
        if (j > 0) {
          // O_t's previous product is complete: S_t(j) was issued after it
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
      // the scaled, shifted scores two at a time; one pair in four takes its
      // exponentials on the FMA pipe; four paired sum chains
      const uint64_t c2p = f2_pack(c2, c2), nmp = f2_pack(-m_used, -m_used);
      uint64_t ps2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(sv[c][2 * i]), __uint_as_float(sv[c][2 * i + 1])), c2p, nmp);
          uint64_t p2;
          if ((i & 7) >= 8 - kPolyOf8) {
            p2 = exp2_fma2(x2);
          } else {
            float x0, x1;
            f2_unpack(x2, x0, x1);
            p2 = f2_pack(fast_exp2(x0), fast_exp2(x1));
          }
          ps2[i & 3] = f2_add(ps2[i & 3], p2);
          float p0, p1;
          f2_unpack(p2, p0, p1);
          pk[i] = pack_bf16x2(p0, p1);
        }
        tmem_st16(s_addr + 16 * c, pk);
      }
      tmem_wait_st();
      {
        const uint64_t s01 = f2_add(f2_add(ps2[0], ps2[1]), f2_add(ps2[2], ps2[3]));
        float lo, hi;
        f2_unpack(s01, lo, hi);
        l += lo + hi;
      }
      fence_before_sync();
      mbar_arrive(bar(B_PF + t));
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(B_OF + t), 0, abort_flag, a.err, a.wait_cycles));
    if (ok) {
      fence_after_sync();
      const long long row = m0 + t * TQ + q4 * 32 + lane;
      const bool store = row < q_end;
      const float inv = 1.f / l;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t ov[16];
        tmem_ld16(o_addr + 16 * c, ov);
        tmem_wait_ld();
        if (!store) continue;
        const long long ob = row * a.o_row + (long long)h * a.o_head + 16 * c;
        if (a.out_f32) {
          float4* dst = reinterpret_cast<float4*>(static_cast<float*>(a.out) + ob);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            dst[i] = make_float4(__uint_as_float(ov[4 * i]) * inv, __uint_as_float(ov[4 * i + 1]) * inv,
                                 __uint_as_float(ov[4 * i + 2]) * inv, __uint_as_float(ov[4 * i + 3]) * inv);
        } else {
          uint4 u0, u1;
          u0.x = pack_bf16x2(__uint_as_float(ov[0]) * inv, __uint_as_float(ov[1]) * inv);
          u0.y = pack_bf16x2(__uint_as_float(ov[2]) * inv, __uint_as_float(ov[3]) * inv);
          u0.z = pack_bf16x2(__uint_as_float(ov[4]) * inv, __uint_as_float(ov[5]) * inv);
          u0.w = pack_bf16x2(__uint_as_float(ov[6]) * inv, __uint_as_float(ov[7]) * inv);
          u1.x = pack_bf16x2(__uint_as_float(ov[8]) * inv, __uint_as_float(ov[9]) * inv);
          u1.y = pack_bf16x2(__uint_as_float(ov[10]) * inv, __uint_as_float(ov[11]) * inv);
          u1.z = pack_bf16x2(__uint_as_float(ov[12]) * inv, __uint_as_float(ov[13]) * inv);
          u1.w = pack_bf16x2(__uint_as_float(ov[14]) * inv, __uint_as_float(ov[15]) * inv);
          uint4* dst = reinterpret_cast<uint4*>(static_cast<bf16*>(a.out) + ob);
          dst[0] = u0;
          dst[1] = u1;
        }
      }
      if (store && a.lse)
        a.lse[row * a.lse_row + (long long)h * a.lse_head] = (m_used + log2f(l)) * 0.6931471805599453f;
    }
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 2) {
    fence_after_sync();
    tmem_dealloc(tbase, kCols);
  }
}

// ---------------------------------------------------------------------------
// host: tensor maps

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
    cudaGetLastError();
  });
  return fn;
}

}  // namespace

namespace {
__global__ void exp2_selftest_kernel(const float* __restrict__ x, float* __restrict__ y, long long n) {
  const long long i = 2 * ((long long)blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const bool two = i + 1 < n;
  float r0, r1;
  f2_unpack(exp2_fma2(f2_pack(x[i], two ? x[i + 1] : 0.f)), r0, r1);
  y[i] = r0;
  if (two) y[i + 1] = r1;
}
}  // namespace

cudaError_t launch_exp2_selftest(const float* x, float* y, long long n, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  const long long pairs = (n + 1) / 2;
  exp2_selftest_kernel<<<(unsigned)((pairs + 255) / 256), 256, 0, st>>>(x, y, n);
  return cudaGetLastError();
}

// 3-D tiled map over bf16 or fp32 data; dims/strides innermost first, strides in bytes.
bool make_tmap_3d(CUtensorMap* m, bool fp32, const void* base, unsigned long long d0,
                  unsigned long long d1, unsigned long long d2, unsigned long long s1,
                  unsigned long long s2, unsigned b0, unsigned b1, unsigned b2) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {s1, s2};
  cuuint32_t box[3] = {b0, b1, b2};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(m, fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                  const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Tiled map of any rank up to 5 over bf16 data (128-byte swizzle, out-of-range
// elements read as zero); dims/box innermost first, strides (rank - 1 of them) in bytes.
bool make_tmap(CUtensorMap* m, const void* base, int rank, const unsigned long long* dims,
               const unsigned long long* strides, const unsigned* box) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr || rank < 1 || rank > 5) return false;
  cuuint64_t d[5], st[4];
  cuuint32_t b[5], es[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    b[i] = box[i];
    es[i] = 1;
    if (i + 1 < rank) st[i] = strides[i];
  }
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void*>(base), d, st, b,
                  es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

cudaError_t launch_attn_tc(const AttnTcArgs& a, const bf16* q, const bf16* k, const bf16* v,
                           long long kv_rows, cudaStream_t st) {
  if (a.n_q <= 0) return cudaSuccess;
  const unsigned long long H = (unsigned long long)a.H;
  CUtensorMap mq, mk, mv;
  // Q is token-major [n_q][H][64]: dims (64, H, n_q)
  bool ok = make_tmap_3d(&mq, false, q, 64, H, (unsigned long long)a.n_q, 128, H * 128, 64, 1, 128);
  if (a.kv_head_major) {  // [H][kv_rows][64]: dims (64, kv_rows, H)
    ok = ok && make_tmap_3d(&mk, false, k, 64, (unsigned long long)kv_rows, H, 128,
                            (unsigned long long)kv_rows * 128, 64, 128, 1);
    ok = ok && make_tmap_3d(&mv, false, v, 64, (unsigned long long)kv_rows, H, 128,
                            (unsigned long long)kv_rows * 128, 64, 128, 1);
  } else {  // [kv_rows][H][64]: dims (64, H, kv_rows)
    ok = ok && make_tmap_3d(&mk, false, k, 64, H, (unsigned long long)kv_rows, 128, H * 128, 64, 1, 128);
    ok = ok && make_tmap_3d(&mv, false, v, 64, H, (unsigned long long)kv_rows, 128, H * 128, 64, 1, 128);
  }
  if (!ok) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, attn_tc_kernel);
  if (e != cudaSuccess) return e;
  if (fa.numRegs != kLaunchRegs) return cudaErrorInvalidConfiguration;
  AttnTcArgs b = a;
  unsigned gx;
  if (a.seg_len > 0) {
    b.seg_ctas = (a.seg_len + NQT * TQ - 1) / (NQT * TQ);
    gx = (unsigned)(((a.n_q + a.seg_len - 1) / a.seg_len) * b.seg_ctas);
  } else {
    b.seg_ctas = 1;
    gx = (unsigned)((a.n_q + NQT * TQ - 1) / (NQT * TQ));
  }
  dim3 grid(gx, (unsigned)a.H);
  attn_tc_kernel<<<grid, kThreads, kSmemBytes, st>>>(mq, mk, mv, b);
  return cudaGetLastError();
}

}  // namespace gsa
