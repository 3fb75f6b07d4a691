// Shared device helpers for libgsa (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gsa.h"

namespace gsa {

// Derived sizes, passed to kernels by value.
struct Dims {
  int N, S, Hp, Wp, H, P, K, Keff;
  int L, E, Bh, Bw, Bf;
  int keep;          // GSA_KEEP_SPECIALS or GSA_KEEP_REFERENCE
  long long T, Tc, NB, NS;
  long long NK;      // always-kept tokens of the selection branch
  long long B0;      // first top-K candidate block (Bf when frame 0 is kept whole)
  float scale;       // softmax scale
  float scale_log2;  // scale * log2(e)
  long long wait_cycles;  // limit of the in-kernel waits of one role on another
  // floor((2^32 - 1) / x) for x = E, Bf, Bw, Tc: quotients by these on the
  // integer pipe (udiv31)
  uint32_t mE, mBf, mBw, mTc;
};

// floor(n / x) for 0 <= n < 2^31 and 1 <= x < 2^31, from m = floor((2^32 - 1) / x):
// hi32(n m) is the quotient or one less (n m / 2^32 > n / x - 2n / 2^32 > n / x - 1),
// so one correction step is exact.  Avoids the float reciprocal of a general
// integer division, whose conversions share a pipe with the exponentials.
__device__ __forceinline__ int udiv31(int n, int x, uint32_t m) {
  int q = (int)__umulhi((uint32_t)n, m);
  if (n - q * x >= x) ++q;
  return q;
}

// Bits of the device error word (first word of every workspace).
enum : unsigned { kErrTimeout = 1u, kErrDeviceCheck = 2u };

constexpr int kHeadDim = 64;
constexpr int kMaxPool = 4;   // P*P <= 16 token slots per block
constexpr int kMaxTopK = 128;

typedef __nv_bfloat16 bf16;

// ---------------------------------------------------------------------------
// token geometry (same conventions as include/gsa.h)

// Compressed entry of fine token t.
__device__ __forceinline__ long long entry_of_token(const Dims& d, long long t) {
  long long f = t / d.L;
  int i = (int)(t - f * d.L);
  if (i < d.S) return f * d.E + i;
  int p = i - d.S;
  int r = p / d.Wp, c = p - (p / d.Wp) * d.Wp;
  return f * d.E + d.S + (r / d.P) * d.Bw + c / d.P;
}

// Compressed entry of patch block beta.
__device__ __forceinline__ long long entry_of_block(const Dims& d, long long beta) {
  long long f = beta / d.Bf;
  return f * d.E + d.S + (beta - f * d.Bf);
}

// Token id held in slot `slot` (0 <= slot < P*P, row-major in the block) of
// patch block `beta`, or -1 when that patch lies outside the grid.
__device__ __forceinline__ long long block_slot_token(const Dims& d, long long beta, int slot) {
  if (slot >= d.P * d.P) return -1;
  long long f = beta / d.Bf;
  int j = (int)(beta - f * d.Bf);
  int br = j / d.Bw, bc = j - (j / d.Bw) * d.Bw;
  int r = br * d.P + slot / d.P, c = bc * d.P + slot % d.P;
  if (r >= d.Hp || c >= d.Wp) return -1;
  return f * d.L + d.S + (long long)r * d.Wp + c;
}

// Token id of always-kept token i (0 <= i < NK): special i (frame-major) for
// GSA_KEEP_SPECIALS; frame 0's token i, then frame (i - L + 1)'s camera token
// (special slot 0) for GSA_KEEP_REFERENCE.
__host__ __device__ __forceinline__ long long kept_token(const Dims& d, long long i) {
  if (d.keep == GSA_KEEP_SPECIALS) {
    const long long f = i / d.S;
    return f * d.L + (i - f * d.S);
  }
  return i < d.L ? i : (i - d.L + 1) * d.L;
}

// Token id held in slot `slot` of compressed entry a (a special entry holds its
// token in slot 0), or -1.
__device__ __forceinline__ long long entry_slot_token(const Dims& d, long long a, int slot) {
  long long f = a / d.E;
  int j = (int)(a - f * d.E);
  if (j < d.S) return slot == 0 ? f * d.L + j : -1;
  return block_slot_token(d, f * d.Bf + (j - d.S), slot);
}

// ---------------------------------------------------------------------------
// PTX wrappers: cp.async, ldmatrix, mma.sync (bf16, fp32 accumulate)

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

// 16-byte async copy global -> shared; zero-fills when !valid (no bytes read).
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(n)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D += A * B, m16n8k16, A row-major bf16, B column-major bf16, fp32 accumulate.
__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Byte offset of 16-byte chunk `chunk` (0..7) of row `row` in a [rows][64] bf16
// tile whose chunks are XOR-swizzled by (row & 7): ldmatrix over 8 rows hits 8
// distinct bank groups.
__device__ __forceinline__ uint32_t swz(int row, int chunk) {
  return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4));
}

}  // namespace gsa
