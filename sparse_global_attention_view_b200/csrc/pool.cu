// Step 1: P x P average pooling of the patch grid of every frame, plus the
// head-major copies of the always-kept tokens' K / V (Speed3R technical
// summary 2.1, compression branch; 2.2, Speed3R-VGGT).
//
// One CTA per patch block (or per special token), H*8 threads, each thread
// owning 8 consecutive channels (16 bytes) of a token's [H][64] row, so every
// token row (H*128 bytes) is read with fully coalesced 16-byte loads.  The
// kernel is HBM-bound: it reads Q, K, V once and writes the pooled tensors.
#include "internal.h"

namespace gsa {
namespace {

__device__ __forceinline__ void add8(float (&acc)[8], const uint4& u) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(h[i]);
    acc[2 * i] += f.x;
    acc[2 * i + 1] += f.y;
  }
}

__device__ __forceinline__ void store8_f32(float* dst, const float (&x)[8]) {
  reinterpret_cast<float4*>(dst)[0] = make_float4(x[0], x[1], x[2], x[3]);
  reinterpret_cast<float4*>(dst)[1] = make_float4(x[4], x[5], x[6], x[7]);
}

__device__ __forceinline__ uint4 pack8_bf16(const float (&x)[8]) {
  uint4 u;
  u.x = pack_bf16x2(x[0], x[1]);
  u.y = pack_bf16x2(x[2], x[3]);
  u.z = pack_bf16x2(x[4], x[5]);
  u.w = pack_bf16x2(x[6], x[7]);
  return u;
}

__device__ __forceinline__ void unpack8(const uint4& u, float (&x)[8]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) x[i] = 0.f;
  add8(x, u);
}

__global__ void pool_kernel(Dims d, const bf16* __restrict__ q, const bf16* __restrict__ k,
                            const bf16* __restrict__ v, float* __restrict__ qc32,
                            float* __restrict__ kc32, bf16* __restrict__ vc, bf16* __restrict__ qc,
                            bf16* __restrict__ kc, bf16* __restrict__ ks, bf16* __restrict__ vs) {
  const int tid = threadIdx.x;                 // channel group: channels [8*tid, 8*tid+8)
  const long long row = (long long)d.H * kHeadDim;  // elements per token
  const long long id = blockIdx.x;
  if (id < d.NB) {
    const long long beta = id;
    float sq[8], sk[8], sv[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) sq[i] = sk[i] = sv[i] = 0.f;
    int cnt = 0;
#pragma unroll 4
    for (int slot = 0; slot < kMaxPool * kMaxPool; ++slot) {
      long long t = block_slot_token(d, beta, slot);
      if (t < 0) continue;
      const long long off = t * row + tid * 8;
      uint4 uq = __ldg(reinterpret_cast<const uint4*>(q + off));
      uint4 uk = __ldg(reinterpret_cast<const uint4*>(k + off));
      uint4 uv = __ldg(reinterpret_cast<const uint4*>(v + off));
      add8(sq, uq);
      add8(sk, uk);
      add8(sv, uv);
      ++cnt;
    }
    // mean = fp32 sum / count (correctly rounded division)
    const float fc = (float)cnt;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      sq[i] = __fdiv_rn(sq[i], fc);
      sk[i] = __fdiv_rn(sk[i], fc);
      sv[i] = __fdiv_rn(sv[i], fc);
    }
    const long long a = entry_of_block(d, beta);
    const long long o = a * row + tid * 8;
    store8_f32(qc32 + o, sq);
    store8_f32(kc32 + o, sk);
    *reinterpret_cast<uint4*>(vc + o) = pack8_bf16(sv);
    if (qc) *reinterpret_cast<uint4*>(qc + o) = pack8_bf16(sq);
    if (kc) *reinterpret_cast<uint4*>(kc + o) = pack8_bf16(sk);
  } else if (id < d.NB + d.NS) {
    const long long s = id - d.NB;  // special index f*S + j
    const long long f = s / d.S;
    const int j = (int)(s - f * d.S);
    const long long t = f * d.L + j;
    const long long a = f * d.E + j;
    const long long off = t * row + tid * 8;
    uint4 uq = __ldg(reinterpret_cast<const uint4*>(q + off));
    uint4 uk = __ldg(reinterpret_cast<const uint4*>(k + off));
    uint4 uv = __ldg(reinterpret_cast<const uint4*>(v + off));
    float fq[8], fk[8];
    unpack8(uq, fq);
    unpack8(uk, fk);
    const long long o = a * row + tid * 8;
    store8_f32(qc32 + o, fq);
    store8_f32(kc32 + o, fk);
    *reinterpret_cast<uint4*>(vc + o) = uv;
    if (qc) *reinterpret_cast<uint4*>(qc + o) = uq;
    if (kc) *reinterpret_cast<uint4*>(kc + o) = uk;
    if (ks && d.keep == GSA_KEEP_SPECIALS) {
      // the specials are the always-kept tokens, in this order
      const int h = tid >> 3, dd = (tid & 7) * 8;
      const long long so = ((long long)h * d.NK + s) * kHeadDim + dd;
      *reinterpret_cast<uint4*>(ks + so) = uk;
      *reinterpret_cast<uint4*>(vs + so) = uv;
    }
  } else {
    // GSA_KEEP_REFERENCE: head-major copy of always-kept token i
    const long long i = id - d.NB - d.NS;
    const long long off = kept_token(d, i) * row + tid * 8;
    const int h = tid >> 3, dd = (tid & 7) * 8;
    const long long so = ((long long)h * d.NK + i) * kHeadDim + dd;
    *reinterpret_cast<uint4*>(ks + so) = __ldg(reinterpret_cast<const uint4*>(k + off));
    *reinterpret_cast<uint4*>(vs + so) = __ldg(reinterpret_cast<const uint4*>(v + off));
  }
}

}  // namespace

cudaError_t launch_pool(const Dims& d, const bf16* q, const bf16* k, const bf16* v, float* qc32,
                        float* kc32, bf16* vc, bf16* qc, bf16* kc, bf16* ks, bf16* vs,
                        cudaStream_t st) {
  // patch blocks, specials, and (reference-frame mode, when copies are wanted)
  // the always-kept tokens
  const long long n = d.NB + d.NS + (ks != nullptr && d.keep == GSA_KEEP_REFERENCE ? d.NK : 0);
  if (n > 0) {
    pool_kernel<<<(unsigned)n, d.H * 8, 0, st>>>(d, q, k, v, qc32, kc32, vc, qc, kc, ks, vs);
  }
  return cudaGetLastError();
}

}  // namespace gsa
