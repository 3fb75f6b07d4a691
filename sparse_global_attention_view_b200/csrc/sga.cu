// Subsampled global attention ("AVGGT: Rethinking Global Attention for
// Accelerating VGGT", section 2.2, SGA): every query attends to the special
// tokens and to the patch tokens sampled at the top-left of every
// sub_h x sub_w window of every frame, to its own key/value when that one was
// not sampled (the diagonal), and to one extra pair holding the means of all
// dropped keys and values.
//
// Four kernels around the tcgen05 attention kernel:
//   sga_gather      head-major copies Ks/Vs [H][NK][64] of the kept keys;
//   sga_frame_sums  per frame, fp32 sums of the dropped patch tokens' K and V
//                   (one CTA per frame, HBM-bound single pass over K and V);
//   sga_means       the frame sums added in frame order (deterministic) and
//                   divided by the number of dropped tokens;
//   (attention of every query over Ks/Vs: normalised fp32 output and lse)
//   sga_combine     the own-key and mean-pair logits merged into that softmax
//                   by their log-sum-exp, written as bf16.
// Each thread of the gather / sums / combine kernels owns 8 consecutive
// channels (16 bytes) of a token's [H][64] row, so rows are read with
// coalesced 16-byte loads.
#include <math_constants.h>

#include "internal.h"

namespace gsa {
namespace {

struct SgaGeo {
  int sub_h, sub_w, nh, nw;  // window, sampled rows / columns per frame
  long long per;             // kept keys per frame: S + nh * nw
};

__device__ __forceinline__ long long kept_key_token(const Dims& d, const SgaGeo& g, long long i) {
  const long long f = i / g.per;
  const int j = (int)(i - f * g.per);
  if (j < d.S) return f * d.L + j;
  const int p = j - d.S;
  const int r = (p / g.nw) * g.sub_h, c = (p % g.nw) * g.sub_w;
  return f * d.L + d.S + (long long)r * d.Wp + c;
}

__device__ __forceinline__ bool token_is_kept(const Dims& d, const SgaGeo& g, long long t) {
  const int i = (int)(t % d.L);
  if (i < d.S) return true;
  const int p = i - d.S;
  return (p / d.Wp) % g.sub_h == 0 && (p % d.Wp) % g.sub_w == 0;
}

__device__ __forceinline__ void acc8(float (&a)[8], const uint4& u) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    a[2 * i] += f.x;
    a[2 * i + 1] += f.y;
  }
}

__global__ void sga_gather_kernel(Dims d, SgaGeo g, const bf16* __restrict__ k,
                                  const bf16* __restrict__ v, bf16* __restrict__ ks,
                                  bf16* __restrict__ vs, long long nk) {
  const int tid = threadIdx.x;
  const long long i = blockIdx.x;
  const long long off = kept_key_token(d, g, i) * d.H * kHeadDim + tid * 8;
  const int h = tid >> 3, dd = (tid & 7) * 8;
  const long long so = ((long long)h * nk + i) * kHeadDim + dd;
  *reinterpret_cast<uint4*>(ks + so) = __ldg(reinterpret_cast<const uint4*>(k + off));
  *reinterpret_cast<uint4*>(vs + so) = __ldg(reinterpret_cast<const uint4*>(v + off));
}

// part[f][0 or 1][H*64]: sums of K (0) and V (1) over frame f's dropped patches
__global__ void sga_frame_sums_kernel(Dims d, SgaGeo g, const bf16* __restrict__ k,
                                      const bf16* __restrict__ v, float* __restrict__ part) {
  const int tid = threadIdx.x;
  const long long f = blockIdx.x;
  const long long row = (long long)d.H * kHeadDim;
  float sk[8], sv[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) sk[i] = sv[i] = 0.f;
  for (int r = 0; r < d.Hp; ++r) {
    if (r % g.sub_h == 0) {
      // a sampled row: every column but the sampled ones
      for (int c = 0; c < d.Wp; ++c) {
        if (c % g.sub_w == 0) continue;
        const long long off = (f * d.L + d.S + (long long)r * d.Wp + c) * row + tid * 8;
        acc8(sk, __ldg(reinterpret_cast<const uint4*>(k + off)));
        acc8(sv, __ldg(reinterpret_cast<const uint4*>(v + off)));
      }
    } else {
#pragma unroll 4
      for (int c = 0; c < d.Wp; ++c) {
        const long long off = (f * d.L + d.S + (long long)r * d.Wp + c) * row + tid * 8;
        acc8(sk, __ldg(reinterpret_cast<const uint4*>(k + off)));
        acc8(sv, __ldg(reinterpret_cast<const uint4*>(v + off)));
      }
    }
  }
  float* pk = part + (f * 2) * row + tid * 8;
  float* pv = pk + row;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    pk[i] = sk[i];
    pv[i] = sv[i];
  }
}

// mean[0 or 1][H*64] = (sum over frames of part) / n_dropped, frames in order
__global__ void sga_means_kernel(int n_frames, long long row, long long n_dropped,
                                 const float* __restrict__ part, float* __restrict__ mean) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;  // over 2*row
  if (i >= 2 * row) return;
  float s = 0.f;
  for (int f = 0; f < n_frames; ++f) s += part[(long long)f * 2 * row + i];
  mean[i] = n_dropped > 0 ? s / (float)n_dropped : 0.f;
}

__device__ __forceinline__ void load8f(float (&x)[8], const bf16* p) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
#pragma unroll
  for (int i = 0; i < 8; ++i) x[i] = 0.f;
  acc8(x, u);
}

// out[t,h] from the softmax over the kept keys (o_kept normalised, lse natural
// log) and two more logits: the own key (when not kept) and the mean key.
__global__ void sga_combine_kernel(Dims d, SgaGeo g, long long n_dropped, const bf16* __restrict__ q,
                                   const bf16* __restrict__ k, const bf16* __restrict__ v,
                                   const float* __restrict__ mean, const float* __restrict__ o_kept,
                                   const float* __restrict__ lse, bf16* __restrict__ out) {
  const int tid = threadIdx.x, h = tid >> 3;
  const long long t = blockIdx.x;
  const long long row = (long long)d.H * kHeadDim;
  const long long off = t * row + tid * 8;
  float qv[8], kv[8], vv[8];
  load8f(qv, q + off);
  load8f(kv, k + off);
  load8f(vv, v + off);
  const float* km = mean + tid * 8;
  const float* vm = mean + row + tid * 8;
  float s_own = 0.f, s_mean = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    s_own = fmaf(qv[i], kv[i], s_own);
    s_mean = fmaf(qv[i], km[i], s_mean);
  }
  // the 8 threads of one head are 8 consecutive lanes; a block of H*8 threads
  // may end in a partial warp, so the mask names only the lanes that exist
  const int in_warp = min(32, (int)blockDim.x - (tid & ~31));
  const unsigned lanes = in_warp == 32 ? 0xffffffffu : ((1u << in_warp) - 1u);
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) {
    s_own += __shfl_xor_sync(lanes, s_own, o);
    s_mean += __shfl_xor_sync(lanes, s_mean, o);
  }
  s_own = token_is_kept(d, g, t) ? -CUDART_INF_F : s_own * d.scale;
  s_mean = n_dropped > 0 ? s_mean * d.scale : -CUDART_INF_F;
  const float l0 = lse[t * d.H + h];
  const float m = fmaxf(l0, fmaxf(s_own, s_mean));
  const float w0 = __expf(l0 - m), w1 = __expf(s_own - m), w2 = __expf(s_mean - m);
  const float inv = 1.f / (w0 + w1 + w2);
  const float* ok = o_kept + off;
  float r[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) r[i] = (w0 * ok[i] + w1 * vv[i] + w2 * vm[i]) * inv;
  uint4 u;
  u.x = pack_bf16x2(r[0], r[1]);
  u.y = pack_bf16x2(r[2], r[3]);
  u.z = pack_bf16x2(r[4], r[5]);
  u.w = pack_bf16x2(r[6], r[7]);
  *reinterpret_cast<uint4*>(out + off) = u;
}

}  // namespace

SgaSizes sga_sizes(const Dims& d, int sub_h, int sub_w) {
  SgaSizes z;
  z.nh = (d.Hp + sub_h - 1) / sub_h;
  z.nw = (d.Wp + sub_w - 1) / sub_w;
  z.NK = (long long)d.N * (d.S + (long long)z.nh * z.nw);
  z.n_dropped = (long long)d.N * ((long long)d.Hp * d.Wp - (long long)z.nh * z.nw);
  return z;
}

cudaError_t launch_sga(const Dims& d, int sub_h, int sub_w, const bf16* q, const bf16* k,
                       const bf16* v, bf16* out, bf16* ks, bf16* vs, float* part, float* mean,
                       float* o_kept, float* lse, unsigned* err, cudaStream_t st, int* launched) {
  const SgaSizes z = sga_sizes(d, sub_h, sub_w);
  SgaGeo g;
  g.sub_h = sub_h;
  g.sub_w = sub_w;
  g.nh = z.nh;
  g.nw = z.nw;
  g.per = d.S + (long long)z.nh * z.nw;
  const int threads = d.H * 8;
  const long long row = (long long)d.H * kHeadDim;
  *launched = 0;
  sga_gather_kernel<<<(unsigned)z.NK, threads, 0, st>>>(d, g, k, v, ks, vs, z.NK);
  ++*launched;
  sga_frame_sums_kernel<<<(unsigned)d.N, threads, 0, st>>>(d, g, k, v, part);
  ++*launched;
  sga_means_kernel<<<(unsigned)((2 * row + 255) / 256), 256, 0, st>>>(d.N, row, z.n_dropped, part,
                                                                    mean);
  ++*launched;
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  AttnTcArgs a;
  a.n_q = d.T;
  a.n_k = z.NK;
  a.H = d.H;
  a.c2 = d.scale_log2;
  a.out = o_kept;
  a.out_f32 = 1;
  a.o_row = row;
  a.o_head = kHeadDim;
  a.lse = lse;
  a.lse_row = d.H;
  a.lse_head = 1;
  a.err = err;
  a.kv_head_major = 1;
  a.seg_len = 0;
  a.wait_cycles = d.wait_cycles;
  e = launch_attn_tc(a, q, ks, vs, z.NK, st);
  if (e != cudaSuccess) return e;
  ++*launched;
  sga_combine_kernel<<<(unsigned)d.T, threads, 0, st>>>(d, g, z.n_dropped, q, k, v, mean, o_kept,
                                                         lse, out);
  ++*launched;
  return cudaGetLastError();
}

}  // namespace gsa
