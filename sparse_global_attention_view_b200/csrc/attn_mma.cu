// Flash-style exact attention on the warp-level tensor-core path (mma.sync
// m16n8k16 bf16 -> fp32), for a strided [rows][H][64] layout.
//
// Used for the dense global attention (Speed3R technical summary 1: the
// all-to-all attention GSA replaces) and for the attention inside the pooled
// sequence (technical summary 2.1, compression branch).  One CTA = 4 warps =
// 64 query rows of one head; K/V tiles of 64 keys are double-buffered in
// shared memory with cp.async (16-byte chunks, XOR-swizzled rows so ldmatrix
// is conflict-free).  Scores stay in registers: online softmax in base 2 with
// one rescale of the running output per tile.
#include <math_constants.h>

#include "internal.h"

namespace gsa {
namespace {

constexpr int BM = 64;
constexpr int BN = 64;

template <bool OUT_F32>
__global__ void __launch_bounds__(128) attn_mma_kernel(AttnArgs a) {
  __shared__ __align__(128) uint8_t sQ[BM * 128];
  __shared__ __align__(128) uint8_t sK[2][BN * 128];
  __shared__ __align__(128) uint8_t sV[2][BN * 128];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.y;
  const long long m0 = (long long)blockIdx.x * BM;
  const bf16* qh = a.q + (long long)h * a.q_head;
  const bf16* kh = a.k + (long long)h * a.kv_head;
  const bf16* vh = a.v + (long long)h * a.kv_head;

  for (int i = tid; i < BM * 8; i += 128) {
    const int r = i >> 3, c = i & 7;
    const long long row = m0 + r;
    const bool ok = row < a.n_q;
    cp_async16(smem_u32(sQ) + swz(r, c), qh + (ok ? row : 0) * a.q_row + c * 8, ok);
  }
  auto load_kv = [&](int buf, long long n0) {
    for (int i = tid; i < BN * 8; i += 128) {
      const int r = i >> 3, c = i & 7;
      const long long row = n0 + r;
      const bool ok = row < a.n_k;
      const long long off = (ok ? row : 0) * a.kv_row + c * 8;
      cp_async16(smem_u32(sK[buf]) + swz(r, c), kh + off, ok);
      cp_async16(smem_u32(sV[buf]) + swz(r, c), vh + off, ok);
    }
  };
  const long long n_tiles = (a.n_k + BN - 1) / BN;
  load_kv(0, 0);
  cp_async_commit();

  float o[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m_r[2] = {-CUDART_INF_F, -CUDART_INF_F};
  float l_r[2] = {0.f, 0.f};
  uint32_t qf[4][4];
  const int mi = lane >> 3, r8 = lane & 7;
  const float c2 = a.scale_log2;

  for (long long j = 0; j < n_tiles; ++j) {
    if (j + 1 < n_tiles) load_kv((int)((j + 1) & 1), (j + 1) * BN);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    if (j == 0) {
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        ldsm_x4(smem_u32(sQ) + swz(warp * 16 + r8 + 8 * (mi & 1), ks * 2 + (mi >> 1)), qf[ks][0],
                qf[ks][1], qf[ks][2], qf[ks][3]);
    }
    const int buf = (int)(j & 1);
    const uint32_t kb = smem_u32(sK[buf]), vb = smem_u32(sV[buf]);

    float s[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(kb + swz(np * 16 + r8 + 8 * (mi >> 1), ks * 2 + (mi & 1)), b0, b1, b2, b3);
        mma16816(s[2 * np], qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3], b0, b1);
        mma16816(s[2 * np + 1], qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3], b2, b3);
      }
    }
    if ((j + 1) * BN > a.n_k) {
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (j * BN + nt * 8 + 2 * (lane & 3) + (e & 1) >= a.n_k) s[nt][e] = -CUDART_INF_F;
    }
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      float mx = m_r[hf];
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) mx = fmaxf(mx, fmaxf(s[nt][2 * hf], s[nt][2 * hf + 1]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float corr = exp2f((m_r[hf] - mx) * c2);
      m_r[hf] = mx;
      const float ms = mx * c2;
      float sum = 0.f;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const float p0 = exp2f(fmaf(s[nt][2 * hf], c2, -ms));
        const float p1 = exp2f(fmaf(s[nt][2 * hf + 1], c2, -ms));
        s[nt][2 * hf] = p0;
        s[nt][2 * hf + 1] = p1;
        sum += p0 + p1;
      }
      l_r[hf] = l_r[hf] * corr + sum;
#pragma unroll
      for (int dt = 0; dt < 8; ++dt) {
        o[dt][2 * hf] *= corr;
        o[dt][2 * hf + 1] *= corr;
      }
    }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const uint32_t a0 = pack_bf16x2(s[2 * kk][0], s[2 * kk][1]);
      const uint32_t a1 = pack_bf16x2(s[2 * kk][2], s[2 * kk][3]);
      const uint32_t a2 = pack_bf16x2(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      const uint32_t a3 = pack_bf16x2(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
      for (int dp = 0; dp < 4; ++dp) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(vb + swz(kk * 16 + r8 + 8 * (mi & 1), dp * 2 + (mi >> 1)), b0, b1, b2, b3);
        mma16816(o[2 * dp], a0, a1, a2, a3, b0, b1);
        mma16816(o[2 * dp + 1], a0, a1, a2, a3, b2, b3);
      }
    }
    __syncthreads();
  }

#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    float l = l_r[hf];
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    const float inv = 1.f / l;
    const long long row = m0 + warp * 16 + (lane >> 2) + 8 * hf;
    if (row < a.n_q) {
      const long long base = row * a.o_row + (long long)h * a.o_head + 2 * (lane & 3);
#pragma unroll
      for (int dt = 0; dt < 8; ++dt) {
        const float x0 = o[dt][2 * hf] * inv, x1 = o[dt][2 * hf + 1] * inv;
        if (OUT_F32) {
          *reinterpret_cast<float2*>(static_cast<float*>(a.o) + base + dt * 8) = make_float2(x0, x1);
        } else {
          *reinterpret_cast<uint32_t*>(static_cast<bf16*>(a.o) + base + dt * 8) = pack_bf16x2(x0, x1);
        }
      }
      if (a.lse && (lane & 3) == 0)
        a.lse[row * a.lse_row + (long long)h * a.lse_head] = m_r[hf] * a.scale + logf(l);
    }
  }
}

}  // namespace

cudaError_t launch_attn_mma(const AttnArgs& a, cudaStream_t st) {
  if (a.n_q <= 0) return cudaSuccess;
  dim3 grid((unsigned)((a.n_q + BM - 1) / BM), (unsigned)a.H);
  if (a.o_f32)
    attn_mma_kernel<true><<<grid, 128, 0, st>>>(a);
  else
    attn_mma_kernel<false><<<grid, 128, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace gsa
