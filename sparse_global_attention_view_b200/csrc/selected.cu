// Step 5 (and, fused, step 6): the selection branch (Speed3R technical summary
// 2.1; the always-kept special tokens of 2.2, Speed3R-VGGT).
//
// One warp per (compressed entry a, head h): the entry's <=16 fine tokens are
// the 16 rows of one m16n8k16 tile.  Each warp runs a single online softmax
// over two key segments:
//   1. the NK always-kept tokens (all N*S specials, or frame 0 plus every
//      camera token), in 64-key tiles shared by the CTA's 4 warps (cp.async
//      double buffer from the head-major copy ks/vs);
//   2. the entry's selected blocks, one 16-slot block per step, gathered by
//      the warp itself (16 token rows of 128 bytes straight from K/V, a
//      3-stage cp.async pipeline per warp; patches outside the grid are
//      zero-filled and masked to -inf).
// When the specials segment was already computed elsewhere (o_spec, lse_spec:
// its normalised output and log-sum-exp per token and head), the warp starts
// its online softmax from that state instead of running segment 1: running
// maximum lse/scale, row sum 1, output o_spec.
// The epilogue normalises and either writes o_sel (+lse) or applies the gate
// g = sigmoid(qc32[a,h] . w[h]) and writes g*oc + (1-g)*o_sel.
#include <math_constants.h>
#include <stddef.h>

#include "internal.h"

namespace gsa {
namespace {

constexpr int SW = 4;       // warps (entries) per CTA
constexpr int SBN = 64;     // special keys per shared tile
constexpr int SSTAGE = 3;   // per-warp block pipeline depth

// Shared memory of one CTA.  The special-token tiles are only used when the
// kernel runs that segment itself; without them three CTAs fit on an SM.
struct SelSmem {
  uint8_t q[SW][16 * 128];
  uint8_t kb[SW][SSTAGE][16 * 128];
  uint8_t vb[SW][SSTAGE][16 * 128];
  int sel[SW][kMaxTopK];
  uint8_t ks[2][SBN * 128];
  uint8_t vs[2][SBN * 128];
};
constexpr size_t kSmemNoSpecials = offsetof(SelSmem, ks);

// A patch block's first token (top-left patch) and how many of its P rows and
// P columns lie inside the grid.
struct BlockGeo {
  long long base;
  int nr, nc;
};
__device__ __forceinline__ BlockGeo block_geo(const Dims& d, long long beta) {
  const long long f = beta / d.Bf;
  const int j = (int)(beta - f * d.Bf);
  const int br = j / d.Bw, bc = j - br * d.Bw;
  BlockGeo g;
  g.base = f * d.L + d.S + (long long)(br * d.P) * d.Wp + bc * d.P;
  g.nr = min(d.P, d.Hp - br * d.P);
  g.nc = min(d.P, d.Wp - bc * d.P);
  return g;
}

// One key tile of NT*8 keys: S = Q K^T, mask, online softmax, O += P V.
template <int NT, typename Masked>
__device__ __forceinline__ void tile_step(uint32_t kb, uint32_t vb, const uint32_t (&qf)[4][4],
                                          float (&o)[8][4], float (&m_r)[2], float (&l_r)[2],
                                          float c2, int lane, Masked masked) {
  const int mi = lane >> 3, r8 = lane & 7;
  float s[NT][4];
#pragma unroll
  for (int i = 0; i < NT; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
  for (int ks = 0; ks < 4; ++ks) {
#pragma unroll
    for (int np = 0; np < NT / 2; ++np) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4(kb + swz(np * 16 + r8 + 8 * (mi >> 1), ks * 2 + (mi & 1)), b0, b1, b2, b3);
      mma16816(s[2 * np], qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3], b0, b1);
      mma16816(s[2 * np + 1], qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3], b2, b3);
    }
  }
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e)
      if (masked(nt * 2 + (e & 1), nt * 8 + 2 * (lane & 3) + (e & 1))) s[nt][e] = -CUDART_INF_F;
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    float mx = m_r[hf];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) mx = fmaxf(mx, fmaxf(s[nt][2 * hf], s[nt][2 * hf + 1]));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float corr = exp2f((m_r[hf] - mx) * c2);
    m_r[hf] = mx;
    const float ms = mx * c2;
    float sum = 0.f;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
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
  for (int kk = 0; kk < NT / 2; ++kk) {
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
}

__global__ void __launch_bounds__(SW * 32)
    selected_kernel(Dims d, const bf16* __restrict__ q, const bf16* __restrict__ k,
                    const bf16* __restrict__ v, const bf16* __restrict__ ks,
                    const bf16* __restrict__ vs, const int* __restrict__ sel,
                    const float* __restrict__ qc32, const float* __restrict__ w,
                    const float* __restrict__ oc, bf16* __restrict__ out, float* __restrict__ lse,
                    const float* __restrict__ o_spec, const float* __restrict__ lse_spec,
                    unsigned* __restrict__ err) {
  extern __shared__ __align__(128) unsigned char sel_smem_raw[];
  SelSmem& sm = *reinterpret_cast<SelSmem*>(sel_smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.y;
  const long long a = (long long)blockIdx.x * SW + warp;
  const bool live = a < d.Tc;
  const long long row = (long long)d.H * kHeadDim;
  const float c2 = d.scale_log2;

  // this warp's query rows (slot r = row r) and selection list
  for (int i = lane; i < 16 * 8; i += 32) {
    const int slot = i >> 3, c = i & 7;
    const long long t = live ? entry_slot_token(d, a, slot) : -1;
    cp_async16(smem_u32(sm.q[warp]) + swz(slot, c), q + (t >= 0 ? t : 0) * row + h * kHeadDim + c * 8,
               t >= 0);
  }
  for (int i = lane; i < d.K; i += 32) sm.sel[warp][i] = live ? sel[((long long)h * d.Tc + a) * d.K + i] : -1;

  float o[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m_r[2] = {-CUDART_INF_F, -CUDART_INF_F};
  float l_r[2] = {0.f, 0.f};
  uint32_t qf[4][4];
  const int mi = lane >> 3, r8 = lane & 7;
  auto load_qf = [&]() {
#pragma unroll
    for (int kq = 0; kq < 4; ++kq)
      ldsm_x4(smem_u32(sm.q[warp]) + swz(r8 + 8 * (mi & 1), kq * 2 + (mi >> 1)), qf[kq][0], qf[kq][1],
              qf[kq][2], qf[kq][3]);
  };

  // ---- segment 1: the special tokens ----
  const long long NS = d.NK;  // the always-kept tokens
  if (o_spec != nullptr) {
    // state of a softmax over the specials alone, computed by another kernel
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const long long t = live ? entry_slot_token(d, a, (lane >> 2) + 8 * hf) : -1;
      if (t < 0) continue;
      const long long th = t * d.H + h;
      m_r[hf] = lse_spec[th] / d.scale;
      l_r[hf] = (lane & 3) == 0 ? 1.f : 0.f;
      const float* os = o_spec + th * kHeadDim + 2 * (lane & 3);
#pragma unroll
      for (int dt = 0; dt < 8; ++dt) {
        const float2 x = *reinterpret_cast<const float2*>(os + dt * 8);
        o[dt][2 * hf] = x.x;
        o[dt][2 * hf + 1] = x.y;
      }
    }
    cp_async_wait<0>();
    __syncthreads();
    load_qf();
  } else {
    auto load_sp = [&](int buf, long long n0) {
      for (int i = tid; i < SBN * 8; i += SW * 32) {
        const int r = i >> 3, c = i & 7;
        const long long idx = n0 + r;
        const bool ok = idx < NS;
        const long long off = ((long long)h * NS + (ok ? idx : 0)) * kHeadDim + c * 8;
        cp_async16(smem_u32(sm.ks[buf]) + swz(r, c), ks + off, ok);
        cp_async16(smem_u32(sm.vs[buf]) + swz(r, c), vs + off, ok);
      }
    };
    const long long n_sp = (NS + SBN - 1) / SBN;
    if (n_sp > 0) load_sp(0, 0);
    cp_async_commit();
    for (long long j = 0; j < n_sp; ++j) {
      if (j + 1 < n_sp) load_sp((int)((j + 1) & 1), (j + 1) * SBN);
      cp_async_commit();
      cp_async_wait<1>();
      __syncthreads();
      if (j == 0) load_qf();
      const long long base = j * SBN;
      tile_step<8>(smem_u32(sm.ks[j & 1]), smem_u32(sm.vs[j & 1]), qf, o, m_r, l_r, c2, lane,
                   [&](int, int key) { return base + key >= NS; });
      __syncthreads();
    }
    if (n_sp == 0) {
      cp_async_wait<0>();
      __syncthreads();
      load_qf();
    }
  }

  // ---- segment 2: the selected blocks (per warp) ----
  // ids come from the caller's buffer: a value outside [0, NB) ends the list
  // and raises the device-check bit instead of being dereferenced
  int nsel = 0;
  while (nsel < d.K && sm.sel[warp][nsel] >= 0) {
    if (sm.sel[warp][nsel] >= d.NB) {
      if (lane == 0) atomicOr(err, kErrDeviceCheck);
      break;
    }
    ++nsel;
  }
  // Slots this lane touches: in the gather (slot (lane >> 3) + 4 it) and in
  // the score fragment (keys 2 (lane & 3) + {0, 1} + {0, 8}).  Their (row,
  // column) inside a block depend only on P, so they are computed once.
  int ldr[4], ldc[4], mdr[4], mdc[4];
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    const int sl = (lane >> 3) + 4 * it;
    ldr[it] = sl < d.P * d.P ? sl / d.P : kMaxPool;
    ldc[it] = sl % d.P;
    const int km = (it >> 1) * 8 + 2 * (lane & 3) + (it & 1);
    mdr[it] = km < d.P * d.P ? km / d.P : kMaxPool;
    mdc[it] = km % d.P;
  }
  auto load_blk = [&](int stage, long long beta) {
    const BlockGeo g = block_geo(d, beta);
    const int c = lane & 7;
#pragma unroll
    for (int it = 0; it < 4; ++it) {
      const int sl = (lane >> 3) + 4 * it;
      const bool ok = ldr[it] < g.nr && ldc[it] < g.nc;
      const long long t = ok ? g.base + (long long)ldr[it] * d.Wp + ldc[it] : 0;
      const long long off = t * row + h * kHeadDim + c * 8;
      cp_async16(smem_u32(sm.kb[warp][stage]) + swz(sl, c), k + off, ok);
      cp_async16(smem_u32(sm.vb[warp][stage]) + swz(sl, c), v + off, ok);
    }
  };
#pragma unroll
  for (int s = 0; s < SSTAGE - 1; ++s) {
    if (s < nsel) load_blk(s, sm.sel[warp][s]);
    cp_async_commit();
  }
  for (int i = 0; i < nsel; ++i) {
    if (i + SSTAGE - 1 < nsel) load_blk((i + SSTAGE - 1) % SSTAGE, sm.sel[warp][i + SSTAGE - 1]);
    cp_async_commit();
    cp_async_wait<SSTAGE - 1>();
    __syncwarp();
    const BlockGeo g = block_geo(d, sm.sel[warp][i]);
    const int st = i % SSTAGE;
    tile_step<2>(smem_u32(sm.kb[warp][st]), smem_u32(sm.vb[warp][st]), qf, o, m_r, l_r, c2, lane,
                 [&](int m, int) { return !(mdr[m] < g.nr && mdc[m] < g.nc); });
    __syncwarp();
  }
  if (!live) return;

  // ---- epilogue ----
  float g = 0.f;
  if (w) {
    const float* qa = qc32 + (a * d.H + h) * kHeadDim;
    const float* wh = w + (long long)h * kHeadDim;
    float z = qa[lane] * wh[lane] + qa[lane + 32] * wh[lane + 32];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
    g = 1.f / (1.f + expf(-z));
  }
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    float l = l_r[hf];
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    const float inv = 1.f / l;
    const int slot = (lane >> 2) + 8 * hf;
    const long long t = entry_slot_token(d, a, slot);
    if (t < 0) continue;
    const long long ob = t * row + h * kHeadDim + 2 * (lane & 3);
    if (w) {
      const float* oca = oc + (a * d.H + h) * kHeadDim + 2 * (lane & 3);
#pragma unroll
      for (int dt = 0; dt < 8; ++dt) {
        const float2 cm = *reinterpret_cast<const float2*>(oca + dt * 8);
        const float x0 = g * cm.x + (1.f - g) * (o[dt][2 * hf] * inv);
        const float x1 = g * cm.y + (1.f - g) * (o[dt][2 * hf + 1] * inv);
        *reinterpret_cast<uint32_t*>(out + ob + dt * 8) = pack_bf16x2(x0, x1);
      }
    } else {
#pragma unroll
      for (int dt = 0; dt < 8; ++dt)
        *reinterpret_cast<uint32_t*>(out + ob + dt * 8) =
            pack_bf16x2(o[dt][2 * hf] * inv, o[dt][2 * hf + 1] * inv);
      if (lse && (lane & 3) == 0) lse[t * d.H + h] = m_r[hf] * d.scale + logf(l);
    }
  }
}

}  // namespace

cudaError_t launch_selected(const Dims& d, const bf16* q, const bf16* k, const bf16* v,
                            const bf16* ks, const bf16* vs, const int* sel, const float* qc32,
                            const float* w, const float* oc, bf16* out, float* lse,
                            const float* o_spec, const float* lse_spec, unsigned* err,
                            cudaStream_t st) {
  const bool own_specials = d.NK > 0 && o_spec == nullptr;
  const size_t smem = own_specials ? sizeof(SelSmem) : kSmemNoSpecials;
  cudaError_t e = cudaFuncSetAttribute(selected_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)sizeof(SelSmem));
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((d.Tc + SW - 1) / SW), (unsigned)d.H);
  selected_kernel<<<grid, SW * 32, smem, st>>>(d, q, k, v, ks, vs, sel, qc32, w, oc, out, lse, o_spec,
                                                lse_spec, err);
  return cudaGetLastError();
}

}  // namespace gsa
