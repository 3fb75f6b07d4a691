// Steps 3-4 of the stage calls: S_guide block scores with a streaming Top-K,
// and the merge of the per-slice candidate lists into the selection (Speed3R
// technical summary 2.1, selection branch; S_guide on the it page, section 2);
// and the union of the two ranking passes gsa_forward runs for 64 < K <= 128.
//
// Block scores are fp32 dot products of the fp32 pooled query and key means,
// times the softmax scale.  Each thread owns one compressed query row and
// streams the patch blocks of its slice in ascending id order, keeping its K
// best (score, id) pairs in shared memory with the current K-th best as the
// admission threshold: a candidate enters only if it beats the threshold
// strictly, so among equal scores the earlier (lower) id stays, and the
// evicted pair is the worst by (score ascending, id descending).  The full
// score matrix is never written to memory.
#include <math_constants.h>

#include "internal.h"

namespace gsa {
namespace {

constexpr int TK_ROWS = 128;  // threads per CTA = query rows per CTA
constexpr int TK_TILE = 32;   // patch blocks per shared-memory key tile

__global__ void __launch_bounds__(TK_ROWS)
    block_scores_topk_kernel(Dims d, const float* __restrict__ qc32, const float* __restrict__ kc32,
                             float* __restrict__ cand_s, int* __restrict__ cand_i, int n_split) {
  extern __shared__ __align__(16) float tk_smem[];
  float* sk = tk_smem;                        // [2][TK_TILE][64]
  float* ls = tk_smem + 2 * TK_TILE * 64;     // [K][TK_ROWS]
  int* li = reinterpret_cast<int*>(ls + d.K * TK_ROWS);

  const int tid = threadIdx.x;
  const int h = blockIdx.y, sp = blockIdx.z;
  const long long a = (long long)blockIdx.x * TK_ROWS + tid;
  const bool active = a < d.Tc;
  const long long row = (long long)d.H * kHeadDim;
  // candidate blocks [B0, NB), cut into n_split slices
  const long long per = (d.NB - d.B0 + n_split - 1) / n_split;
  const long long b0 = d.B0 + (long long)sp * per;
  const long long b1 = b0 + per < d.NB ? b0 + per : d.NB;

  float q[64];
  if (active) {
    const float4* qp = reinterpret_cast<const float4*>(qc32 + a * row + h * kHeadDim);
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      float4 x = qp[c];
      q[4 * c] = x.x, q[4 * c + 1] = x.y, q[4 * c + 2] = x.z, q[4 * c + 3] = x.w;
    }
  } else {
#pragma unroll
    for (int c = 0; c < 64; ++c) q[c] = 0.f;
  }

  auto load_tile = [&](int buf, long long t0) {
    for (int i = tid; i < TK_TILE * 16; i += TK_ROWS) {
      const int r = i >> 4, c = i & 15;
      const long long beta = t0 + r;
      const bool ok = beta < b1;
      const long long e = ok ? entry_of_block(d, beta) : 0;
      cp_async16(smem_u32(sk + (buf * TK_TILE + r) * 64 + c * 4), kc32 + e * row + h * kHeadDim + c * 4,
                 ok);
    }
  };

  int cnt = 0, minpos = 0;
  float tau = -CUDART_INF_F;
  auto rescan = [&]() {
    float ws = CUDART_INF_F;
    int wid = -1, wp = 0;
    for (int kk = 0; kk < d.K; ++kk) {
      const float v = ls[kk * TK_ROWS + tid];
      const int id = li[kk * TK_ROWS + tid];
      if (v < ws || (v == ws && id > wid)) ws = v, wid = id, wp = kk;
    }
    tau = ws;
    minpos = wp;
  };

  const long long n = b1 > b0 ? b1 - b0 : 0;
  const long long n_tiles = (n + TK_TILE - 1) / TK_TILE;
  if (n_tiles > 0) load_tile(0, b0);
  cp_async_commit();
  for (long long j = 0; j < n_tiles; ++j) {
    if (j + 1 < n_tiles) load_tile((int)((j + 1) & 1), b0 + (j + 1) * TK_TILE);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const float* kt = sk + (int)(j & 1) * TK_TILE * 64;
    const long long t0 = b0 + j * TK_TILE;
    const int nk = (int)(b1 - t0 < TK_TILE ? b1 - t0 : TK_TILE);
    for (int jj = 0; jj < nk; ++jj) {
      const float4* kr = reinterpret_cast<const float4*>(kt + jj * 64);
      float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const float4 kv = kr[c];
        s0 = fmaf(q[4 * c], kv.x, s0);
        s1 = fmaf(q[4 * c + 1], kv.y, s1);
        s2 = fmaf(q[4 * c + 2], kv.z, s2);
        s3 = fmaf(q[4 * c + 3], kv.w, s3);
      }
      const float sc = ((s0 + s1) + (s2 + s3)) * d.scale;
      if (active && sc > tau) {
        const int beta = (int)(t0 + jj);
        if (cnt < d.K) {
          ls[cnt * TK_ROWS + tid] = sc;
          li[cnt * TK_ROWS + tid] = beta;
          if (++cnt == d.K) rescan();
        } else {
          ls[minpos * TK_ROWS + tid] = sc;
          li[minpos * TK_ROWS + tid] = beta;
          rescan();
        }
      }
    }
    __syncthreads();
  }
  if (!active) return;
  const long long out = ((h * d.Tc + a) * n_split + sp) * d.K;
  for (int kk = 0; kk < d.K; ++kk) {
    cand_s[out + kk] = kk < cnt ? ls[kk * TK_ROWS + tid] : -CUDART_INF_F;
    cand_i[out + kk] = kk < cnt ? li[kk * TK_ROWS + tid] : -1;
  }
}

constexpr int MG_WARPS = 4;

// One warp per (head, entry): K_eff rounds of a warp-wide arg-max over the
// candidates (ties to the lower id), then a rank sort of the chosen ids.
__global__ void __launch_bounds__(MG_WARPS * 32)
    topk_merge_kernel(Dims d, const float* __restrict__ cand_s, const int* __restrict__ cand_i,
                      int n_split, int* __restrict__ sel) {
  extern __shared__ __align__(16) unsigned char mg_smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nc = n_split * d.K;
  float* cs = reinterpret_cast<float*>(mg_smem) + warp * nc;
  int* ci = reinterpret_cast<int*>(reinterpret_cast<float*>(mg_smem) + MG_WARPS * nc) + warp * nc;
  int* chosen = reinterpret_cast<int*>(reinterpret_cast<float*>(mg_smem) + 2 * MG_WARPS * nc) +
                warp * kMaxTopK;
  const long long rid = (long long)blockIdx.x * MG_WARPS + warp;  // = h*Tc + a
  if (rid >= (long long)d.H * d.Tc) return;
  const float* src_s = cand_s + rid * nc;
  const int* src_i = cand_i + rid * nc;
  for (int i = lane; i < nc; i += 32) {
    cs[i] = src_s[i];
    ci[i] = src_i[i];
  }
  __syncwarp();
  for (int r = 0; r < d.Keff; ++r) {
    float bs = -CUDART_INF_F;
    int bid = -1, bpos = -1;
    for (int i = lane; i < nc; i += 32) {
      const float s = cs[i];
      const int id = ci[i];
      if (id >= 0 && (s > bs || (s == bs && (unsigned)id < (unsigned)bid))) bs = s, bid = id, bpos = i;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float s2 = __shfl_xor_sync(0xffffffffu, bs, off);
      const int i2 = __shfl_xor_sync(0xffffffffu, bid, off);
      const int p2 = __shfl_xor_sync(0xffffffffu, bpos, off);
      if (i2 >= 0 && (s2 > bs || (s2 == bs && (unsigned)i2 < (unsigned)bid))) bs = s2, bid = i2, bpos = p2;
    }
    if (lane == 0) {
      chosen[r] = bid;
      if (bpos >= 0) ci[bpos] = -1;
    }
    __syncwarp();
  }
  int* dst = sel + rid * d.K;
  for (int i = lane; i < d.Keff; i += 32) {
    const int me = chosen[i];
    int rank = 0;
    for (int j = 0; j < d.Keff; ++j) rank += chosen[j] < me;
    dst[rank] = me;
  }
  for (int i = d.Keff + lane; i < d.K; i += 32) dst[i] = -1;
}

// One thread per (head, entry): merge of two ascending lists (-1 padded).
__global__ void selection_union_kernel(long long rows, int na, int nb, int K, const int* __restrict__ sel_a,
                                       const int* __restrict__ sel_b, int* __restrict__ sel) {
  const long long rid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (rid >= rows) return;
  const int* a = sel_a + rid * na;
  const int* b = sel_b + rid * nb;
  int* o = sel + rid * K;
  int i = 0, j = 0, n = 0;
  while (n < K) {
    const int x = i < na ? a[i] : -1;
    const int y = j < nb ? b[j] : -1;
    if (x < 0 && y < 0) break;
    if (y < 0 || (x >= 0 && x < y)) {
      o[n++] = x;
      ++i;
    } else {
      o[n++] = y;
      ++j;
    }
  }
  for (; n < K; ++n) o[n] = -1;
}

}  // namespace

cudaError_t launch_selection_union(const Dims& d, const int* sel_a, int na, const int* sel_b, int nb,
                                   int* sel, cudaStream_t st) {
  const long long rows = (long long)d.H * d.Tc;
  selection_union_kernel<<<(unsigned)((rows + 255) / 256), 256, 0, st>>>(rows, na, nb, d.K, sel_a, sel_b,
                                                                           sel);
  return cudaGetLastError();
}

cudaError_t launch_block_scores_topk(const Dims& d, const float* qc32, const float* kc32,
                                     float* cand_score, int* cand_idx, int n_split,
                                     cudaStream_t st) {
  const size_t smem = (size_t)2 * TK_TILE * 64 * sizeof(float) + (size_t)d.K * TK_ROWS * 8;
  cudaError_t e = cudaFuncSetAttribute(block_scores_topk_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((d.Tc + TK_ROWS - 1) / TK_ROWS), (unsigned)d.H, (unsigned)n_split);
  block_scores_topk_kernel<<<grid, TK_ROWS, smem, st>>>(d, qc32, kc32, cand_score, cand_idx, n_split);
  return cudaGetLastError();
}

cudaError_t launch_topk_merge(const Dims& d, const float* cand_score, const int* cand_idx,
                              int n_split, int* sel, cudaStream_t st) {
  const int nc = n_split * d.K;
  const size_t smem = (size_t)MG_WARPS * (nc * 8 + kMaxTopK * 4);
  cudaError_t e =
      cudaFuncSetAttribute(topk_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long long rows = (long long)d.H * d.Tc;
  topk_merge_kernel<<<(unsigned)((rows + MG_WARPS - 1) / MG_WARPS), MG_WARPS * 32, smem, st>>>(
      d, cand_score, cand_idx, n_split, sel);
  return cudaGetLastError();
}

}  // namespace gsa
