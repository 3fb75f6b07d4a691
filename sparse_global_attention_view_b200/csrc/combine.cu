// Step 6: gated aggregation with nearest up-sampling (Speed3R technical
// summary 2.1: a learnable sigmoid gate computed from the query mixes the
// compression and selection branches).  One warp per (token, head); lane l
// owns channels 2l and 2l+1.  HBM-bound: reads o_sel and the entry's oc row,
// writes out.
#include "internal.h"

namespace gsa {
namespace {

__global__ void __launch_bounds__(256)
    gate_combine_kernel(Dims d, const float* __restrict__ qc32, const float* __restrict__ w,
                        const float* __restrict__ oc, const bf16* __restrict__ o_sel,
                        bf16* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const long long gid = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (gid >= d.T * d.H) return;
  const long long t = gid / d.H;
  const int h = (int)(gid - t * d.H);
  const long long a = entry_of_token(d, t);
  const long long ea = (a * d.H + h) * kHeadDim;
  const float2 qv = reinterpret_cast<const float2*>(qc32 + ea)[lane];
  const float2 wv = reinterpret_cast<const float2*>(w + (long long)h * kHeadDim)[lane];
  float z = qv.x * wv.x + qv.y * wv.y;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
  const float g = 1.f / (1.f + expf(-z));
  const float2 cm = reinterpret_cast<const float2*>(oc + ea)[lane];
  const long long et = (t * d.H + h) * kHeadDim;
  const float2 sv = __bfloat1622float2(reinterpret_cast<const __nv_bfloat162*>(o_sel + et)[lane]);
  reinterpret_cast<uint32_t*>(out + et)[lane] =
      pack_bf16x2(g * cm.x + (1.f - g) * sv.x, g * cm.y + (1.f - g) * sv.y);
}

}  // namespace

cudaError_t launch_gate_combine(const Dims& d, const float* qc32, const float* w, const float* oc,
                                const bf16* o_sel, bf16* out, cudaStream_t st) {
  const long long warps = d.T * d.H;
  if (warps > 0)
    gate_combine_kernel<<<(unsigned)((warps + 7) / 8), 256, 0, st>>>(d, qc32, w, oc, o_sel, out);
  return cudaGetLastError();
}

}  // namespace gsa
