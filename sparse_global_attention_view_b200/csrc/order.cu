// Processing order of the selection branch's (head, entry) pairs.
//
// The selected blocks of the pairs that run at the same time should be few
// enough to stay in L2 (126 MB), but the K/V of one head is 2 x T x 128 bytes
// (352 MB for 1000 VGGT frames).  Pairs in frame order select blocks spread
// over the whole scene; pairs grouped by the grid position of their best
// block select blocks around that position in every frame.  So the pairs are
// counting-sorted by (head, position of the best block): a histogram, an
// exclusive scan and a scatter.  The order among pairs of one group is left
// to the atomics; it changes no result, since every pair is computed on its own.
#include "internal.h"

namespace gsa {
namespace {

__device__ __forceinline__ int bucket_of(const Dims& d, const int* best, long long pair) {
  const int h = (int)(pair / d.Tc);
  const int id = best[pair];
  return h * d.Bf + (id >= 0 ? id % d.Bf : 0);
}

__global__ void order_count_kernel(Dims d, const int* __restrict__ best, int* __restrict__ counts) {
  const long long n = (long long)d.H * d.Tc;
  for (long long p = (long long)blockIdx.x * blockDim.x + threadIdx.x; p < n; p += (long long)gridDim.x * blockDim.x)
    atomicAdd(&counts[bucket_of(d, best, p)], 1);
}

// Exclusive scan of the nb bucket counts in place (one CTA); counts[nb]
// receives the total.
__global__ void order_scan_kernel(int* __restrict__ counts, int nb) {
  __shared__ int part[1024];
  const int t = threadIdx.x;
  const int per = (nb + blockDim.x - 1) / blockDim.x;
  const int b0 = min(nb, t * per), b1 = min(nb, b0 + per);
  int s = 0;
  for (int b = b0; b < b1; ++b) s += counts[b];
  part[t] = s;
  __syncthreads();
  for (int off = 1; off < (int)blockDim.x; off <<= 1) {
    const int v = t >= off ? part[t - off] : 0;
    __syncthreads();
    part[t] += v;
    __syncthreads();
  }
  int run = part[t] - s;  // exclusive prefix of this thread's range
  for (int b = b0; b < b1; ++b) {
    const int c = counts[b];
    counts[b] = run;
    run += c;
  }
  if (t == (int)blockDim.x - 1) counts[nb] = part[t];
}

__global__ void order_scatter_kernel(Dims d, const int* __restrict__ best, int* __restrict__ cursor,
                                     int* __restrict__ order) {
  const long long n = (long long)d.H * d.Tc;
  for (long long p = (long long)blockIdx.x * blockDim.x + threadIdx.x; p < n; p += (long long)gridDim.x * blockDim.x)
    order[atomicAdd(&cursor[bucket_of(d, best, p)], 1)] = (int)p;
}

}  // namespace

cudaError_t launch_selection_order(const Dims& d, const int* best, int* counts, int* order, cudaStream_t st) {
  const int nb = d.H * d.Bf;
  cudaError_t e = cudaMemsetAsync(counts, 0, sizeof(int) * (size_t)(nb + 1), st);
  if (e != cudaSuccess) return e;
  const long long n = (long long)d.H * d.Tc;
  const unsigned grid = (unsigned)min((n + 255) / 256, 148LL * 16);
  order_count_kernel<<<grid, 256, 0, st>>>(d, best, counts);
  order_scan_kernel<<<1, 1024, 0, st>>>(counts, nb);
  order_scatter_kernel<<<grid, 256, 0, st>>>(d, best, counts, order);
  return cudaGetLastError();
}

}  // namespace gsa
