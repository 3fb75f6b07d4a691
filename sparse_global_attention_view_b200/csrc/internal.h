// Launchers shared between the C-ABI layer (host.cu) and the kernel files.
// Each returns cudaGetLastError() after enqueueing on `st`; arguments are
// validated by the caller.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"

namespace gsa {

cudaError_t launch_pool(const Dims& d, const bf16* q, const bf16* k, const bf16* v, float* qc32,
                        float* kc32, bf16* vc, bf16* qc, bf16* kc, bf16* ks, bf16* vs,
                        cudaStream_t st);

// Flash-style attention over rows of a strided [rows][H][64] layout, per head.
struct AttnArgs {
  const bf16* q;
  long long q_row, q_head;  // element strides
  long long n_q;
  const bf16* k;
  const bf16* v;
  long long kv_row, kv_head;
  long long n_k;
  void* o;  // bf16 or fp32
  long long o_row, o_head;
  bool o_f32;
  float* lse;  // nullable, [n_q][H] with strides lse_row, lse_head
  long long lse_row, lse_head;
  int H;
  float scale, scale_log2;
};
cudaError_t launch_attn_mma(const AttnArgs& a, cudaStream_t st);

// Attention on tcgen05/TMEM fed by TMA.  Q is token-major [n_q][H][64]; K/V are
// token-major [kv_rows][H][64] or, with kv_head_major, [H][kv_rows][64].
struct AttnTcArgs {
  long long n_q, n_k;
  int H;
  float c2;  // softmax scale * log2(e)
  void* out;
  int out_f32;
  long long o_row, o_head;
  float* lse;  // nullable: natural-log sum of exp of the scaled logits
  long long lse_row, lse_head;
  unsigned* err;  // device error word
  int kv_head_major;
  long long seg_len;   // > 0: attention within consecutive segments of this many tokens
  long long seg_ctas;  // set by the launcher
  long long wait_cycles;  // limit of the in-kernel waits of one role on another
};
cudaError_t launch_attn_tc(const AttnTcArgs& a, const bf16* q, const bf16* k, const bf16* v,
                           long long kv_rows, cudaStream_t st);
// y[i] = the attention softmax's FMA-pipe 2^x of x[i] (self-test of that path).
cudaError_t launch_exp2_selftest(const float* x, float* y, long long n, cudaStream_t st);

// 3-D tiled TMA map (128-byte swizzle) over bf16 or fp32 data; dims and
// strides innermost first, strides in bytes.  False if the driver refuses it.
bool make_tmap_3d(CUtensorMap* m, bool fp32, const void* base, unsigned long long d0,
                  unsigned long long d1, unsigned long long d2, unsigned long long s1,
                  unsigned long long s2, unsigned b0, unsigned b1, unsigned b2);

// Tiled map of rank <= 5 over bf16 data (128-byte swizzle); dims and box
// innermost first, rank - 1 strides in bytes.  False if the driver refuses it.
bool make_tmap(CUtensorMap* m, const void* base, int rank, const unsigned long long* dims,
               const unsigned long long* strides, const unsigned* box);

// Compressed attention on tcgen05 fused with the S_guide streaming top-K
// (one candidate list per row, i.e. n_split = 1); needs K <= 64.  Writes the
// candidate lists when cand_score/cand_idx are non-null and the final
// selection (ascending ids, -1 padding) when sel is non-null.
// A second launch ranks the next K pairs: with `ub` set, only pairs whose key
// (score bits, then the complement of the compressed entry index: a larger
// key is a better pair) is strictly below ub[h*Tc + row] are candidates;
// `root` (nullable) receives each row's K-th best key (0 when fewer than K
// candidates exist); `scores_only` skips the attention (no V, P, PV or oc).
struct CmpPass {
  const unsigned long long* ub = nullptr;
  unsigned long long* root = nullptr;
  int scores_only = 0;
  int* best = nullptr;  // nullable [H][Tc]: each row's best-scoring block id (-1 if none)
  // Debug dump of the kernel's own unscaled logits qc32 . kc32 (tf32 products)
  // for rows [dump_row0, dump_row0 + dump_rows): dump[h][row - dump_row0][Tc].
  float* dump = nullptr;
  long long dump_row0 = 0;
  int dump_rows = 0;
  // Query tiles of the grid: tiles [tile0, tile0 + tiles) (tiles = 0: all).
  int tile0 = 0, tiles = 0;
};
bool compressed_tc_supported(const Dims& d);
constexpr int kFusedTopK = 64;  // heap capacity of one pass of the fused kernel
constexpr int kCmpTileRows = 128;  // compressed-query rows per CTA of the fused kernel
cudaError_t launch_compressed_tc(const Dims& d, const float* qc32, const float* kc32, const bf16* vc,
                                 float* oc, float* cand_score, int* cand_idx, int* sel, unsigned* err,
                                 cudaStream_t st, const CmpPass& cp = CmpPass());
// sel[h][a][0..K) = ascending union of two ascending, -1-padded lists of
// na and nb ids per row (the two ranking passes), -1 padded.
cudaError_t launch_selection_union(const Dims& d, const int* sel_a, int na, const int* sel_b, int nb,
                                   int* sel, cudaStream_t st);

cudaError_t launch_block_scores_topk(const Dims& d, const float* qc32, const float* kc32,
                                     float* cand_score, int* cand_idx, int n_split,
                                     cudaStream_t st);
cudaError_t launch_topk_merge(const Dims& d, const float* cand_score, const int* cand_idx,
                              int n_split, int* sel, cudaStream_t st);

// Selection branch on tcgen05 (transposed products per compressed entry).
// With o_spec/lse_spec the always-kept segment comes from them; otherwise,
// when NK > 0, the kernel streams the kept keys ks/vs itself.  `order`
// (nullable, H*Tc entries of h*Tc + a) is the order in which (head, entry)
// pairs are processed.  With `w` non-null the gate is fused and `out`
// receives g*oc + (1-g)*o_sel; otherwise o_sel (and lse if non-null).
cudaError_t launch_selected_tc(const Dims& d, const bf16* q, const bf16* k, const bf16* v,
                               const bf16* ks, const bf16* vs, const int* sel, const int* order,
                               const float* qc32, const float* w, const float* oc, bf16* out,
                               float* lse, const float* o_spec, const float* lse_spec, unsigned* err,
                               cudaStream_t st);

// Processing order of the (head, entry) pairs for the selection branch:
// grouped by head and by the grid position (id mod Bh*Bw) of each pair's
// best-scoring block, so pairs whose selections cover the same region of
// every frame run at the same time and share their K/V blocks in L2.
// `counts` holds H * Bf + 1 ints of scratch; order receives H * Tc ints.
cudaError_t launch_selection_order(const Dims& d, const int* best, int* counts, int* order, cudaStream_t st);

// Subsampled global attention (AVGGT SGA): sizes and the five launches.
struct SgaSizes {
  int nh, nw;             // sampled patch rows / columns per frame
  long long NK;           // kept keys: N * (S + nh * nw)
  long long n_dropped;    // patch tokens whose keys are replaced by the mean pair
};
SgaSizes sga_sizes(const Dims& d, int sub_h, int sub_w);
cudaError_t launch_sga(const Dims& d, int sub_h, int sub_w, const bf16* q, const bf16* k,
                       const bf16* v, bf16* out, bf16* ks, bf16* vs, float* part, float* mean,
                       float* o_kept, float* lse, unsigned* err, cudaStream_t st, int* launched);

cudaError_t launch_gate_combine(const Dims& d, const float* qc32, const float* w, const float* oc,
                                const bf16* o_sel, bf16* out, cudaStream_t st);

}  // namespace gsa
