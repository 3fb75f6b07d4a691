// The C ABI of libgsa (include/gsa.h): argument validation, size derivation,
// workspace layout, and the enqueueing of each step on the caller's stream.
// Nothing here allocates device memory or keeps state between calls.
#include <math.h>
#include <stdint.h>

#include "internal.h"

using gsa::bf16;
using gsa::Dims;

namespace {

inline bool al16(const void* p) { return ((uintptr_t)p & 15u) == 0; }
inline bool dev_ptr(const void* p) { return p != nullptr && al16(p); }
inline bool opt_ptr(const void* p) { return p == nullptr || al16(p); }
inline size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }
inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }
inline gsa_status cuda_status(cudaError_t e) { return e == cudaSuccess ? GSA_OK : GSA_ERR_CUDA; }

gsa_status make_dims(const gsa_shape* s, Dims* d, gsa_sizes* z) {
  if (s == nullptr) return GSA_ERR_INVALID_ARG;
  if (s->n_frames < 1 || s->n_special < 0 || s->hp < 1 || s->wp < 1 || s->n_heads < 1 ||
      s->head_dim < 1 || s->pool < 1 || s->top_k < 1)
    return GSA_ERR_INVALID_ARG;
  if (s->keep != GSA_KEEP_SPECIALS && s->keep != GSA_KEEP_REFERENCE) return GSA_ERR_INVALID_ARG;
  if (!(s->scale >= 0.f) || isinf(s->scale)) return GSA_ERR_INVALID_ARG;
  if (s->wait_limit_ns < 0) return GSA_ERR_INVALID_ARG;
  if (s->head_dim != gsa::kHeadDim || s->pool > gsa::kMaxPool || s->top_k > gsa::kMaxTopK ||
      s->n_heads > 128)
    return GSA_ERR_UNSUPPORTED;
  const long long L = (long long)s->n_special + (long long)s->hp * s->wp;
  const long long Bh = (s->hp + s->pool - 1) / s->pool, Bw = (s->wp + s->pool - 1) / s->pool;
  const long long Bf = Bh * Bw, E = s->n_special + Bf;
  const long long N = s->n_frames;
  const long long T = N * L, Tc = N * E, NB = N * Bf, NS = N * s->n_special;
  const bool ref = s->keep == GSA_KEEP_REFERENCE;
  const long long NK = ref ? L + (N - 1) * (s->n_special > 0 ? 1 : 0) : NS;
  const long long B0 = ref ? Bf : 0;
  // token / block ids are int32 on the device, grids are at most 2^31-1 wide
  if (L > INT32_MAX || T > INT32_MAX || NB + NS + NK > INT32_MAX) return GSA_ERR_INVALID_ARG;
  Dims t;
  t.N = s->n_frames;
  t.S = s->n_special;
  t.Hp = s->hp;
  t.Wp = s->wp;
  t.H = s->n_heads;
  t.P = s->pool;
  t.K = s->top_k;
  t.Keff = (int)(NB - B0 < s->top_k ? NB - B0 : s->top_k);
  t.keep = s->keep;
  t.NK = NK;
  t.B0 = B0;
  t.L = (int)L;
  t.E = (int)E;
  t.Bh = (int)Bh;
  t.Bw = (int)Bw;
  t.Bf = (int)Bf;
  t.T = T;
  t.Tc = Tc;
  t.NB = NB;
  t.NS = NS;
  t.scale = s->scale > 0.f ? s->scale : 1.f / sqrtf((float)s->head_dim);
  t.scale_log2 = t.scale * 1.4426950408889634f;
  // SM clocks stay below 2 GHz: two cycles per nanosecond is at least the time asked
  t.wait_cycles = s->wait_limit_ns > 0 ? 2LL * s->wait_limit_ns : 4000000000LL;
  t.mE = 0xffffffffu / (uint32_t)(E > 0 ? E : 1);
  t.mBf = 0xffffffffu / (uint32_t)(Bf > 0 ? Bf : 1);
  t.mBw = 0xffffffffu / (uint32_t)(Bw > 0 ? Bw : 1);
  t.mTc = 0xffffffffu / (uint32_t)(Tc > 0 ? Tc : 1);
  if (d) *d = t;
  if (z) {
    z->T = T;
    z->Tc = Tc;
    z->NB = NB;
    z->NS = NS;
    z->NK = NK;
    z->B0 = B0;
    z->L = t.L;
    z->E = t.E;
    z->Bh = t.Bh;
    z->Bw = t.Bw;
    z->Bf = t.Bf;
    z->K_eff = t.Keff;
  }
  return GSA_OK;
}

constexpr int kMaxCandidates = 2048;  // n_split * K per row in the merge

// K in (64, 128]: the fused kernel runs twice (top 64, then the next K - 64
// below the first pass's 64th-best key) and the two selections are merged.
bool two_pass(const Dims& d) { return d.K > gsa::kFusedTopK && d.K <= 2 * gsa::kFusedTopK; }
// gsa_forward ranks on the fused tensor-core kernel (one or two passes)
bool fused_path(const Dims& d) { return gsa::compressed_tc_supported(d) || two_pass(d); }

int forward_splits(const Dims& d) {
  if (gsa::compressed_tc_supported(d) || two_pass(d)) return 1;
  const long long row_ctas = ((d.Tc + 127) / 128) * d.H;
  long long ns = (2 * 148 + row_ctas - 1) / row_ctas;
  if (ns < 1) ns = 1;
  if (ns > 16) ns = 16;
  if (ns > d.NB - d.B0) ns = d.NB - d.B0;
  if (ns < 1) ns = 1;
  while (ns > 1 && ns * d.K > kMaxCandidates) --ns;
  return (int)ns;
}

struct Layout {
  size_t qc32, kc32, vc, qc, kc, ks, vs, oc, cs, ci, sel, ospec, lspec, sel_a, sel_b, root, best, order,
      counts, total;
  int n_split;
};

Layout forward_layout(const Dims& d) {
  Layout l;
  l.n_split = forward_splits(d);
  const size_t ent = (size_t)d.Tc * d.H * gsa::kHeadDim;
  const size_t spc = (size_t)d.NK * d.H * gsa::kHeadDim;
  // the fused compressed kernel writes the selection directly: no candidate lists
  const bool fused = gsa::compressed_tc_supported(d) || two_pass(d);
  const size_t cand = fused ? 0 : (size_t)d.H * d.Tc * l.n_split * d.K;
  size_t o = GSA_WS_HEADER_BYTES;
  auto take = [&](size_t bytes) {
    size_t at = o;
    o += up256(bytes);
    return at;
  };
  l.qc32 = take(ent * 4);
  l.kc32 = take(ent * 4);
  l.vc = take(ent * 2);
  l.qc = take(ent * 2);
  l.kc = take(ent * 2);
  l.ks = take(spc * 2);
  l.vs = take(spc * 2);
  l.oc = take(ent * 4);
  l.cs = take(cand * 4);
  l.ci = take(cand * 4);
  l.sel = take((size_t)d.H * d.Tc * d.K * 4);
  // the always-kept segment of the selection branch: normalised output and lse
  const size_t tok_heads = d.NK > 0 ? (size_t)d.T * d.H : 0;
  l.ospec = take(tok_heads * gsa::kHeadDim * 4);
  l.lspec = take(tok_heads * 4);
  // the two ranking passes of K in (64, 128]: their selections and the bound
  const size_t rows2 = two_pass(d) ? (size_t)d.H * d.Tc : 0;
  l.sel_a = take(rows2 * gsa::kFusedTopK * 4);
  l.sel_b = take(rows2 * gsa::kFusedTopK * 4);
  l.root = take(rows2 * 8);
  // the processing order of the selection branch (fused paths): each row's
  // best block, the (head, entry) pairs sorted by its position, the buckets
  const size_t rows_o = fused ? (size_t)d.H * d.Tc : 0;
  l.best = take(rows_o * 4);
  l.order = take(rows_o * 4);
  l.counts = take(fused ? ((size_t)d.H * d.Bf + 1) * 4 : 0);
  l.total = o;
  return l;
}

}  // namespace

extern "C" {

const char* gsa_status_string(gsa_status s) {
  switch (s) {
    case GSA_OK: return "ok";
    case GSA_ERR_INVALID_ARG: return "invalid argument";
    case GSA_ERR_UNSUPPORTED: return "unsupported shape (head_dim must be 64, pool <= 4, top_k <= 128, n_heads <= 128)";
    case GSA_ERR_WORKSPACE: return "workspace too small";
    case GSA_ERR_CUDA: return "CUDA error";
    case GSA_ERR_TIMEOUT: return "device wait timed out";
    case GSA_ERR_DEVICE_CHECK: return "device-side check failed";
    case GSA_ERR_SCRATCH_LIMIT:
      return "shape needs more scratch than gsa_forward_noalloc's fixed device array "
             "(GSA_NOALLOC_SCRATCH_BYTES); use gsa_forward with a workspace";
  }
  return "unknown status";
}

int32_t gsa_last_cuda_error(void) { return (int32_t)cudaPeekAtLastError(); }

const char* gsa_cuda_error_name(int32_t code) { return cudaGetErrorName((cudaError_t)code); }

gsa_status gsa_derive(const gsa_shape* shape, gsa_sizes* out) {
  if (out == nullptr) return GSA_ERR_INVALID_ARG;
  return make_dims(shape, nullptr, out);
}

gsa_status gsa_workspace_size(const gsa_shape* shape, size_t* bytes) {
  Dims d;
  if (bytes == nullptr) return GSA_ERR_INVALID_ARG;
  gsa_status st = make_dims(shape, &d, nullptr);
  if (st != GSA_OK) return st;
  *bytes = forward_layout(d).total;
  return GSA_OK;
}

gsa_status gsa_workspace_init(void* ws, void* stream) {
  if (!dev_ptr(ws)) return GSA_ERR_INVALID_ARG;
  return cuda_status(cudaMemsetAsync(ws, 0, GSA_WS_HEADER_BYTES, as_stream(stream)));
}

gsa_status gsa_pool_kv(const gsa_shape* shape, const gsa_bf16* q, const gsa_bf16* k,
                       const gsa_bf16* v, float* qc32, float* kc32, gsa_bf16* vc, gsa_bf16* qc,
                       gsa_bf16* kc, gsa_bf16* ks, gsa_bf16* vs, void* ws, void* stream) {
  Dims d;
  gsa_status st = make_dims(shape, &d, nullptr);
  if (st != GSA_OK) return st;
  if (!dev_ptr(q) || !dev_ptr(k) || !dev_ptr(v) || !dev_ptr(qc32) || !dev_ptr(kc32) ||
      !dev_ptr(vc) || !opt_ptr(qc) || !opt_ptr(kc) || !opt_ptr(ks) || !opt_ptr(vs) || !dev_ptr(ws))
    return GSA_ERR_INVALID_ARG;
  if ((ks == nullptr) != (vs == nullptr)) return GSA_ERR_INVALID_ARG;
  if (d.NK == 0) ks = vs = nullptr;
  return cuda_status(gsa::launch_pool(d, (const bf16*)q, (const bf16*)k, (const bf16*)v, qc32, kc32,
                                      (bf16*)vc, (bf16*)qc, (bf16*)kc, (bf16*)ks, (bf16*)vs,
                                      as_stream(stream)));
}

gsa_status gsa_compressed_attn(const gsa_shape* shape, const gsa_bf16* qc, const gsa_bf16* kc,
                               const gsa_bf16* vc, const float* qc32, const float* kc32,
                               float* oc, float* cand_score, int32_t* cand_idx, int32_t n_split,
                               void* ws, void* stream) {
  Dims d;
  gsa_status st = make_dims(shape, &d, nullptr);
  if (st != GSA_OK) return st;
  if (!dev_ptr(qc) || !dev_ptr(kc) || !dev_ptr(vc) || !dev_ptr(qc32) || !dev_ptr(kc32) ||
      !dev_ptr(oc) || !dev_ptr(cand_score) || !dev_ptr(cand_idx) || !dev_ptr(ws))
    return GSA_ERR_INVALID_ARG;
  if (n_split < 1 || n_split > 64 || (long long)n_split * d.K > kMaxCandidates)
    return GSA_ERR_INVALID_ARG;
  cudaStream_t s = as_stream(stream);
  if (n_split == 1 && gsa::compressed_tc_supported(d))
    return cuda_status(gsa::launch_compressed_tc(d, qc32, kc32, (const bf16*)vc, oc, cand_score,
                                                 cand_idx, nullptr, (unsigned*)ws, s));
  gsa::AttnArgs a;
  a.q = (const bf16*)qc;
  a.k = (const bf16*)kc;
  a.v = (const bf16*)vc;
  a.q_row = a.kv_row = a.o_row = (long long)d.H * gsa::kHeadDim;
  a.q_head = a.kv_head = a.o_head = gsa::kHeadDim;
  a.n_q = a.n_k = d.Tc;
  a.o = oc;
  a.o_f32 = true;
  a.lse = nullptr;
  a.lse_row = a.lse_head = 0;
  a.H = d.H;
  a.scale = d.scale;
  a.scale_log2 = d.scale_log2;
  cudaError_t e = gsa::launch_attn_mma(a, s);
  if (e != cudaSuccess) return GSA_ERR_CUDA;
  return cuda_status(gsa::launch_block_scores_topk(d, qc32, kc32, cand_score, cand_idx, n_split, s));
}

gsa_status gsa_guide_logits(const gsa_shape* shape, const float* qc32, const float* kc32,
                            const gsa_bf16* vc, int64_t row0, int32_t n_rows, float* logits, void* ws,
                            void* stream) {
  Dims d;
  gsa_status st = make_dims(shape, &d, nullptr);
  if (st != GSA_OK) return st;
  if (!dev_ptr(qc32) || !dev_ptr(kc32) || !dev_ptr(vc) || !dev_ptr(logits) || !dev_ptr(ws))
    return GSA_ERR_INVALID_ARG;
  if (row0 < 0 || n_rows < 1 || row0 + n_rows > d.Tc) return GSA_ERR_INVALID_ARG;
  // the fused kernel ranks alongside (its lists are not written); its heaps
  // hold at most kFusedTopK pairs
  if (d.K > gsa::kFusedTopK) d.K = gsa::kFusedTopK;
  gsa::CmpPass cp;
  cp.scores_only = 1;
  cp.dump = logits;
  cp.dump_row0 = row0;
  cp.dump_rows = n_rows;
  cp.tile0 = (int)(row0 / gsa::kCmpTileRows);
  cp.tiles = (int)((row0 + n_rows - 1) / gsa::kCmpTileRows) - cp.tile0 + 1;
  return cuda_status(gsa::launch_compressed_tc(d, qc32, kc32, (const bf16*)vc, nullptr, nullptr, nullptr,
                                               nullptr, (unsigned*)ws, as_stream(stream), cp));
}

gsa_status gsa_topk_blocks(const gsa_shape* shape, const float* cand_score,
                           const int32_t* cand_idx, int32_t n_split, int32_t* sel, void* ws,
                           void* stream) {
  Dims d;
  gsa_status st = make_dims(shape, &d, nullptr);
  if (st != GSA_OK) return st;
  if (!dev_ptr(cand_score) || !dev_ptr(cand_idx) || !dev_ptr(sel) || !dev_ptr(ws))
    return GSA_ERR_INVALID_ARG;
  if (n_split < 1 || n_split > 64 || (long long)n_split * d.K > kMaxCandidates)
    return GSA_ERR_INVALID_ARG;
  return cuda_status(gsa::launch_topk_merge(d, cand_score, cand_idx, n_split, sel, as_stream(stream)));
}

gsa_status gsa_selected_attn(const gsa_shape* shape, const gsa_bf16* q, const gsa_bf16* k,
                             const gsa_bf16* v, const gsa_bf16* ks, const gsa_bf16* vs,
                             const int32_t* sel, gsa_bf16* o_sel, float* lse, void* ws,
                             void* stream) {
  Dims d;
  gsa_status st = make_dims(shape, &d, nullptr);
  if (st != GSA_OK) return st;
  if (!dev_ptr(q) || !dev_ptr(k) || !dev_ptr(v) || !dev_ptr(sel) || !dev_ptr(o_sel) ||
      !opt_ptr(lse) || !dev_ptr(ws))
    return GSA_ERR_INVALID_ARG;
  if (d.NK > 0 && (!dev_ptr(ks) || !dev_ptr(vs))) return GSA_ERR_INVALID_ARG;
  return cuda_status(gsa::launch_selected_tc(d, (const bf16*)q, (const bf16*)k, (const bf16*)v,
                                             (const bf16*)ks, (const bf16*)vs, sel, nullptr, nullptr,
                                             nullptr, nullptr, (bf16*)o_sel, lse, nullptr, nullptr,
                                             (unsigned*)ws, as_stream(stream)));
}

gsa_status gsa_gate_combine(const gsa_shape* shape, const float* qc32, const float* w,
                            const float* oc, const gsa_bf16* o_sel, gsa_bf16* out, void* ws,
                            void* stream) {
  Dims d;
  gsa_status st = make_dims(shape, &d, nullptr);
  if (st != GSA_OK) return st;
  if (!dev_ptr(qc32) || !dev_ptr(w) || !dev_ptr(oc) || !dev_ptr(o_sel) || !dev_ptr(out) ||
      !dev_ptr(ws))
    return GSA_ERR_INVALID_ARG;
  return cuda_status(
      gsa::launch_gate_combine(d, qc32, w, oc, (const bf16*)o_sel, (bf16*)out, as_stream(stream)));
}

gsa_status dense_global_attn(const gsa_shape* shape, const gsa_bf16* q, const gsa_bf16* k,
                             const gsa_bf16* v, gsa_bf16* out, void* ws, void* stream) {
  Dims d;
  gsa_status st = make_dims(shape, &d, nullptr);
  if (st != GSA_OK) return st;
  if (!dev_ptr(q) || !dev_ptr(k) || !dev_ptr(v) || !dev_ptr(out) || !dev_ptr(ws))
    return GSA_ERR_INVALID_ARG;
  gsa::AttnTcArgs a;
  a.n_q = a.n_k = d.T;
  a.H = d.H;
  a.c2 = d.scale_log2;
  a.out = out;
  a.out_f32 = 0;
  a.o_row = (long long)d.H * gsa::kHeadDim;
  a.o_head = gsa::kHeadDim;
  a.lse = nullptr;
  a.lse_row = a.lse_head = 0;
  a.err = (unsigned*)ws;
  a.kv_head_major = 0;
  a.seg_len = 0;
  a.wait_cycles = d.wait_cycles;
  return cuda_status(gsa::launch_attn_tc(a, (const bf16*)q, (const bf16*)k, (const bf16*)v, d.T,
                                         as_stream(stream)));
}

gsa_status frame_attn(const gsa_shape* shape, const gsa_bf16* q, const gsa_bf16* k,
                      const gsa_bf16* v, gsa_bf16* out, void* ws, void* stream) {
  Dims d;
  gsa_status st = make_dims(shape, &d, nullptr);
  if (st != GSA_OK) return st;
  if (!dev_ptr(q) || !dev_ptr(k) || !dev_ptr(v) || !dev_ptr(out) || !dev_ptr(ws))
    return GSA_ERR_INVALID_ARG;
  gsa::AttnTcArgs a;
  a.n_q = a.n_k = d.T;
  a.H = d.H;
  a.c2 = d.scale_log2;
  a.out = out;
  a.out_f32 = 0;
  a.o_row = (long long)d.H * gsa::kHeadDim;
  a.o_head = gsa::kHeadDim;
  a.lse = nullptr;
  a.lse_row = a.lse_head = 0;
  a.err = (unsigned*)ws;
  a.kv_head_major = 0;
  a.seg_len = d.L;
  a.wait_cycles = d.wait_cycles;
  return cuda_status(gsa::launch_attn_tc(a, (const bf16*)q, (const bf16*)k, (const bf16*)v, d.T,
                                         as_stream(stream)));
}

namespace {

struct SgaLayout {
  size_t ks, vs, part, mean, o, lse, total;
};

SgaLayout sga_layout(const Dims& d, int sub_h, int sub_w) {
  const gsa::SgaSizes z = gsa::sga_sizes(d, sub_h, sub_w);
  const size_t row = (size_t)d.H * gsa::kHeadDim;
  SgaLayout l;
  size_t o = GSA_WS_HEADER_BYTES;
  auto take = [&](size_t bytes) {
    size_t at = o;
    o += up256(bytes);
    return at;
  };
  l.ks = take((size_t)z.NK * row * 2);
  l.vs = take((size_t)z.NK * row * 2);
  l.part = take((size_t)d.N * 2 * row * 4);
  l.mean = take(2 * row * 4);
  l.o = take((size_t)d.T * row * 4);
  l.lse = take((size_t)d.T * d.H * 4);
  l.total = o;
  return l;
}

}  // namespace

gsa_status sga_workspace_size(const gsa_shape* shape, int32_t sub_h, int32_t sub_w, size_t* bytes) {
  Dims d;
  if (bytes == nullptr || sub_h < 1 || sub_w < 1) return GSA_ERR_INVALID_ARG;
  gsa_status st = make_dims(shape, &d, nullptr);
  if (st != GSA_OK) return st;
  *bytes = sga_layout(d, sub_h, sub_w).total;
  return GSA_OK;
}

gsa_status sga_attn(const gsa_shape* shape, int32_t sub_h, int32_t sub_w, const gsa_bf16* q,
                    const gsa_bf16* k, const gsa_bf16* v, gsa_bf16* out, void* ws, size_t ws_bytes,
                    void* stream) {
  Dims d;
  gsa_status st = make_dims(shape, &d, nullptr);
  if (st != GSA_OK) return st;
  if (sub_h < 1 || sub_w < 1) return GSA_ERR_INVALID_ARG;
  if (!dev_ptr(q) || !dev_ptr(k) || !dev_ptr(v) || !dev_ptr(out) || !dev_ptr(ws))
    return GSA_ERR_INVALID_ARG;
  const SgaLayout l = sga_layout(d, sub_h, sub_w);
  if (ws_bytes < l.total) return GSA_ERR_WORKSPACE;
  char* base = static_cast<char*>(ws);
  int launched = 0;
  return cuda_status(gsa::launch_sga(d, sub_h, sub_w, (const bf16*)q, (const bf16*)k, (const bf16*)v,
                                     (bf16*)out, (bf16*)(base + l.ks), (bf16*)(base + l.vs),
                                     (float*)(base + l.part), (float*)(base + l.mean),
                                     (float*)(base + l.o), (float*)(base + l.lse), (unsigned*)ws,
                                     as_stream(stream), &launched));
}

gsa_status dense_global_attn_mma(const gsa_shape* shape, const gsa_bf16* q, const gsa_bf16* k,
                                 const gsa_bf16* v, gsa_bf16* out, void* ws, void* stream) {
  Dims d;
  gsa_status st = make_dims(shape, &d, nullptr);
  if (st != GSA_OK) return st;
  if (!dev_ptr(q) || !dev_ptr(k) || !dev_ptr(v) || !dev_ptr(out) || !dev_ptr(ws))
    return GSA_ERR_INVALID_ARG;
  gsa::AttnArgs a;
  a.q = (const bf16*)q;
  a.k = (const bf16*)k;
  a.v = (const bf16*)v;
  a.q_row = a.kv_row = a.o_row = (long long)d.H * gsa::kHeadDim;
  a.q_head = a.kv_head = a.o_head = gsa::kHeadDim;
  a.n_q = a.n_k = d.T;
  a.o = out;
  a.o_f32 = false;
  a.lse = nullptr;
  a.lse_row = a.lse_head = 0;
  a.H = d.H;
  a.scale = d.scale;
  a.scale_log2 = d.scale_log2;
  return cuda_status(gsa::launch_attn_mma(a, as_stream(stream)));
}

gsa_status gsa_forward_timed(const gsa_shape* shape, const gsa_bf16* q, const gsa_bf16* k,
                             const gsa_bf16* v, const float* w, gsa_bf16* out, void* ws,
                             size_t ws_bytes, void* const* events, int32_t* n_launched,
                             void* stream) {
  Dims d;
  gsa_status st = make_dims(shape, &d, nullptr);
  if (st != GSA_OK) return st;
  if (!dev_ptr(q) || !dev_ptr(k) || !dev_ptr(v) || !dev_ptr(w) || !dev_ptr(out) || !dev_ptr(ws))
    return GSA_ERR_INVALID_ARG;
  if (events != nullptr)
    for (int i = 0; i <= GSA_FORWARD_STEPS; ++i)
      if (events[i] == nullptr) return GSA_ERR_INVALID_ARG;
  const Layout l = forward_layout(d);
  if (ws_bytes < l.total) return GSA_ERR_WORKSPACE;
  char* base = static_cast<char*>(ws);
  float* qc32 = (float*)(base + l.qc32);
  float* kc32 = (float*)(base + l.kc32);
  bf16* vc = (bf16*)(base + l.vc);
  bf16* qc = (bf16*)(base + l.qc);
  bf16* kc = (bf16*)(base + l.kc);
  bf16* ks = d.NK > 0 ? (bf16*)(base + l.ks) : nullptr;
  bf16* vs = d.NK > 0 ? (bf16*)(base + l.vs) : nullptr;
  float* oc = (float*)(base + l.oc);
  float* cs = (float*)(base + l.cs);
  int* ci = (int*)(base + l.ci);
  int* sel = (int*)(base + l.sel);
  int* best = (fused_path(d)) ? (int*)(base + l.best) : nullptr;
  int* order = (fused_path(d)) ? (int*)(base + l.order) : nullptr;
  cudaStream_t s = as_stream(stream);
  int launched = 0;
  auto mark = [&](int i) -> bool {
    return events == nullptr || cudaEventRecord((cudaEvent_t)events[i], s) == cudaSuccess;
  };
  auto step = [&](cudaError_t e, int i) -> bool {
    ++launched;
    return e == cudaSuccess && mark(i);
  };
  // the ordering of the selection branch's work: three kernels
  auto step3 = [&](cudaError_t e, int i) -> bool {
    launched += 3;
    return e == cudaSuccess && mark(i);
  };
  if (!mark(0)) return GSA_ERR_CUDA;
  const bool fused = gsa::compressed_tc_supported(d);
  const bool twice = two_pass(d);
  if (!step(gsa::launch_pool(d, (const bf16*)q, (const bf16*)k, (const bf16*)v, qc32, kc32, vc,
                             (fused || twice) ? nullptr : qc, (fused || twice) ? nullptr : kc, ks, vs, s),
            1))
    return GSA_ERR_CUDA;
  if (twice) {
    // step 2: attention + the top 64 of every row (and its 64th-best key);
    // step 3: a ranking-only pass for the next K - 64 below that key (its
    // heap holds K - 64);
    // step 4: the ascending union of the two selections
    Dims d64 = d, drest = d;
    d64.K = gsa::kFusedTopK;
    drest.K = d.K - gsa::kFusedTopK;
    int* sel_a = (int*)(base + l.sel_a);
    int* sel_b = (int*)(base + l.sel_b);
    unsigned long long* root = (unsigned long long*)(base + l.root);
    gsa::CmpPass first, second;
    first.root = root;
    first.best = best;
    second.ub = root;
    second.scores_only = 1;
    if (!step(gsa::launch_compressed_tc(d64, qc32, kc32, vc, oc, nullptr, nullptr, sel_a, (unsigned*)ws, s,
                                        first),
              2) ||
        !step(gsa::launch_compressed_tc(drest, qc32, kc32, vc, oc, nullptr, nullptr, sel_b, (unsigned*)ws, s,
                                        second),
              3) ||
        gsa::launch_selection_union(d, sel_a, gsa::kFusedTopK, sel_b, drest.K, sel, s) != cudaSuccess ||
        !step3(gsa::launch_selection_order(d, best, (int*)(base + l.counts), order, s), 4))
      return GSA_ERR_CUDA;
    ++launched;  // the union
  } else if (fused) {
    // steps 1-3 in one kernel (its lists hold each row's final top-K, written
    // to sel in ascending order); step 3's interval holds the ordering of the
    // selection branch's work
    gsa::CmpPass cp;
    cp.best = best;
    if (!step(gsa::launch_compressed_tc(d, qc32, kc32, vc, oc, nullptr, nullptr, sel, (unsigned*)ws, s, cp),
              2) ||
        !mark(3) || !step3(gsa::launch_selection_order(d, best, (int*)(base + l.counts), order, s), 4))
      return GSA_ERR_CUDA;
  } else {
    gsa::AttnArgs a;
    a.q = qc;
    a.k = kc;
    a.v = vc;
    a.q_row = a.kv_row = a.o_row = (long long)d.H * gsa::kHeadDim;
    a.q_head = a.kv_head = a.o_head = gsa::kHeadDim;
    a.n_q = a.n_k = d.Tc;
    a.o = oc;
    a.o_f32 = true;
    a.lse = nullptr;
    a.lse_row = a.lse_head = 0;
    a.H = d.H;
    a.scale = d.scale;
    a.scale_log2 = d.scale_log2;
    if (!step(gsa::launch_attn_mma(a, s), 2)) return GSA_ERR_CUDA;
    if (!step(gsa::launch_block_scores_topk(d, qc32, kc32, cs, ci, l.n_split, s), 3)) return GSA_ERR_CUDA;
  }
  if (!fused && !twice && !step(gsa::launch_topk_merge(d, cs, ci, l.n_split, sel, s), 4))
    return GSA_ERR_CUDA;
  float* ospec = nullptr;
  float* lspec = nullptr;
  if (d.NK > 0) {
    // the always-kept tokens: every token attends to all NK of them
    ospec = (float*)(base + l.ospec);
    lspec = (float*)(base + l.lspec);
    gsa::AttnTcArgs a;
    a.n_q = d.T;
    a.n_k = d.NK;
    a.H = d.H;
    a.c2 = d.scale_log2;
    a.out = ospec;
    a.out_f32 = 1;
    a.o_row = (long long)d.H * gsa::kHeadDim;
    a.o_head = gsa::kHeadDim;
    a.lse = lspec;
    a.lse_row = d.H;
    a.lse_head = 1;
    a.err = (unsigned*)ws;
    a.kv_head_major = 1;
    a.seg_len = 0;
    a.wait_cycles = d.wait_cycles;
    if (!step(gsa::launch_attn_tc(a, (const bf16*)q, ks, vs, d.NK, s), 5)) return GSA_ERR_CUDA;
  } else if (!mark(5)) {
    return GSA_ERR_CUDA;
  }
  if (!step(gsa::launch_selected_tc(d, (const bf16*)q, (const bf16*)k, (const bf16*)v, ks, vs, sel, order,
                                    qc32, w, oc, (bf16*)out, nullptr, ospec, lspec, (unsigned*)ws, s),
            6))
    return GSA_ERR_CUDA;
  if (n_launched) *n_launched = launched;
  return GSA_OK;
}

gsa_status gsa_forward(const gsa_shape* shape, const gsa_bf16* q, const gsa_bf16* k,
                       const gsa_bf16* v, const float* w, gsa_bf16* out, void* ws,
                       size_t ws_bytes, void* stream) {
  return gsa_forward_timed(shape, q, k, v, w, out, ws, ws_bytes, nullptr, nullptr, stream);
}

gsa_status gsa_workspace_offsets(const gsa_shape* shape, gsa_ws_offsets* out) {
  Dims d;
  if (out == nullptr) return GSA_ERR_INVALID_ARG;
  gsa_status st = make_dims(shape, &d, nullptr);
  if (st != GSA_OK) return st;
  const Layout l = forward_layout(d);
  out->qc32 = l.qc32;
  out->kc32 = l.kc32;
  out->vc = l.vc;
  out->qc = l.qc;
  out->kc = l.kc;
  out->ks = l.ks;
  out->vs = l.vs;
  out->oc = l.oc;
  out->cand_score = l.cs;
  out->cand_idx = l.ci;
  out->sel = l.sel;
  out->o_spec = l.ospec;
  out->lse_spec = l.lspec;
  out->total = l.total;
  out->n_split = l.n_split;
  out->best = l.best;
  out->order = l.order;
  return GSA_OK;
}

gsa_status gsa_selftest_exp2(const float* x, float* y, int64_t n, void* stream) {
  if (n < 0 || (n > 0 && (x == nullptr || y == nullptr))) return GSA_ERR_INVALID_ARG;
  return cuda_status(gsa::launch_exp2_selftest(x, y, (long long)n, as_stream(stream)));
}

gsa_status gsa_check_device_error(void* ws, void* stream) {
  if (!dev_ptr(ws)) return GSA_ERR_INVALID_ARG;
  cudaStream_t s = as_stream(stream);
  unsigned word = 0;
  if (cudaMemcpyAsync(&word, ws, sizeof(word), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return GSA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return GSA_ERR_CUDA;
  if (word != 0 && cudaMemsetAsync(ws, 0, 3 * sizeof(word), s) != cudaSuccess) return GSA_ERR_CUDA;
  if (word & gsa::kErrTimeout) return GSA_ERR_TIMEOUT;
  if (word & gsa::kErrDeviceCheck) return GSA_ERR_DEVICE_CHECK;
  return GSA_OK;
}

}  // extern "C"
