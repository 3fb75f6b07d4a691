/*
 * gsa.h -- C ABI of libgsa: sparse global attention over N views (GSA) and the
 * dense global attention it replaces, hand-written CUDA for sm_100a (B200).
 *
 * The operation is the global self-attention layer of VGGT-style feed-forward
 * multi-view reconstruction in the sparse dual-branch form of
 * "Speed3R: Sparse Feed-forward 3D Reconstruction Models" (technical summary,
 * section 2.1 "Dual-branch attention", and section 2.2 "Speed3R-VGGT"):
 *   - compression branch: per frame, 4x4 (generally P x P) average pooling of
 *     Q, K and V over the patch grid, dense attention in the pooled sequence,
 *     output up-sampled (nearest) back to the fine tokens;
 *   - S_guide: the pooled scores of each compressed query against every patch
 *     block; the Top-K blocks per (query block, head) are selected;
 *   - selection branch: fine attention of each token over the tokens of its
 *     block's selected blocks plus an always-kept token set: every special
 *     token (keep = GSA_KEEP_SPECIALS), or the whole reference frame 0 plus
 *     the camera token of every frame (keep = GSA_KEEP_REFERENCE, the
 *     Speed3R-VGGT reading of "reference-frame and camera tokens are always
 *     kept"; frame 0's blocks are then not top-K candidates);
 *   - gated aggregation: g = sigmoid(q_mean . w_h) per (query block, head),
 *     out = g * up(O_cmp) + (1 - g) * O_sel.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Tokens: frame f holds S special tokens, then Hp*Wp patch tokens (row-major);
 * frames are concatenated: T = N * (S + Hp*Wp).  Q, K, V, out are row-major
 * [T][H][64] bf16 (gsa_bf16 = the raw 16-bit pattern).
 * Compressed sequence: per frame, the S specials then the Bh*Bw blocks
 * (row-major), Bh = ceil(Hp/P), Bw = ceil(Wp/P): Tc = N * (S + Bh*Bw) entries,
 * stored [Tc][H][64].  Patch block id beta = f*Bh*Bw + br*Bw + bc (0 <= beta <
 * NB = N*Bh*Bw).  A block at the right/bottom edge holds only the patches that
 * exist; its pooled value is the mean over those.
 * Always-kept copies: [H][NK][64] bf16 (head-major) of the always-kept tokens'
 * K / V in token order: NK = N*S (all specials, frame-major) for
 * GSA_KEEP_SPECIALS; NK = (S + Hp*Wp) + (N-1)*min(S,1) for GSA_KEEP_REFERENCE
 * (frame 0's tokens, then special slot 0 -- the camera token -- of frames
 * 1..N-1).  Top-K candidates are the blocks beta >= B0 (B0 = 0, or Bh*Bw for
 * GSA_KEEP_REFERENCE); K_eff = min(K, NB - B0), which may be 0.
 *
 * Pointers: every buffer pointer is a device pointer (cudaMalloc'd or a slice of
 * one) and must be 16-byte aligned; the caller owns all memory and the library
 * never allocates, frees or keeps a pointer after a call returns.  `stream` is
 * a cudaStream_t (NULL = the legacy default stream); all work is enqueued on it
 * and the calls return without synchronising (except gsa_check_device_error).
 *
 * Workspace: every compute call takes `ws`, device memory of at least
 * GSA_WS_HEADER_BYTES whose first word is the device error word.  Zero it once
 * after allocation (gsa_workspace_init); kernels only set bits in it, and
 * gsa_check_device_error reads and clears it.  gsa_forward also carves its
 * intermediates from `ws` (size from gsa_workspace_size).
 *
 * Errors: arguments are validated on the host before anything is enqueued; a
 * failed check returns GSA_ERR_INVALID_ARG / GSA_ERR_UNSUPPORTED /
 * GSA_ERR_WORKSPACE and launches nothing.  A launch failure returns
 * GSA_ERR_CUDA.  Nothing in the library traps the device.
 */
#ifndef GSA_H_
#define GSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t gsa_bf16; /* bfloat16 bit pattern */

typedef enum {
  GSA_OK = 0,
  GSA_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size or count */
  GSA_ERR_UNSUPPORTED = 2,   /* valid but not built for (head_dim != 64, pool > 4, top_k > 128) */
  GSA_ERR_WORKSPACE = 3,     /* workspace smaller than required */
  GSA_ERR_CUDA = 4,          /* a CUDA launch or runtime call failed */
  GSA_ERR_TIMEOUT = 5,       /* device error word: a bounded wait ran out */
  GSA_ERR_DEVICE_CHECK = 6,  /* device error word: an in-kernel bounds check failed */
  GSA_ERR_SCRATCH_LIMIT = 7  /* gsa_forward_noalloc: the shape needs more than its fixed scratch */
} gsa_status;

/* One layer call's sizes.  All fields are read by every entry point. */
typedef struct {
  int32_t n_frames;  /* N >= 1 */
  int32_t n_special; /* S >= 0 special tokens per frame (camera/register) */
  int32_t hp;        /* patch grid height >= 1 */
  int32_t wp;        /* patch grid width >= 1 */
  int32_t n_heads;   /* H in [1, 128] */
  int32_t head_dim;  /* D; only 64 is built */
  int32_t pool;      /* P in [1, 4]: P x P average pooling of the patch grid */
  int32_t top_k;     /* K in [1, 128]: selected blocks per (query block, head) */
  float scale;       /* softmax scale; 0 means 1/sqrt(D) */
  int32_t keep;      /* always-kept set of the selection branch: GSA_KEEP_* */
  int32_t wait_limit_ns; /* >= 0; 0 = default.  Every in-kernel wait of one pipeline role
                            on another (a TMA copy, a tensor-core product, a softmax tile)
                            gives up after about this many nanoseconds (default about 2 s)
                            and records GSA_ERR_TIMEOUT in the error word; the kernel then
                            drains its own copies and products and returns.  A tiny value
                            exercises that path (test hook). */
} gsa_shape;

#define GSA_KEEP_SPECIALS 0  /* every special token of every frame */
#define GSA_KEEP_REFERENCE 1 /* frame 0 whole + each frame's camera token (slot 0) */

/* Derived sizes (see the conventions above). */
typedef struct {
  int64_t T;     /* fine tokens N*(S+Hp*Wp) */
  int64_t Tc;    /* compressed entries N*(S+Bh*Bw) */
  int64_t NB;    /* patch blocks N*Bh*Bw (top-K candidates) */
  int64_t NS;    /* special tokens N*S */
  int64_t NK;    /* always-kept tokens (see keep) */
  int64_t B0;    /* first top-K candidate block id */
  int32_t L;     /* tokens per frame S+Hp*Wp */
  int32_t E;     /* compressed entries per frame S+Bh*Bw */
  int32_t Bh, Bw, Bf;
  int32_t K_eff; /* min(K, NB - B0) */
} gsa_sizes;

#define GSA_WS_HEADER_BYTES 256

/* Validate `shape` and fill `out`.  Pure host code (needs no GPU). */
gsa_status gsa_derive(const gsa_shape* shape, gsa_sizes* out);

/* Bytes of workspace gsa_forward needs for `shape` (header included).  Host only. */
gsa_status gsa_workspace_size(const gsa_shape* shape, size_t* bytes);

/* Zero the workspace header (the device error word) on `stream`. */
gsa_status gsa_workspace_init(void* ws, void* stream);

/*
 * Step 1, compression by pooling (Speed3R technical summary 2.1, compression
 * branch: spatial down-sampling, e.g. 4x4 average pooling, to a coarse context).
 * Reads q, k, v [T][H][64] bf16.  Writes, per compressed entry a and head h:
 *   qc32, kc32   [Tc][H][64] fp32  mean of Q / K (scores and the gate use these)
 *   vc           [Tc][H][64] bf16  mean of V (round-to-nearest-even)
 *   qc, kc       [Tc][H][64] bf16  mean of Q / K (may be NULL: not written)
 *   ks, vs       [H][NK][64] bf16 copies of the always-kept tokens' K / V
 *                (ignored when NK == 0; may be NULL: not written)
 * A special token's entry is the token itself.
 */
gsa_status gsa_pool_kv(const gsa_shape* shape, const gsa_bf16* q, const gsa_bf16* k,
                       const gsa_bf16* v, float* qc32, float* kc32, gsa_bf16* vc, gsa_bf16* qc,
                       gsa_bf16* kc, gsa_bf16* ks, gsa_bf16* vs, void* ws, void* stream);

/*
 * Steps 2-3, attention in the compressed space and its block scores
 * (technical summary 2.1; S_guide on the it page, section 2).
 *   oc [Tc][H][64] fp32: softmax(scale * qc kc^T) vc over all Tc entries.
 *   cand_score / cand_idx [H][Tc][n_split][K]: for every (head, entry) and each
 *   of `n_split` equal slices of the candidate block range [B0, NB), the K largest
 *   S_guide[h][a][beta] = scale * (qc32[a,h] . kc32[entry(beta),h]) of that
 *   slice with their block ids, unordered, padded with (-inf, -1).
 * qc / kc are the bf16 pooled tensors of gsa_pool_kv, qc32 / kc32 the fp32 ones.
 * n_split in [1, 64], n_split * K <= 2048.  With n_split == 1 and K <= 64 this
 * runs the fused tcgen05 kernel (scores from tf32 products of qc32 / kc32,
 * the list of each row being its exact top-K); otherwise warp-level bf16
 * attention from qc / kc and an fp32 scorer over the slices -- an inspection
 * path for per-slice candidate lists, many times slower at large N.  For
 * 64 < K <= 128 gsa_forward ranks on the tensor cores in two passes (see
 * gsa_forward_timed) and is the path to use.  Blocks below B0 are never
 * candidates.
 */
gsa_status gsa_compressed_attn(const gsa_shape* shape, const gsa_bf16* qc, const gsa_bf16* kc,
                               const gsa_bf16* vc, const float* qc32, const float* kc32,
                               float* oc, float* cand_score, int32_t* cand_idx, int32_t n_split,
                               void* ws, void* stream);

/*
 * Debug output of steps 2-3: the fused kernel's own unscaled compressed
 * logits, the values its streaming top-K ranks (S_guide = scale * logit;
 * it page, section 2), for the compressed query rows [row0, row0 + n_rows):
 *   logits [H][n_rows][Tc] fp32: tf32 tensor-core products qc32[a,h] . kc32[c,h]
 *   for every compressed entry c (special entries included).
 * qc32 / kc32 / vc as for gsa_compressed_attn (vc is only mapped, not read).
 * Runs only the CTAs of the rows asked for; their ranking pass writes nothing
 * else.  0 <= row0, n_rows >= 1, row0 + n_rows <= Tc, else GSA_ERR_INVALID_ARG.
 * With the same inputs the values equal those gsa_forward ranks, so a test
 * can check that its selection is the exact top-K of these logits.
 */
gsa_status gsa_guide_logits(const gsa_shape* shape, const float* qc32, const float* kc32,
                            const gsa_bf16* vc, int64_t row0, int32_t n_rows, float* logits, void* ws,
                            void* stream);

/*
 * Step 4, Top-K block selection (technical summary 2.1, selection branch:
 * the K most relevant token regions per query by the compressed scores).
 * Merges the n_split candidate lists of gsa_compressed_attn into
 *   sel [H][Tc][K] int32: the K_eff blocks with the largest score (ties go to
 *   the lower block id), in ascending id order, padded with -1.
 */
gsa_status gsa_topk_blocks(const gsa_shape* shape, const float* cand_score,
                           const int32_t* cand_idx, int32_t n_split, int32_t* sel, void* ws,
                           void* stream);

/*
 * Step 5, selected attention (technical summary 2.1, selection branch;
 * 2.2, Speed3R-VGGT keeps the reference-frame / camera tokens).  For token t
 * in compressed entry a and head h: one softmax over the valid tokens of the
 * blocks sel[h][a][:] plus the NK always-kept tokens (ks/vs from gsa_pool_kv,
 * NULL when NK == 0):
 *   o_sel [T][H][64] bf16, and lse [T][H] fp32 = log sum exp of the scaled
 *   logits (may be NULL).
 * Runs on tcgen05, one (entry, head) pair at a time with the entry's queries
 * as the N = 16 side; this stage call streams the NK always-kept keys for
 * every pair as well, whereas gsa_forward computes that segment once for all
 * tokens on the M = 128 attention kernel and passes its softmax state on.
 * An id outside [0, NB) ends the pair's list and sets the device-check bit.
 */
gsa_status gsa_selected_attn(const gsa_shape* shape, const gsa_bf16* q, const gsa_bf16* k,
                             const gsa_bf16* v, const gsa_bf16* ks, const gsa_bf16* vs,
                             const int32_t* sel, gsa_bf16* o_sel, float* lse, void* ws,
                             void* stream);

/*
 * Step 6, gated aggregation and nearest up-sampling (technical summary 2.1:
 * a learnable sigmoid gate computed from the query mixes the two branches).
 *   g[a,h] = sigmoid(qc32[a,h] . w[h]),  w [H][64] fp32
 *   out[t,h] = g * oc[a(t),h] + (1 - g) * o_sel[t,h]   -> out [T][H][64] bf16
 */
gsa_status gsa_gate_combine(const gsa_shape* shape, const float* qc32, const float* w,
                            const float* oc, const gsa_bf16* o_sel, gsa_bf16* out, void* ws,
                            void* stream);

/*
 * Dense global attention (technical summary 1: the quadratic all-to-all
 * attention GSA replaces): out = softmax(scale * q k^T) v over all T tokens,
 * per head, on tcgen05/TMEM fed by TMA.  Uses n_frames, n_special, hp, wp,
 * n_heads, head_dim, scale.  A wait that runs out of time sets GSA_ERR_TIMEOUT
 * in the workspace's error word (see gsa_check_device_error).
 */
gsa_status dense_global_attn(const gsa_shape* shape, const gsa_bf16* q, const gsa_bf16* k,
                             const gsa_bf16* v, gsa_bf16* out, void* ws, void* stream);

/*
 * Frame attention ("AVGGT: Rethinking Global Attention for Accelerating
 * VGGT", section 2.2: the early global layers of VGGT converted to attention
 * within each frame, O((NL)^2) -> O(N L^2)): every token attends only to the
 * S + Hp*Wp tokens of its own frame.  out = softmax(scale * q k_f^T) v_f per
 * frame f and head; same layouts, ownership and errors as dense_global_attn.
 */
gsa_status frame_attn(const gsa_shape* shape, const gsa_bf16* q, const gsa_bf16* k,
                      const gsa_bf16* v, gsa_bf16* out, void* ws, void* stream);

/*
 * Subsampled global attention ("AVGGT: Rethinking Global Attention for
 * Accelerating VGGT", section 2.2, SGA).  Every query t attends, in one
 * softmax (scale from `shape`), to
 *   - every special token,
 *   - the patch at the top-left of every sub_h x sub_w window of every frame
 *     (rows 0, sub_h, 2 sub_h, ... and columns 0, sub_w, ... of the grid),
 *   - its own key/value when it is not one of those (the diagonal),
 *   - one extra key/value pair: the means of the keys and of the values of
 *     all patch tokens not sampled (absent when none is dropped), taken as a
 *     single ordinary key.
 * Uses n_frames, n_special, hp, wp, n_heads, head_dim, scale of `shape`;
 * q, k, v, out [T][H][64] bf16.  sub_h, sub_w >= 1 (1 x 1 is dense
 * attention).  `ws` (ws_bytes >= sga_workspace_size) holds the head-major
 * copies of the kept keys, the dropped-token means and the fp32 softmax over
 * the kept keys; its first word is the device error word as for every call.
 * Returns GSA_ERR_WORKSPACE when ws_bytes is too small.
 */
gsa_status sga_workspace_size(const gsa_shape* shape, int32_t sub_h, int32_t sub_w, size_t* bytes);
gsa_status sga_attn(const gsa_shape* shape, int32_t sub_h, int32_t sub_w, const gsa_bf16* q,
                    const gsa_bf16* k, const gsa_bf16* v, gsa_bf16* out, void* ws, size_t ws_bytes,
                    void* stream);

/*
 * dense_global_attn on the warp-level tensor-core instruction (mma.sync
 * m16n8k16), the pre-tcgen05 path; kept as a measured baseline for the
 * tcgen05 kernel.  Same arguments and result.
 */
gsa_status dense_global_attn_mma(const gsa_shape* shape, const gsa_bf16* q, const gsa_bf16* k,
                                 const gsa_bf16* v, gsa_bf16* out, void* ws, void* stream);

/*
 * The whole GSA layer: steps 1-6 enqueued on `stream`, intermediates in `ws`
 * (ws_bytes >= gsa_workspace_size); K up to 128 (see gsa_forward_timed for
 * how K > 64 is ranked).  w [H][64] fp32 gate vectors; out
 * [T][H][64] bf16.  The attention over the always-kept tokens runs on the
 * tensor-core attention kernel into the workspace; the selected blocks
 * continue that softmax in the step-5 kernel, which also applies the gate.
 */
gsa_status gsa_forward(const gsa_shape* shape, const gsa_bf16* q, const gsa_bf16* k,
                       const gsa_bf16* v, const float* w, gsa_bf16* out, void* ws,
                       size_t ws_bytes, void* stream);

/*
 * gsa_forward with per-kernel timing: `events` is NULL or GSA_FORWARD_STEPS + 1
 * cudaEvent_t handles created by the caller; events[0] is recorded on `stream`
 * before the first kernel and events[i+1] after step i, the steps being
 *   0 pooling, 1 compressed attention, 2 S_guide block scores with the
 *   streaming top-K, 3 top-K merge and the ordering of the selection branch's
 *   work, 4 attention of every token over the always-kept tokens, 5 attention
 *   over the selected blocks, merged with step 4, with the gate.
 * For K <= 64 steps 1-2 are one fused kernel (step 1's interval holds it) and
 * step 3 sorts the (head, entry) pairs by the grid position of their
 * best-scoring block, so that pairs whose selections cover the same region of
 * every frame run together and share K/V blocks in L2.
 * For 64 < K <= 128 step 1 is the fused kernel ranking the top 64 (and
 * recording each row's 64th-best (score, entry) key), step 2 a second,
 * ranking-only pass of it for the next K - 64 pairs strictly below that key,
 * and step 3 the ascending union of the two selections and the ordering
 * (Speed3R technical summary 4: a larger Top-K at test time).
 * A step fused into another one (or absent, such as step 4 when NK == 0)
 * records an empty interval.  If `n_launched` is not NULL it receives
 * the number of kernels enqueued.
 */
#define GSA_FORWARD_STEPS 6
gsa_status gsa_forward_timed(const gsa_shape* shape, const gsa_bf16* q, const gsa_bf16* k,
                             const gsa_bf16* v, const float* w, gsa_bf16* out, void* ws,
                             size_t ws_bytes, void* const* events, int32_t* n_launched,
                             void* stream);

/* Byte offsets of gsa_forward's intermediates inside its workspace (host only),
 * for inspecting them after a call: the buffers of gsa_pool_kv (qc32, kc32, vc,
 * qc, kc, ks, vs), oc, the candidates (n_split lists per row), sel, the
 * always-kept segment's fp32 output [T][H][64] and lse [T][H] (empty when
 * NK == 0), and the ordering of the selection branch's work: best [H][Tc]
 * int32, each row's best-scoring block (-1 when it has none), and order
 * [H*Tc] int32, the pairs h*Tc + a sorted by (h, best mod Bh*Bw). */
typedef struct {
  size_t qc32, kc32, vc, qc, kc, ks, vs, oc, cand_score, cand_idx, sel, o_spec, lse_spec, total;
  int32_t n_split;
  size_t best, order;
} gsa_ws_offsets;
gsa_status gsa_workspace_offsets(const gsa_shape* shape, gsa_ws_offsets* out);

/*
 * gsa_forward without a workspace argument, for callers that cannot allocate
 * device memory.  (The Speed3R pages have no counterpart: this is a deployment
 * variant of gsa_forward.)  Some host programs may not call cudaMalloc at all:
 * applications whose own memory manager owns every byte of device memory and
 * forbids allocations it does not make, or latency-critical loops where a
 * cudaMalloc/cudaFree would synchronise the device.  Such callers still pass
 * q, k, v, w and out, which they own; the layer's intermediates go to one
 * fixed array of GSA_NOALLOC_SCRATCH_BYTES in the library's device memory,
 * which every GPU that loads the library holds until the process exits.
 *
 * - Shapes whose gsa_workspace_size exceeds GSA_NOALLOC_SCRATCH_BYTES are
 *   rejected with GSA_ERR_SCRATCH_LIMIT before any work is enqueued (the
 *   32 MiB array fits the VGGT token layout up to 4 frames: 4 x (5 + 37x37)
 *   tokens, 16 heads, K = 16).
 * - The first call on each device looks up the array's device address (with
 *   that device current) and caches it; make that first call before any
 *   stream capture.
 * - Every call on a device shares the one array and leaves its intermediates
 *   in it.  Each call zeroes the array's error-word header first.  Calls that
 *   overlap on the GPU (on different streams, or from several host threads
 *   without ordering) race on the array and corrupt each other's results:
 *   order them.
 * - Allocates nothing: no cudaMalloc / cudaFree and no allocating library call.
 * - In-kernel failures (a bounded wait that ran out, a selection id out of
 *   range) set bits in the array's error word, as they do in a workspace's;
 *   read them with gsa_noalloc_check_device_error before the next no-alloc
 *   call on the device, which zeroes the word again.
 */
#define GSA_NOALLOC_SCRATCH_BYTES (32u << 20)
gsa_status gsa_forward_noalloc(const gsa_shape* shape, const gsa_bf16* q, const gsa_bf16* k,
                               const gsa_bf16* v, const float* w, gsa_bf16* out, void* stream);

/* gsa_check_device_error for gsa_forward_noalloc: synchronise `stream`, read
 * and clear the error word of the fixed array on the current device, and
 * return GSA_OK, GSA_ERR_TIMEOUT or GSA_ERR_DEVICE_CHECK (GSA_ERR_CUDA if the
 * array's address cannot be looked up).  Allocates nothing. */
gsa_status gsa_noalloc_check_device_error(void* stream);

/* Synchronise `stream`, read the device error word in `ws`, clear it, and
 * return GSA_OK, GSA_ERR_TIMEOUT or GSA_ERR_DEVICE_CHECK.  For diagnosis, the
 * header's words 1 and 2 record the first in-kernel wait that ran out (its
 * barrier's shared-memory address | 1, and threadIdx.x << 8 | phase parity);
 * they are cleared with the error word. */
gsa_status gsa_check_device_error(void* ws, void* stream);

/* Self-test of the exponential the attention kernels' softmax takes on the
 * FMA pipe for a quarter of its terms (2^x by range reduction and a cubic, a
 * relative error below 7.5e-5 on [-125, 0], the clamp at -125 included):
 *   y[i] = that 2^x[i] for i < n, computed on the device as the softmax does
 *   (two lanes per instruction).
 * x, y: device float arrays of n elements (y written, x read), launched on
 * `stream`; GSA_ERR_INVALID_ARG for n < 0 or a NULL array with n > 0.  Not part of the
 * attention path: for tests that compare it with the exact 2^x. */
gsa_status gsa_selftest_exp2(const float* x, float* y, int64_t n, void* stream);

/* Static text for a status code. */
const char* gsa_status_string(gsa_status status);

/* What a GSA_ERR_CUDA was: the CUDA runtime's last error in the calling host
 * thread (cudaPeekAtLastError: not cleared; a fault of a kernel stays set for
 * the context) and the static name of a CUDA error code. */
int32_t gsa_last_cuda_error(void);
const char* gsa_cuda_error_name(int32_t code);

#ifdef __cplusplus
}
#endif

#endif /* GSA_H_ */
