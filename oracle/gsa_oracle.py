"""CPU oracle for sparse global attention over N views (GSA) and dense global attention.

TEST INFRASTRUCTURE ONLY.  Only the tests, the package entry's ``smoke()``
check and the ``cpu_baseline`` / ``--impl reference`` legs of the benchmark
may import this module.  The CUDA library never calls it and shares no code
with it; both are fed from the seeded generators in ``synthetic``.

Everything is computed in float64 from the exact values of the bf16 inputs,
step by step in the order the Speed3R pages give the method:

  "Speed3R: Sparse Feed-forward 3D Reconstruction Models" (gist.science, ja
  and it), technical summary, section 2.1 "Dual-branch attention mechanism"
  (ja) / section 2 "Methodology" (it):
    1. compression branch -- spatial down-sampling of the tokens (e.g. 4x4
       average pooling), attention in the compressed space, the result
       up-sampled back to the original resolution;
    2. the compressed branch's scores (S_guide, it page) pick, for every
       query, the Top-K most relevant token regions;
    3. selection branch -- fine-grained attention over only the selected
       key/value regions;
    4. gated aggregation -- a learnable sigmoid gate computed from the query
       mixes the two branch outputs;
  plus the Speed3R-VGGT adaptation (section 2.2: the selection branch is made
  to retain the reference frame and the camera tokens at all times) and the
  dense global attention the module replaces (section 1, background).

Where the pages are silent, the readings used here are:
  * queries, keys and values are all pooled in the compression branch; the
    up-sampling is nearest (each fine token takes its block's output);
  * special tokens are singleton entries of the compressed sequence (they
    are not pooled), take part in compressed attention as queries and keys,
    and are not top-K candidates;
  * the always-kept set of the selection branch is, by default ("specials"),
    every special token of every frame; the "reference" reading of the
    Speed3R-VGGT adaptation keeps instead the whole reference frame (frame
    0: its specials and patches) plus the camera token (special slot 0) of
    every other frame, and frame 0's blocks are then not top-K candidates
    (they are attended to already); the register tokens (slots >= 1) of
    frames 1..N-1 then take part in the compression branch only;
  * the score ranked by top-K is the scaled logit (q_mean . k_mean) / sqrt(D);
    selection is per head and per query block; ties go to the lower block id;
    K_eff = min(K, number of candidate blocks), which is 0 for one frame in
    the "reference" reading;
  * a selected partial edge block contributes only its valid tokens;
  * one softmax scale 1/sqrt(D) for every attention;
  * the gate is g = sigmoid(q_mean . w_h) per (query block, head); g weights
    the compression branch and (1 - g) the selection branch.
The other readings of two of these points are available as variants of
``gsa_layer``: fine queries against the pooled keys in the compression
branch (``queries="fine"``) and a gate per fine token (``gate_per="token"``).

Inputs are torch tensors (bf16 or fp32, CPU) or NumPy arrays of shape
[T, H, D]; they are read in slices and converted exactly to float64, so the
full-size workloads never need a float64 copy of the whole tensor.
"""

from __future__ import annotations

import contextlib
import dataclasses
import functools
import math

import numpy as np
import torch


# ----------------------------------------------------------------------------
# sizes at which the same arithmetic switches to a chunked or threaded form


@dataclasses.dataclass(frozen=True)
class Chunking:
    """Where the oracle splits work to bound host memory or to use every core.

    None of these changes what is computed, only in which pieces: each form
    is pinned against the unsplit one and against a library routine or the
    brute force by forcing tiny values (``chunking``).

    softmax_torch_elems  arrays of at least this many elements go through
                         float64 torch ops (multi-threaded) instead of NumPy
    pool_frames          frames pooled per slice of the input
    layer_chunk_elems    compressed logits [entries, H, Tc] formed at once
    dense_key_chunk      longer sequences take dense attention's two-pass
                         form over key slices of this many tokens
    dense_max_bytes      bytes of logits of one key slice (row chunking)
    sga_mean_tokens      dropped tokens summed per slice for SGA's mean pair
    sga_row_elems        logits [rows, H, keys] SGA forms at once
    """

    softmax_torch_elems: int = 1 << 20
    pool_frames: int = 32
    layer_chunk_elems: int = 50_000_000
    dense_key_chunk: int = 1 << 14
    dense_max_bytes: int = 1 << 30
    sga_mean_tokens: int = 1 << 16
    sga_row_elems: int = 1 << 27


CHUNKS = Chunking()


def spans(n: int, step: int) -> list[tuple[int, int]]:
    """(start, stop) of the consecutive slices of range(n), ``step`` long; the
    last one may be shorter."""
    step = max(1, int(step))
    return [(i, min(n, i + step)) for i in range(0, n, step)]


@contextlib.contextmanager
def chunking(**sizes):
    """Temporarily use other split sizes (tests force every split form with
    tiny values)."""
    global CHUNKS
    old = CHUNKS
    CHUNKS = dataclasses.replace(old, **sizes)
    try:
        yield CHUNKS
    finally:
        CHUNKS = old


# ----------------------------------------------------------------------------
# token geometry


@dataclasses.dataclass(frozen=True)
class Geometry:
    """Sizes of one layer call.

    Frame f holds ``S`` special tokens then ``Hp*Wp`` patch tokens (row-major).
    Pooling with factor ``P`` cuts each frame's patch grid into
    ``Bh x Bw`` blocks (``Bh = ceil(Hp/P)``); a block at the right or bottom
    edge holds only the patches that exist.  The compressed sequence has, per
    frame, the ``S`` specials followed by the ``Bh*Bw`` blocks (row-major), so
    entry ``a`` of frame f is ``f*E + j`` with ``E = S + Bh*Bw``.  Patch block
    ``beta`` (a top-K candidate id) of frame f, grid position (br, bc), is
    ``f*Bh*Bw + br*Bw + bc``.
    """

    N: int
    S: int
    Hp: int
    Wp: int
    H: int
    D: int
    P: int
    K: int
    scale: float | None = None
    keep: str = "specials"  # "specials" | "reference"

    @property
    def L(self) -> int:
        return self.S + self.Hp * self.Wp

    @property
    def T(self) -> int:
        return self.N * self.L

    @property
    def Bh(self) -> int:
        return -(-self.Hp // self.P)

    @property
    def Bw(self) -> int:
        return -(-self.Wp // self.P)

    @property
    def Bf(self) -> int:
        return self.Bh * self.Bw

    @property
    def E(self) -> int:
        return self.S + self.Bf

    @property
    def Tc(self) -> int:
        return self.N * self.E

    @property
    def NB(self) -> int:
        return self.N * self.Bf

    @property
    def B0(self) -> int:
        """First top-K candidate block: frame 0's blocks are excluded when
        frame 0 is kept whole."""
        return self.Bf if self.keep == "reference" else 0

    @property
    def K_eff(self) -> int:
        return min(self.K, self.NB - self.B0)

    @property
    def sm_scale(self) -> float:
        return 1.0 / math.sqrt(self.D) if self.scale is None else float(self.scale)

    @property
    def NS(self) -> int:
        return self.N * self.S

    # --- index maps -------------------------------------------------------

    def special_token(self, f: int, j: int) -> int:
        return f * self.L + j

    def patch_token(self, f: int, r: int, c: int) -> int:
        return f * self.L + self.S + r * self.Wp + c

    def block_rows_cols(self, br: int, bc: int) -> tuple[range, range]:
        return (range(self.P * br, min(self.P * br + self.P, self.Hp)),
                range(self.P * bc, min(self.P * bc + self.P, self.Wp)))

    def block_tokens(self, beta: int) -> np.ndarray:
        """Valid token ids of patch block ``beta``."""
        f, j = divmod(int(beta), self.Bf)
        br, bc = divmod(j, self.Bw)
        rows, cols = self.block_rows_cols(br, bc)
        # patch_token(f, r, c) for r in rows, c in cols (row-major)
        r = np.arange(rows.start, rows.stop, dtype=np.int64)
        c = np.arange(cols.start, cols.stop, dtype=np.int64)
        return (f * self.L + self.S + r[:, None] * self.Wp + c[None, :]).ravel()

    def entry_of_block(self, beta: int) -> int:
        f, j = divmod(int(beta), self.Bf)
        return f * self.E + self.S + j

    def entry_of_token(self, t: int) -> int:
        f, i = divmod(int(t), self.L)
        if i < self.S:
            return f * self.E + i
        r, c = divmod(i - self.S, self.Wp)
        return f * self.E + self.S + (r // self.P) * self.Bw + (c // self.P)

    def tokens_of_entry(self, a: int) -> np.ndarray:
        f, j = divmod(int(a), self.E)
        if j < self.S:
            return np.array([self.special_token(f, j)], dtype=np.int64)
        return self.block_tokens(f * self.Bf + (j - self.S))

    def special_tokens(self) -> np.ndarray:
        return _special_tokens(self)

    def kept_tokens(self) -> np.ndarray:
        """Token ids the selection branch always attends to, each listed once."""
        return _kept_tokens(self)

    def patch_block_entries(self) -> np.ndarray:
        """Compressed-sequence index of every patch block, in block-id order
        (entry_of_block over all ids)."""
        beta = np.arange(self.NB, dtype=np.int64)
        return (beta // self.Bf) * self.E + self.S + beta % self.Bf


@functools.lru_cache(maxsize=64)
def _special_tokens(geo: Geometry) -> np.ndarray:
    ids = np.array([geo.special_token(f, j) for f in range(geo.N) for j in range(geo.S)], dtype=np.int64)
    ids.flags.writeable = False
    return ids


@functools.lru_cache(maxsize=64)
def _kept_tokens(geo: Geometry) -> np.ndarray:
    if geo.keep == "specials":
        return _special_tokens(geo)
    assert geo.keep == "reference", geo.keep
    frame0 = list(range(geo.L))
    cameras = [geo.special_token(f, 0) for f in range(1, geo.N)] if geo.S > 0 else []
    ids = np.array(frame0 + cameras, dtype=np.int64)
    ids.flags.writeable = False
    return ids


def geometry_of(workload, **overrides) -> Geometry:
    """Geometry of a ``synthetic.Workload`` (fields copied by name)."""
    g = Geometry(N=workload.n_frames, S=workload.n_special, Hp=workload.hp, Wp=workload.wp,
                 H=workload.n_heads, D=workload.head_dim, P=workload.pool, K=workload.top_k,
                 keep="reference" if getattr(workload, "keep", 0) == 1 else "specials")
    return dataclasses.replace(g, **overrides) if overrides else g


# ----------------------------------------------------------------------------
# exact float64 views of the inputs


def f64(x, rows=None) -> np.ndarray:
    """Exact float64 copy of ``x`` or of ``x[rows]`` (bf16/fp32 -> fp64 is exact)."""
    if isinstance(x, torch.Tensor):
        if rows is None:
            t = x
        elif isinstance(rows, slice):
            t = x[rows]
        else:
            t = x[torch.as_tensor(np.array(rows, dtype=np.int64))]
        return t.to(torch.float64).numpy()
    a = np.asarray(x)
    return (a if rows is None else a[rows]).astype(np.float64)


def f64_head_all(x, h: int) -> np.ndarray:
    """Exact float64 copy of head h of every row of ``x``: [rows, D]."""
    if isinstance(x, torch.Tensor):
        return x[:, h].to(torch.float64).numpy()
    return np.asarray(x)[:, h].astype(np.float64)


def f64_head(x, rows, h: int) -> np.ndarray:
    """Exact float64 copy of ``x[rows, h]``: [len(rows), D]."""
    if isinstance(x, torch.Tensor):
        return x[torch.as_tensor(np.array(rows, dtype=np.int64)), h].to(torch.float64).numpy()
    return np.asarray(x)[np.asarray(rows), h].astype(np.float64)


def softmax(z: np.ndarray, axis: int = -1) -> np.ndarray:
    """Textbook softmax, shifted by the maximum for range (exact in real
    arithmetic).  Arrays of ``CHUNKS.softmax_torch_elems`` elements or more go
    through float64 torch CPU ops, which use every core; smaller ones stay in
    NumPy (a torch call costs more than the arithmetic there)."""
    z = np.asarray(z, dtype=np.float64)
    if z.size < CHUNKS.softmax_torch_elems:
        m = np.max(z, axis=axis, keepdims=True)
        e = np.exp(z - m)
        return e / np.sum(e, axis=axis, keepdims=True)
    t = torch.from_numpy(z)
    m = torch.amax(t, dim=axis, keepdim=True)
    e = torch.exp(t - m)
    return (e / torch.sum(e, dim=axis, keepdim=True)).numpy()


# ----------------------------------------------------------------------------
# step 1: compression by spatial average pooling


def pool(geo: Geometry, X, frames_per_chunk: int | None = None) -> np.ndarray:
    """Compressed sequence of X: [Tc, H, D] float64.

    Speed3R, technical summary 2.1, compression branch: the tokens are
    down-sampled spatially, e.g. by 4x4 average pooling, into a coarse
    context.  Each patch block's entry is the arithmetic mean over the
    patches the block actually holds (fewer than P*P at the right/bottom
    edges); each special token is copied as its own entry.  The input is
    read ``frames_per_chunk`` frames at a time (``CHUNKS.pool_frames``).
    """
    if frames_per_chunk is None:
        frames_per_chunk = CHUNKS.pool_frames
    out = np.full((geo.Tc, geo.H, geo.D), np.nan)  # NaN marks anything left unwritten
    for f0, f1 in spans(geo.N, frames_per_chunk):
        x = f64(X, slice(f0 * geo.L, f1 * geo.L)).reshape(f1 - f0, geo.L, geo.H, geo.D)
        spec = x[:, :geo.S]
        grid = x[:, geo.S:].reshape(f1 - f0, geo.Hp, geo.Wp, geo.H, geo.D)
        ent = out[f0 * geo.E:f1 * geo.E].reshape(f1 - f0, geo.E, geo.H, geo.D)
        ent[:, :geo.S] = spec
        for br in range(geo.Bh):
            for bc in range(geo.Bw):
                rows, cols = geo.block_rows_cols(br, bc)
                cell = grid[:, rows.start:rows.stop, cols.start:cols.stop]
                ent[:, geo.S + br * geo.Bw + bc] = cell.sum(axis=(1, 2)) / (len(rows) * len(cols))
    return out


# ----------------------------------------------------------------------------
# step 2: attention in the compressed space; step 3: S_guide; step 4: top-K


def heads_first(x: np.ndarray) -> np.ndarray:
    """[n, H, D] -> contiguous [H, n, D] (so per-head products are plain matmuls)."""
    return np.ascontiguousarray(np.asarray(x).transpose(1, 0, 2))


def qk_logits(q: np.ndarray, k: np.ndarray, scale: float) -> np.ndarray:
    """(q . k) * scale for every query row and key row, per head: [rows, H, keys]."""
    s = np.matmul(heads_first(q), heads_first(k).transpose(0, 2, 1)) * scale  # [H, rows, keys]
    return s.transpose(1, 0, 2)


def weighted_values(p: np.ndarray, v: np.ndarray) -> np.ndarray:
    """sum_j p[r, h, j] v[j, h, :]: [rows, H, D]."""
    o = np.matmul(heads_first(p), heads_first(v))  # [H, rows, D]
    return o.transpose(1, 0, 2)


def compressed_logits(geo: Geometry, Qc_rows: np.ndarray, Kc: np.ndarray) -> np.ndarray:
    """Scaled logits of compressed queries against every compressed key: [rows, H, Tc]."""
    return qk_logits(Qc_rows, Kc, geo.sm_scale)


def compressed_attention(geo: Geometry, Qc_rows: np.ndarray, Kc: np.ndarray, Vc: np.ndarray):
    """O_cmp for the given compressed queries, and their logits.

    Speed3R, technical summary 2.1: attention computed in the compressed
    space (every compressed entry, specials included, is a key).
    Returns (O [rows, H, D], logits [rows, H, Tc]).
    """
    s = compressed_logits(geo, Qc_rows, Kc)
    p = softmax(s, axis=-1)
    return weighted_values(p, Vc), s


def guide_scores(geo: Geometry, logits: np.ndarray) -> np.ndarray:
    """S_guide: the compressed logits restricted to patch-block keys, [rows, H, NB].

    Speed3R (it), technical summary 2, compression branch: the branch
    produces a score matrix S_guide that identifies the most relevant regions.
    Column beta is patch block beta; special entries are not candidates.
    """
    idx = torch.from_numpy(geo.patch_block_entries())
    return torch.from_numpy(logits).index_select(-1, idx).numpy()


def largest_values(x: np.ndarray, k: int) -> np.ndarray:
    """The k largest values along the last axis, in descending order:
    [..., k] (torch.topk as the selection routine; only values are used, so
    its order among equal values does not matter)."""
    return torch.topk(torch.from_numpy(x), k, dim=-1, sorted=True).values.numpy()


def top_k_blocks(geo: Geometry, guide: np.ndarray) -> np.ndarray:
    """Top-K patch blocks per (query, head): [rows, H, K] ascending ids, -1 pad.

    Speed3R, technical summary 2.1, selection branch: the K most relevant
    token regions for each query by the compressed branch's scores.  The
    candidates are the blocks beta >= B0; they are ranked by (-score, block
    id), so equal scores go to the lower id; the first K_eff are kept.  (The
    candidates are first narrowed to the blocks scoring at least the K-th
    largest score, which cannot change the ranking's first K_eff entries.)
    """
    rows, H, NB = guide.shape
    k = geo.K_eff
    sel = np.full((rows, H, geo.K), -1, dtype=np.int64)
    if k == 0:
        return sel
    cg = guide[..., geo.B0:]
    kth = largest_values(cg, k)[..., k - 1]
    # every (row, head) has at least k candidates (those tied at the threshold too)
    r, h, c = np.nonzero(cg >= kth[..., None])
    # rank within each (row, head) by score descending, then block id ascending
    order = np.lexsort((c, -cg[r, h, c], h, r))
    r, h, c = r[order], h[order], c[order]
    first = np.ones(r.size, dtype=bool)
    first[1:] = (r[1:] != r[:-1]) | (h[1:] != h[:-1])
    start = np.flatnonzero(first)
    rank = np.arange(r.size) - np.repeat(start, np.diff(np.append(start, r.size)))
    chosen = (geo.B0 + c[rank < k]).reshape(rows, H, k)
    sel[..., :k] = np.sort(chosen, axis=-1)
    return sel


def top_k_gap(geo: Geometry, guide: np.ndarray) -> np.ndarray:
    """s_(K) - s_(K+1) per (query, head), the K-th minus the (K+1)-th largest
    score among the candidate blocks (inf when every candidate is selected)."""
    cg = guide[..., geo.B0:]
    if geo.K_eff >= cg.shape[-1]:
        return np.full(guide.shape[:-1], np.inf)
    k = geo.K_eff
    top = largest_values(cg, k + 1)
    return top[..., k - 1] - top[..., k]


# ----------------------------------------------------------------------------
# step 5: selected (fine) attention


def selected_keys(geo: Geometry, sel_row: np.ndarray) -> np.ndarray:
    """Token ids of the selected regions for one (query block, head): the valid
    tokens of the selected blocks.

    Speed3R, technical summary 2.1 (selection branch: fine-grained attention on
    only the selected key/value regions).
    """
    parts = [geo.block_tokens(b) for b in sel_row if b >= 0]
    return np.concatenate(parts) if parts else np.zeros(0, dtype=np.int64)


def selected_attention(geo: Geometry, Q, K, V, sel: np.ndarray, rows: np.ndarray,
                       entries: np.ndarray) -> np.ndarray:
    """O_sel for fine query tokens ``rows``: [len(rows), H, D].

    ``sel`` is [len(entries), H, K] (the top-K of each compressed entry) and
    row t uses the selection of its own entry (its query block).  The key set
    is selected_keys() plus the always-kept tokens (``Geometry.kept_tokens``;
    Speed3R technical summary 2.2, Speed3R-VGGT keeps the reference-frame /
    camera-token information in the selection branch), and one softmax runs
    over all of it.  The kept keys are the same for every query, so their
    logits are computed once for all rows.
    """
    pos = {int(a): i for i, a in enumerate(entries)}
    rows = np.asarray(rows, dtype=np.int64)
    out = np.full((rows.size, geo.H, geo.D), np.nan)
    q_all = f64(Q, rows)
    kept = geo.kept_tokens()
    k_kept, v_kept = f64(K, kept), f64(V, kept)  # [NK, H, D]
    s_kept = qk_logits(q_all, k_kept, geo.sm_scale)  # [rows, H, NK]
    by_entry: dict[int, list[int]] = {}
    for i, t in enumerate(rows):
        by_entry.setdefault(geo.entry_of_token(int(t)), []).append(i)
    for h in range(geo.H):
        k_h, v_h = f64_head_all(K, h), f64_head_all(V, h)  # [T, D] each
        for a, idx in by_entry.items():
            keys = selected_keys(geo, sel[pos[a], h])
            k, v = k_h[keys], v_h[keys]
            s = np.concatenate([q_all[idx, h] @ k.T * geo.sm_scale, s_kept[idx, h]], axis=-1)
            p = softmax(s, axis=-1)
            out[idx, h] = p[:, :keys.size] @ v + p[:, keys.size:] @ v_kept[:, h]
    return out


# ----------------------------------------------------------------------------
# step 6: gate and nearest up-sampling


def gate(geo: Geometry, Qc_rows: np.ndarray, w) -> np.ndarray:
    """g = sigmoid(q_mean . w_h) per (compressed entry, head): [rows, H].

    Speed3R, technical summary 2.1, gated aggregation: a learnable sigmoid
    gate computed from the query weights the two branch outputs.
    """
    wv = f64(w)
    z = np.sum(Qc_rows * wv[None], axis=-1)
    with np.errstate(over="ignore"):  # exp(-z) = inf gives g = 0 exactly
        return 1.0 / (1.0 + np.exp(-z))


def combine(g_rows: np.ndarray, o_cmp_up: np.ndarray, o_sel: np.ndarray) -> np.ndarray:
    """out = g * up(O_cmp) + (1 - g) * O_sel (g broadcast over D)."""
    return g_rows[..., None] * o_cmp_up + (1.0 - g_rows[..., None]) * o_sel


# ----------------------------------------------------------------------------
# the whole layer


def compressed_attention_fine(geo: Geometry, Q, Kc: np.ndarray, Vc: np.ndarray, rows) -> np.ndarray:
    """Reading A1 of the compression branch, as a variant: each fine query
    attends to the pooled keys and values (no pooling of the queries, so no
    up-sampling of the output).  [len(rows), H, D]."""
    q = f64(Q, np.asarray(rows, dtype=np.int64))
    return weighted_values(softmax(qk_logits(q, Kc, geo.sm_scale), axis=-1), Vc)


def gate_token(geo: Geometry, Q, rows, w) -> np.ndarray:
    """Reading A10 of the gate, as a variant: g = sigmoid(q_t . w_h) for every
    fine token t (the it page's per-token wording taken literally) instead of
    one gate per query block from the pooled query.  [len(rows), H]."""
    return gate(geo, f64(Q, np.asarray(rows, dtype=np.int64)), w)


def gsa_layer(geo: Geometry, Q, K, V, w, rows=None, sel_override=None,
              tie_window: float = 1e-3, chunk_elems: int | None = None, pooled=None,
              queries: str = "pooled", gate_per: str = "block") -> dict:
    """The GSA layer for fine query tokens ``rows`` (all tokens when None).

    Returns a dict of float64 arrays:
      rows, entries (compressed entries owning the rows), own (entry position of
      each row), o_cmp [entries,H,D], sel [entries,H,K] (the oracle's own
      top-K), gap [entries,H] (K-th minus (K+1)-th score), o_sel [rows,H,D],
      g [entries,H], out [rows,H,D], o_cmp_up [rows,H,D]; guide
      [entries,H,NB] and the pooled tensors qc, kc, vc when they are small.

    ``sel_override`` ([Tc, H, K] block ids, -1 pad) is another selection to
    evaluate the selection branch with.  It is checked against this oracle's
    S_guide scores: ``sel_exact`` [entries,H] says it equals the oracle's own
    top-K, ``sel_valid`` [entries,H] that it is a top-K up to ``tie_window``
    (no unchosen block beats a chosen one by ``tie_window`` or more).

    ``pooled`` = (pool(Q), pool(K), pool(V)) from an earlier call on the same
    inputs skips recomputing step 1.  ``queries="fine"`` and ``gate_per="token"``
    evaluate the variant readings A1 (fine queries against the pooled keys in
    the compression branch; the selection still ranks by the pooled scores)
    and A10 (a gate per fine token); the defaults are the readings the CUDA
    path implements.  Steps 2-4 run over the entries in
    chunks whose logits hold about ``chunk_elems`` values
    (``CHUNKS.layer_chunk_elems``).
    """
    if chunk_elems is None:
        chunk_elems = CHUNKS.layer_chunk_elems
    rows = np.arange(geo.T) if rows is None else np.asarray(rows, dtype=np.int64)
    if pooled is None:
        Qc, Kc, Vc = pool(geo, Q), pool(geo, K), pool(geo, V)
    else:
        Qc, Kc, Vc = pooled
    # the same [Tc, H, D] values, stored heads-first once, so that the per-chunk
    # heads_first() calls below are free
    Kc_keys = heads_first(Kc).transpose(1, 0, 2)
    Vc_keys = heads_first(Vc).transpose(1, 0, 2)
    entries = np.array(sorted({geo.entry_of_token(int(t)) for t in rows}), dtype=np.int64)
    nE = entries.size
    # NaN (or an id below -1) marks anything a chunk left unwritten
    o_cmp = np.full((nE, geo.H, geo.D), np.nan)
    sel = np.full((nE, geo.H, geo.K), -2, dtype=np.int64)
    gap = np.full((nE, geo.H), np.nan)
    keep_guide = nE * geo.NB * geo.H <= 50_000_000
    guide_all = np.full((nE, geo.H, geo.NB), np.nan) if keep_guide else None
    other = None
    if sel_override is not None:
        other = np.asarray(sel_override)[entries].astype(np.int64)
        sel_exact = np.zeros((nE, geo.H), dtype=bool)
        sel_valid = np.zeros((nE, geo.H), dtype=bool)
    step = max(1, chunk_elems // (geo.H * geo.Tc))
    for e0, e1 in spans(nE, step):
        o, logits = compressed_attention(geo, Qc[entries[e0:e1]], Kc_keys, Vc_keys)
        o_cmp[e0:e1] = o
        guide = guide_scores(geo, logits)
        sel[e0:e1] = top_k_blocks(geo, guide)
        gap[e0:e1] = top_k_gap(geo, guide)
        if keep_guide:
            guide_all[e0:e1] = guide
        if other is not None:
            sel_exact[e0:e1] = np.all(other[e0:e1] == sel[e0:e1], axis=-1)
            sel_valid[e0:e1] = selection_valid_top_k(geo, guide, other[e0:e1], tie_window)
    sel_used = sel if other is None else other
    o_sel = selected_attention(geo, Q, K, V, sel_used, rows, entries)
    g = gate(geo, Qc[entries], w)
    pos = {int(a): i for i, a in enumerate(entries)}
    own = np.array([pos[geo.entry_of_token(int(t))] for t in rows], dtype=np.int64)
    o_cmp_up = o_cmp[own] if queries == "pooled" else compressed_attention_fine(geo, Q, Kc_keys, Vc_keys, rows)
    g_rows = g[own] if gate_per == "block" else gate_token(geo, Q, rows, w)
    out = combine(g_rows, o_cmp_up, o_sel)
    res = dict(rows=rows, entries=entries, own=own, o_cmp=o_cmp, sel=sel, gap=gap,
               o_sel=o_sel, g=g, out=out, o_cmp_up=o_cmp_up, g_rows=g_rows)
    if other is not None:
        res.update(sel_exact=sel_exact, sel_valid=sel_valid)
    if keep_guide:
        res["guide"] = guide_all
    if geo.Tc * geo.H * geo.D <= 20_000_000:
        res.update(qc=Qc, kc=Kc, vc=Vc)
    return res


# ----------------------------------------------------------------------------
# dense global attention (the layer GSA replaces)


def dense_attention(geo: Geometry, Q, K, V, rows=None, key_chunk: int | None = None,
                    max_bytes: int | None = None) -> np.ndarray:
    """softmax(q K^T / sqrt(D)) V over all T tokens, for fine query ``rows``.

    Speed3R, technical summary 1 (Background): the dense global attention of
    DUSt3R / VGGT-style models, quadratic in the number of tokens.

    Up to ``key_chunk`` keys the whole score row is formed and passed to
    softmax().  Beyond that the same softmax is written out over key slices in
    two passes: the row maximum of the scaled logits over all keys first, then
    sum_j exp(s_j - max) v_j and sum_j exp(s_j - max), divided at the end --
    the textbook formula, without online rescaling.  Rows are taken in chunks
    whose logits of one key slice fit in ``max_bytes``.  (Defaults:
    ``CHUNKS.dense_key_chunk`` and ``CHUNKS.dense_max_bytes``.)
    """
    key_chunk = CHUNKS.dense_key_chunk if key_chunk is None else key_chunk
    max_bytes = CHUNKS.dense_max_bytes if max_bytes is None else max_bytes
    rows = np.arange(geo.T) if rows is None else np.asarray(rows, dtype=np.int64)
    out = np.full((rows.size, geo.H, geo.D), np.nan)
    if geo.T <= key_chunk:
        k_all, v_all = f64(K), f64(V)
        step = max(1, max_bytes // max(geo.H * geo.T * 8, 1))
        for r0, r1 in spans(rows.size, step):
            out[r0:r1] = weighted_values(softmax(qk_logits(f64(Q, rows[r0:r1]), k_all, geo.sm_scale)), v_all)
        return out
    step = max(1, max_bytes // (geo.H * key_chunk * 8))
    slices = [slice(t0, t1) for t0, t1 in spans(geo.T, key_chunk)]
    for r0, r1 in spans(rows.size, step):
        q = f64(Q, rows[r0:r1])
        m = torch.full((r1 - r0, geo.H), -np.inf, dtype=torch.float64)
        for sl in slices:
            s = torch.from_numpy(qk_logits(q, f64(K, sl), geo.sm_scale))
            m = torch.maximum(m, s.amax(dim=-1))
        num = np.zeros((r1 - r0, geo.H, geo.D))
        den = np.zeros((r1 - r0, geo.H))
        for sl in slices:
            s = torch.from_numpy(qk_logits(q, f64(K, sl), geo.sm_scale))
            e = torch.exp(s - m[..., None])
            den += e.sum(dim=-1).numpy()
            num += weighted_values(e.numpy(), f64(V, sl))
        out[r0:r1] = num / den[..., None]
    return out


def frame_attention(geo: Geometry, Q, K, V, rows=None) -> np.ndarray:
    """softmax(q K_f^T / sqrt(D)) V_f where K_f, V_f are the S + Hp*Wp tokens of
    the query's own frame f, for fine query ``rows``.

    "AVGGT: Rethinking Global Attention for Accelerating VGGT", section 2.2:
    the early global attention layers are converted to frame attention, which
    attends within each frame only.
    """
    rows = np.arange(geo.T) if rows is None else np.asarray(rows, dtype=np.int64)
    out = np.full((rows.size, geo.H, geo.D), np.nan)
    frame = rows // geo.L
    for f in np.unique(frame):
        idx = np.nonzero(frame == f)[0]
        keys = slice(int(f) * geo.L, (int(f) + 1) * geo.L)
        k, v = f64(K, keys), f64(V, keys)
        out[idx] = weighted_values(softmax(qk_logits(f64(Q, rows[idx]), k, geo.sm_scale)), v)
    return out


# ----------------------------------------------------------------------------
# AVGGT subsampled global attention (SGA)


def sga_sampled(geo: Geometry, sub_h: int, sub_w: int) -> np.ndarray:
    """Bool [Hp, Wp]: the patch positions whose keys and values SGA keeps.

    "AVGGT: Rethinking Global Attention for Accelerating VGGT", section 2.2
    (SGA): patch tokens are sampled uniformly on the 2D grid, one per
    sub_h x sub_w window; read here as the window's first (top-left) patch.
    """
    keep = np.zeros((geo.Hp, geo.Wp), dtype=bool)
    keep[::sub_h, ::sub_w] = True
    return keep


def sga_key_tokens(geo: Geometry, sub_h: int, sub_w: int) -> np.ndarray:
    """Token ids of the kept keys, frame by frame: the S specials (all kept),
    then the sampled patches row-major."""
    grid = np.flatnonzero(sga_sampled(geo, sub_h, sub_w).ravel())
    per = np.concatenate([np.arange(geo.S), geo.S + grid])
    return (np.arange(geo.N)[:, None] * geo.L + per[None, :]).ravel()


def sga_attention(geo: Geometry, Q, K, V, sub_h: int, sub_w: int, rows=None) -> np.ndarray:
    """SGA output for fine query ``rows``: [len(rows), H, D].

    AVGGT section 2.2: every query is kept; the keys/values are the special
    tokens plus the sampled patches; each token's own key/value (the diagonal)
    is kept as well, once; the dropped columns are replaced by a single pair
    (mean of the dropped keys, mean of the dropped values) -- read here as one
    more ordinary key, with no weight for how many columns it stands for.  One
    softmax runs over [kept keys, own key if dropped, mean key].  The dropped
    tokens are summed ``CHUNKS.sga_mean_tokens`` at a time and the queries
    taken in chunks of about ``CHUNKS.sga_row_elems`` logits.
    """
    rows = np.arange(geo.T) if rows is None else np.asarray(rows, dtype=np.int64)
    kept = sga_key_tokens(geo, sub_h, sub_w)
    is_kept = np.zeros(geo.T, dtype=bool)
    is_kept[kept] = True
    dropped = np.flatnonzero(~is_kept)
    q = f64(Q, rows)
    k_own, v_own = f64(K, rows), f64(V, rows)
    k_kept, v_kept = f64(K, kept), f64(V, kept)
    if dropped.size:
        k_mean = np.zeros((geo.H, geo.D))
        v_mean = np.zeros((geo.H, geo.D))
        for t0, t1 in spans(dropped.size, CHUNKS.sga_mean_tokens):
            part = dropped[t0:t1]
            k_mean += f64(K, part).sum(axis=0)
            v_mean += f64(V, part).sum(axis=0)
        k_mean /= dropped.size
        v_mean /= dropped.size
    out = np.full((rows.size, geo.H, geo.D), np.nan)
    step = max(1, CHUNKS.sga_row_elems // max(geo.H * (kept.size + 2), 1))
    for r0, r1 in spans(rows.size, step):
        qq = q[r0:r1]
        s_kept = qk_logits(qq, k_kept, geo.sm_scale)                               # [r, H, NK]
        s_own = np.sum(qq * k_own[r0:r1], axis=-1) * geo.sm_scale                  # [r, H]
        s_own = np.where(is_kept[rows[r0:r1]][:, None], -np.inf, s_own)
        if dropped.size:
            s_mean = np.sum(qq * k_mean[None], axis=-1) * geo.sm_scale            # [r, H]
        else:
            s_mean = np.full(s_own.shape, -np.inf)
        p = softmax(np.concatenate([s_kept, s_own[..., None], s_mean[..., None]], axis=-1))
        o = weighted_values(p[..., :kept.size], v_kept)
        o += p[..., kept.size, None] * v_own[r0:r1]
        if dropped.size:
            o += p[..., kept.size + 1, None] * v_mean[None]
        out[r0:r1] = o
    return out


# ----------------------------------------------------------------------------
# selection checks used by parity tests


def selection_valid_top_k(geo: Geometry, guide: np.ndarray, chosen: np.ndarray,
                          window: float) -> np.ndarray:
    """[rows, H] bool: ``chosen[r, h]`` (ids, -1 pad) is a top-K of ``guide[r, h]``
    ([rows, H, NB] S_guide) up to ``window``.

    A set is accepted when it has K_eff distinct ids among the candidate blocks
    and no unchosen candidate beats a chosen one by ``window`` or more.  With
    window 0 and no ties this is exactly the oracle's own top-K.
    """
    cg = guide[..., geo.B0:]
    n_c = cg.shape[-1]
    chosen = np.asarray(chosen, dtype=np.int64)
    used = chosen >= 0
    ids = np.where(used, chosen - geo.B0, 0)
    ok = used.sum(axis=-1) == geo.K_eff
    ok &= np.all(~used | ((ids >= 0) & (ids < n_c)), axis=-1)
    srt = np.sort(np.where(used, chosen, -1), axis=-1)
    ok &= ~np.any((srt[..., 1:] == srt[..., :-1]) & (srt[..., 1:] >= 0), axis=-1)
    # padding (and out-of-range ids, already rejected) point at a spare last column
    ids = np.where(used & (ids >= 0) & (ids < n_c), ids, n_c)
    ext = torch.full(cg.shape[:-1] + (n_c + 1,), -np.inf, dtype=torch.float64)
    ext[..., :n_c] = torch.from_numpy(cg)
    ids_t = torch.from_numpy(ids)
    picked = torch.gather(ext, -1, ids_t).numpy()
    lo = np.where(ids < n_c, picked, np.inf).min(axis=-1, initial=np.inf)  # weakest chosen
    ext.scatter_(-1, ids_t, -np.inf)
    hi = ext.amax(dim=-1).numpy()                                          # strongest unchosen
    return ok & (hi - lo < window)


def selection_is_valid_top_k(geo: Geometry, guide_row: np.ndarray, chosen: np.ndarray,
                             window: float) -> bool:
    """selection_valid_top_k for one (row, head)."""
    return bool(selection_valid_top_k(geo, np.asarray(guide_row)[None, None],
                                      np.asarray(chosen)[None, None], window)[0, 0])
