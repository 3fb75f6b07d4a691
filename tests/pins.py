"""Checks that pin the CPU oracle to facts outside itself.

Each ``pin_*`` raises AssertionError when the oracle disagrees with a closed
form, a library routine (torch's scaled_dot_product_attention in float64), the
independent pure-Python brute force in ``bruteforce.py``, or an invariant the
method fixes.  The oracle is looked up through its module at call time so the
mutation tests can plant mistakes in it and see these checks fail.
"""

import numpy as np
import torch

import bruteforce
from oracle import gsa_oracle as O
from synthetic import Workload, generate

TOL = 1e-11


def micro(N=2, S=1, Hp=6, Wp=7, H=2, D=8, P=4, K=2, seed=5, keep="specials"):
    wl = Workload("micro", N, S, Hp, Wp, H, D, P, K, seed, "gaussian")
    x = generate(wl)
    geo = O.Geometry(N=N, S=S, Hp=Hp, Wp=Wp, H=H, D=D, P=P, K=K, keep=keep)
    return geo, x


def sdpa_dense(q, k, v):
    """torch's scaled_dot_product_attention in float64: [T, H, D] -> [T, H, D]."""
    t = lambda x: x.to(torch.float64).permute(1, 0, 2).unsqueeze(0)  # noqa: E731
    o = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v))
    return o.squeeze(0).permute(1, 0, 2).numpy()


def close(a, b, tol=TOL, what=""):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, f"{what}: shape {a.shape} vs {b.shape}"
    err = np.max(np.abs(a - b)) if a.size else 0.0
    assert err <= tol, f"{what}: max abs err {err:.3e} > {tol:.1e}"


def read_block_structure_fixture(path):
    vals = {}
    for line in open(path):
        line = line.split("#", 1)[0].strip()
        if line:
            k, v = line.split("=")
            vals[k.strip()] = int(v)
    return vals


# ---------------------------------------------------------------------------


def pin_block_structure(fixture_path):
    """37x37 grid, P=4: 100 blocks per frame; 81 of 16, 18 of 4, 1 of 1 tokens."""
    want = read_block_structure_fixture(fixture_path)
    geo = O.Geometry(N=1, S=5, Hp=37, Wp=37, H=1, D=64, P=4, K=1)
    sizes = [O.Geometry.block_tokens(geo, b).size for b in range(geo.NB)]
    assert geo.Bf == want["blocks_per_frame"]
    assert sizes.count(16) == want["full_blocks"]
    assert sizes.count(4) == want["edge_blocks"]
    assert sizes.count(1) == want["corner_blocks"]
    assert sum(sizes) == want["patch_tokens"]


def pin_pool_ramp():
    """Pooling a ramp: the block mean has a closed form from the row/col ranges."""
    N, S, Hp, Wp, H, D, P = 2, 2, 7, 6, 2, 3, 4
    geo = O.Geometry(N=N, S=S, Hp=Hp, Wp=Wp, H=H, D=D, P=P, K=1)
    L = S + Hp * Wp
    X = np.zeros((N * L, H, D))
    for f in range(N):
        for j in range(S):
            X[f * L + j] = -(100.0 + 10 * f + j)
        for r in range(Hp):
            for c in range(Wp):
                for h in range(H):
                    for d in range(D):
                        X[f * L + S + r * Wp + c, h, d] = 1000 * f + 10 * r + c + 0.25 * h + 0.125 * d
    got = O.pool(geo, X)
    E = S + (-(-Hp // P)) * (-(-Wp // P))
    assert got.shape == (N * E, H, D)
    for f in range(N):
        for j in range(S):
            close(got[f * E + j], np.full((H, D), -(100.0 + 10 * f + j)), what="special entry")
        i = S
        for r0 in range(0, Hp, P):
            r1 = min(r0 + P, Hp)
            for c0 in range(0, Wp, P):
                c1 = min(c0 + P, Wp)
                mr, mc = (r0 + r1 - 1) / 2.0, (c0 + c1 - 1) / 2.0
                want = np.array([[1000 * f + 10 * mr + mc + 0.25 * h + 0.125 * d for d in range(D)]
                                 for h in range(H)])
                close(got[f * E + i], want, what=f"block ({r0},{c0})")
                i += 1


def pin_dense_matches_sdpa():
    geo, x = micro(N=3, S=2, Hp=5, Wp=4, H=3, D=16)
    close(O.dense_attention(geo, x.q, x.k, x.v), sdpa_dense(x.q, x.k, x.v), what="dense vs sdpa")


def pin_compressed_is_dense_at_pool_1():
    """P=1: every block is one patch, so the compression branch is dense attention."""
    geo, x = micro(N=2, S=2, Hp=4, Wp=5, H=2, D=16, P=1, K=3)
    res = O.gsa_layer(geo, x.q, x.k, x.v, x.w)
    close(res["o_cmp"], sdpa_dense(x.q, x.k, x.v), what="o_cmp(P=1) vs dense")


def pin_selected_is_dense_at_k_all():
    """K >= number of blocks: the selection branch attends to every token once."""
    geo, x = micro(N=2, S=2, Hp=6, Wp=7, H=2, D=16, P=4, K=99)
    res = O.gsa_layer(geo, x.q, x.k, x.v, x.w)
    close(res["o_sel"], sdpa_dense(x.q, x.k, x.v), what="o_sel(K=all) vs dense")


def pin_layer_is_dense_at_pool_1_k_all():
    geo, x = micro(N=2, S=1, Hp=3, Wp=5, H=2, D=8, P=1, K=1000)
    res = O.gsa_layer(geo, x.q, x.k, x.v, x.w)
    close(res["out"], sdpa_dense(x.q, x.k, x.v), what="out(P=1,K=all) vs dense")


def pin_constant_values():
    geo, x = micro(N=2, S=1, Hp=6, Wp=7, H=2, D=8)
    c = np.linspace(-1.5, 2.0, geo.H * geo.D).reshape(geo.H, geo.D)
    v = torch.from_numpy(np.broadcast_to(c, (geo.T, geo.H, geo.D)).copy())
    res = O.gsa_layer(geo, x.q, x.k, v, x.w)
    for name in ("o_cmp", "o_sel", "out"):
        close(res[name], np.broadcast_to(c, res[name].shape), what=f"constant V: {name}")


def pin_zero_queries():
    """Q = 0: every score ties at 0, so blocks 0..K-1 are chosen (lower id wins)
    and each branch returns a plain mean over its keys."""
    N, S, Hp, Wp, H, D, P, K = 2, 1, 6, 7, 2, 8, 4, 3
    geo, x = micro(N=N, S=S, Hp=Hp, Wp=Wp, H=H, D=D, P=P, K=K)
    q = torch.zeros_like(x.q)
    res = O.gsa_layer(geo, q, x.k, x.v, x.w)
    assert (res["sel"] == np.arange(K)).all(), "ties must go to the lowest block ids"
    frames = bruteforce.layout(N, S, Hp, Wp, P)
    blocks = [b for _, bl in frames for b in bl]
    specials = [t for sp, _ in frames for t in sp]
    v = x.v.to(torch.float64).numpy()
    keys = [t for b in blocks[:K] for t in b] + specials
    close(res["o_sel"], np.broadcast_to(v[keys].mean(axis=0), res["o_sel"].shape), what="o_sel(Q=0)")
    entries = []
    for sp, bl in frames:
        entries += [[t] for t in sp] + bl
    vbar = np.stack([v[e].mean(axis=0) for e in entries])
    close(res["o_cmp"], np.broadcast_to(vbar.mean(axis=0), res["o_cmp"].shape), what="o_cmp(Q=0)")
    close(res["g"], np.full(res["g"].shape, 0.5), what="g(Q=0)")


def pin_gate_limits():
    geo, x = micro(N=2, S=1, Hp=6, Wp=7, H=2, D=8)
    q = x.q.clone()
    q[..., 0] = q[..., 0].abs() + 1.0  # every pooled query has q_mean[0] >= 1
    zero = torch.zeros_like(x.w)
    res = O.gsa_layer(geo, q, x.k, x.v, zero)
    close(res["g"], np.full(res["g"].shape, 0.5), what="g(w=0)")
    close(res["out"], 0.5 * (res["o_cmp_up"] + res["o_sel"]), what="out(w=0)")
    big = torch.zeros_like(x.w)
    big[:, 0] = 1000.0
    res = O.gsa_layer(geo, q, x.k, x.v, big)
    close(res["out"], res["o_cmp_up"], tol=1e-9, what="g->1 keeps the compression branch")
    res = O.gsa_layer(geo, q, x.k, x.v, -big)
    close(res["out"], res["o_sel"], tol=1e-9, what="g->0 keeps the selection branch")


def pin_planted_top_k():
    """Every query equals u; block beta's keys all equal c_beta * u, so its score
    is c_beta |u|^2 / sqrt(D).  Special keys score highest of all but are not
    candidates.  Two blocks tie at the boundary: the lower id must win."""
    N, S, Hp, Wp, H, D, P, K = 3, 2, 6, 7, 2, 8, 4, 4
    geo = O.Geometry(N=N, S=S, Hp=Hp, Wp=Wp, H=H, D=D, P=P, K=K)
    rng = np.random.default_rng(11)
    u = rng.standard_normal((H, D))
    NB = geo.NB
    c = rng.permutation(NB).astype(np.float64)  # distinct 0..NB-1
    c[c == NB - K] = NB - K - 1.0  # the K-th largest now ties with the (K+1)-th
    L = S + Hp * Wp
    q = np.broadcast_to(u, (N * L, H, D)).copy()
    k = np.zeros((N * L, H, D))
    frames = bruteforce.layout(N, S, Hp, Wp, P)
    beta = 0
    for sp, bl in frames:
        for t in sp:
            k[t] = 1000.0 * u
        for toks in bl:
            for t in toks:
                k[t] = c[beta] * u
            beta += 1
    v = rng.standard_normal((N * L, H, D))
    res = O.gsa_layer(geo, q, k, v, np.zeros((H, D)))
    want = sorted(sorted(range(NB), key=lambda b: (-c[b], b))[:K])
    for a in range(res["sel"].shape[0]):
        for h in range(H):
            assert list(res["sel"][a, h]) == want, f"planted top-K: {list(res['sel'][a, h])} != {want}"


def pin_bruteforce_layer():
    geo, x = micro(N=2, S=1, Hp=6, Wp=7, H=2, D=8, P=4, K=2)
    res = O.gsa_layer(geo, x.q, x.k, x.v, x.w)
    Q = x.q.to(torch.float64).tolist()
    K = x.k.to(torch.float64).tolist()
    V = x.v.to(torch.float64).tolist()
    W = x.w.to(torch.float64).tolist()
    bf = bruteforce.gsa_bruteforce(Q, K, V, W, geo.N, geo.S, geo.Hp, geo.Wp, geo.P, geo.K)
    close(res["o_cmp"], bf["o_cmp"], what="brute force o_cmp")
    assert res["sel"].tolist() == bf["sel"], "brute force selection"
    close(res["o_sel"], bf["o_sel"], what="brute force o_sel")
    close(res["g"], bf["g"], what="brute force gate")
    close(res["out"], bf["out"], what="brute force out")


def pin_dense_key_slices():
    """The sliced two-pass form of dense_attention (used for long sequences)
    equals torch's SDPA: slices of 7 keys over 60 tokens, ragged last slice,
    row chunks of 3."""
    geo, x = micro(N=2, S=2, Hp=4, Wp=7, H=2, D=8)
    got = O.dense_attention(geo, x.q, x.k, x.v, key_chunk=7, max_bytes=3 * geo.H * 7 * 8)
    close(got, sdpa_dense(x.q, x.k, x.v), what="dense in key slices vs sdpa")


def pin_bruteforce_dense():
    geo, x = micro(N=2, S=1, Hp=3, Wp=4, H=2, D=8)
    Q, K, V = (t.to(torch.float64).tolist() for t in (x.q, x.k, x.v))
    close(O.dense_attention(geo, x.q, x.k, x.v), bruteforce.dense_bruteforce(Q, K, V), what="dense bf")


def pin_frame_permutation():
    """Reordering the frames reorders every output the same way and renames the
    selected blocks by the same permutation (inputs without ties)."""
    geo, x = micro(N=3, S=1, Hp=5, Wp=6, H=2, D=8, P=4, K=3)
    perm = [2, 0, 1]
    L = geo.L
    idx = torch.cat([torch.arange(p * L, (p + 1) * L) for p in perm])
    res = O.gsa_layer(geo, x.q, x.k, x.v, x.w)
    res2 = O.gsa_layer(geo, x.q[idx], x.k[idx], x.v[idx], x.w)
    close(res2["out"], res["out"][idx.numpy()], what="permuted out")
    Bf, E = geo.Bf, geo.E
    new_frame = {p: f for f, p in enumerate(perm)}  # old frame -> new frame
    for f, p in enumerate(perm):
        for j in range(E):
            a2, a = f * E + j, p * E + j
            for h in range(geo.H):
                want = sorted(new_frame[int(b) // Bf] * Bf + int(b) % Bf for b in res["sel"][a, h])
                assert list(res2["sel"][a2, h]) == want, "permuted selection"


def pin_row_subset():
    """Evaluating a subset of query rows gives those rows of the full layer."""
    geo, x = micro(N=2, S=1, Hp=6, Wp=7, H=2, D=8)
    full = O.gsa_layer(geo, x.q, x.k, x.v, x.w)
    rows = np.array([0, 5, 17, 43, geo.T - 1])
    sub = O.gsa_layer(geo, x.q, x.k, x.v, x.w, rows=rows)
    close(sub["out"], full["out"][rows], what="row subset out")
    close(O.dense_attention(geo, x.q, x.k, x.v, rows=rows),
          O.dense_attention(geo, x.q, x.k, x.v)[rows], what="row subset dense")


def pin_frame_attention():
    """Frame attention: one frame = dense attention; several frames = torch's
    SDPA applied to each frame's slice; and the independent brute force."""
    geo1, x1 = micro(N=1, S=2, Hp=4, Wp=5, H=2, D=16)
    close(O.frame_attention(geo1, x1.q, x1.k, x1.v), sdpa_dense(x1.q, x1.k, x1.v), what="frame(N=1)")
    geo, x = micro(N=3, S=1, Hp=3, Wp=4, H=2, D=8)
    got = O.frame_attention(geo, x.q, x.k, x.v)
    L = geo.L
    want = np.concatenate([sdpa_dense(x.q[f * L:(f + 1) * L], x.k[f * L:(f + 1) * L], x.v[f * L:(f + 1) * L])
                           for f in range(geo.N)])
    close(got, want, what="frame vs per-frame sdpa")
    Q, K, V = (t.to(torch.float64).tolist() for t in (x.q, x.k, x.v))
    close(got, bruteforce.frame_bruteforce(Q, K, V, L), what="frame brute force")
    rows = np.array([0, L - 1, L, 2 * L + 3])
    close(O.frame_attention(geo, x.q, x.k, x.v, rows=rows), got[rows], what="frame row subset")


def pin_reference_one_frame():
    """Reference-frame keep, one frame: nothing is ranked (K_eff = 0) and the
    selection branch attends to the whole frame, i.e. it is dense attention."""
    geo, x = micro(N=1, S=3, Hp=6, Wp=5, H=2, D=8, P=2, K=4, keep="reference")
    assert geo.K_eff == 0
    res = O.gsa_layer(geo, x.q, x.k, x.v, x.w)
    assert (res["sel"] == -1).all()
    close(res["o_sel"], sdpa_dense(x.q, x.k, x.v), what="reference keep, one frame")


def pin_reference_k_all():
    """Reference-frame keep with every candidate block selected: the key set is
    every token except the register tokens (special slots >= 1) of frames
    1..N-1, so the selection branch is SDPA under that key mask; with one
    special token per frame it is plain dense attention."""
    geo, x = micro(N=3, S=3, Hp=5, Wp=6, H=2, D=8, P=4, K=64, keep="reference")
    assert geo.K_eff == geo.NB - geo.Bf
    res = O.gsa_layer(geo, x.q, x.k, x.v, x.w)
    L = geo.L
    allowed = torch.ones(geo.T, dtype=torch.bool)
    for f in range(1, geo.N):
        allowed[f * L + 1:f * L + geo.S] = False
    t = lambda z: z.to(torch.float64).permute(1, 0, 2).unsqueeze(0)  # noqa: E731
    mask = allowed[None, None, None, :].expand(1, geo.H, geo.T, geo.T)
    want = torch.nn.functional.scaled_dot_product_attention(t(x.q), t(x.k), t(x.v), attn_mask=mask)
    close(res["o_sel"], want.squeeze(0).permute(1, 0, 2).numpy(), what="reference keep, K = all")
    geo1, x1 = micro(N=3, S=1, Hp=5, Wp=6, H=2, D=8, P=4, K=64, keep="reference")
    res1 = O.gsa_layer(geo1, x1.q, x1.k, x1.v, x1.w)
    close(res1["o_sel"], sdpa_dense(x1.q, x1.k, x1.v), what="reference keep, S=1, K = all")


def pin_reference_bruteforce():
    """Reference-frame keep on a small input with K below the candidate count:
    the whole layer against the independent brute force."""
    geo, x = micro(N=3, S=2, Hp=6, Wp=7, H=2, D=8, P=4, K=3, keep="reference")
    res = O.gsa_layer(geo, x.q, x.k, x.v, x.w)
    Q, K, V, W = (t.to(torch.float64).tolist() for t in (x.q, x.k, x.v, x.w))
    bf = bruteforce.gsa_bruteforce(Q, K, V, W, geo.N, geo.S, geo.Hp, geo.Wp, geo.P, geo.K,
                                   keep="reference")
    assert res["sel"].tolist() == bf["sel"], "brute force selection (reference keep)"
    assert (res["sel"][res["sel"] >= 0] >= geo.Bf).all(), "frame 0 blocks are not ranked"
    close(res["o_sel"], bf["o_sel"], what="brute force o_sel (reference keep)")
    close(res["out"], bf["out"], what="brute force out (reference keep)")


def pin_sga():
    """AVGGT SGA: with windows of 1 x 1 nothing is dropped (no mean pair, the
    diagonal is already a key), so it is dense attention; on a ragged grid it
    matches the independent brute force; and the kept key ids follow the grid."""
    geo, x = micro(N=2, S=2, Hp=5, Wp=7, H=2, D=8)
    close(O.sga_attention(geo, x.q, x.k, x.v, 1, 1), sdpa_dense(x.q, x.k, x.v), what="sga 1x1 = dense")
    Q, K, V = (t.to(torch.float64).tolist() for t in (x.q, x.k, x.v))
    for sh, sw in ((2, 3), (3, 2), (5, 7)):
        got = O.sga_attention(geo, x.q, x.k, x.v, sh, sw)
        want = bruteforce.sga_bruteforce(Q, K, V, geo.L, geo.S, geo.Hp, geo.Wp, sh, sw)
        close(got, want, what=f"sga {sh}x{sw} brute force")
    rows = np.array([0, 3, 9, geo.L + 2, geo.T - 1])
    close(O.sga_attention(geo, x.q, x.k, x.v, 2, 3, rows=rows),
          O.sga_attention(geo, x.q, x.k, x.v, 2, 3)[rows], what="sga row subset")
    ids = O.sga_key_tokens(geo, 2, 3)
    per_frame = geo.S + 3 * 3  # rows 0,2,4 x cols 0,3,6
    assert ids.size == geo.N * per_frame
    assert list(ids[:per_frame]) == [0, 1, 2, 5, 8, 16, 19, 22, 30, 33, 36]


# ---------------------------------------------------------------------------
# the split forms the oracle takes at full size, forced on micro inputs


def _same(a, b, what):
    """Two runs of the oracle that differ only in how the work is split."""
    for key in a:
        if key in b and isinstance(a[key], np.ndarray) and a[key].dtype != bool:
            close(a[key], b[key], tol=1e-12, what=f"{what}: {key}")


def pin_split_layer():
    """The whole layer with every split form forced: torch's threaded softmax
    for every softmax, pooling two frames at a time (three frames: a ragged
    last slice) and steps 2-4 over chunks of five compressed entries (a ragged
    last chunk) equals the unsplit run and the brute force, for both always-kept
    readings and for a subset of rows."""
    for keep in ("specials", "reference"):
        geo, x = micro(N=3, S=2, Hp=6, Wp=7, H=2, D=8, P=4, K=3, keep=keep)
        assert geo.N % 2 == 1 and geo.Tc % 5 != 0
        plain = O.gsa_layer(geo, x.q, x.k, x.v, x.w)
        rows = np.array([0, 2, 9, geo.L + 4, geo.T - 7, geo.T - 1])
        with O.chunking(softmax_torch_elems=1, pool_frames=2, layer_chunk_elems=5 * geo.H * geo.Tc):
            split = O.gsa_layer(geo, x.q, x.k, x.v, x.w)
            sub = O.gsa_layer(geo, x.q, x.k, x.v, x.w, rows=rows)
        _same(plain, split, f"split layer ({keep})")
        close(sub["out"], plain["out"][rows], tol=1e-12, what=f"split layer rows ({keep})")
        Q, K, V, W = (t.to(torch.float64).tolist() for t in (x.q, x.k, x.v, x.w))
        bf = bruteforce.gsa_bruteforce(Q, K, V, W, geo.N, geo.S, geo.Hp, geo.Wp, geo.P, geo.K, keep=keep)
        assert split["sel"].tolist() == bf["sel"], f"split layer selection ({keep})"
        for key in ("o_cmp", "o_sel", "g", "out"):
            close(split[key], bf[key], what=f"split layer vs brute force ({keep}): {key}")


def pin_split_dense():
    """Dense and frame attention with their split forms forced: rows three at a
    time through torch's softmax (short sequences), then key slices of seven
    tokens with rows in chunks of three (long sequences), against torch's SDPA."""
    geo, x = micro(N=3, S=2, Hp=4, Wp=5, H=2, D=8)
    want = sdpa_dense(x.q, x.k, x.v)
    with O.chunking(softmax_torch_elems=1, dense_max_bytes=3 * geo.H * geo.T * 8):
        close(O.dense_attention(geo, x.q, x.k, x.v), want, what="dense, rows in threes, torch softmax")
        L = geo.L
        frames = np.concatenate([sdpa_dense(x.q[f * L:(f + 1) * L], x.k[f * L:(f + 1) * L],
                                            x.v[f * L:(f + 1) * L]) for f in range(geo.N)])
        close(O.frame_attention(geo, x.q, x.k, x.v), frames, what="frame attention, torch softmax")
    with O.chunking(dense_key_chunk=7, dense_max_bytes=3 * geo.H * 7 * 8):
        close(O.dense_attention(geo, x.q, x.k, x.v), want, what="dense in key slices of 7")


def pin_split_sga():
    """SGA with its split forms forced: the dropped tokens summed five at a time,
    queries three at a time, torch's softmax; against the unsplit run and the
    brute force."""
    geo, x = micro(N=2, S=2, Hp=5, Wp=7, H=2, D=8)
    Q, K, V = (t.to(torch.float64).tolist() for t in (x.q, x.k, x.v))
    for sh, sw in ((2, 3), (3, 2)):
        nk = O.sga_key_tokens(geo, sh, sw).size
        plain = O.sga_attention(geo, x.q, x.k, x.v, sh, sw)
        with O.chunking(softmax_torch_elems=1, sga_mean_tokens=5, sga_row_elems=3 * geo.H * (nk + 2)):
            split = O.sga_attention(geo, x.q, x.k, x.v, sh, sw)
        close(split, plain, tol=1e-12, what=f"split sga {sh}x{sw}")
        close(split, bruteforce.sga_bruteforce(Q, K, V, geo.L, geo.S, geo.Hp, geo.Wp, sh, sw),
              what=f"split sga {sh}x{sw} brute force")


def pin_variant_readings():
    """The variant readings A1 (fine queries in the compression branch) and A10
    (a gate per fine token): at P = 1 both equal the default layer; the fine
    compression branch is torch's SDPA of the fine queries over the pooled keys
    and values; a per-token gate is 1/2 for w = 0 and saturates with the sign
    of q_t . w."""
    geo1, x1 = micro(N=2, S=1, Hp=3, Wp=5, H=2, D=8, P=1, K=4)
    base = O.gsa_layer(geo1, x1.q, x1.k, x1.v, x1.w)
    var = O.gsa_layer(geo1, x1.q, x1.k, x1.v, x1.w, queries="fine", gate_per="token")
    close(var["out"], base["out"], what="variants at P = 1")
    geo, x = micro(N=2, S=2, Hp=6, Wp=7, H=2, D=8, P=4, K=3)
    res = O.gsa_layer(geo, x.q, x.k, x.v, x.w, queries="fine")
    Kc, Vc = O.pool(geo, x.k), O.pool(geo, x.v)
    t = lambda z: torch.as_tensor(z, dtype=torch.float64).permute(1, 0, 2).unsqueeze(0)  # noqa: E731
    want = torch.nn.functional.scaled_dot_product_attention(t(x.q.double().numpy()), t(Kc), t(Vc))
    close(res["o_cmp_up"], want.squeeze(0).permute(1, 0, 2).numpy(), what="fine queries vs sdpa over pooled keys")
    zero = O.gsa_layer(geo, x.q, x.k, x.v, torch.zeros_like(x.w), gate_per="token")
    close(zero["g_rows"], np.full(zero["g_rows"].shape, 0.5), what="token gate, w = 0")
    big = torch.zeros_like(x.w)
    big[:, 0] = 1000.0
    q = x.q.clone()
    q[..., 0] = torch.where(q[..., 0] >= 0, q[..., 0].abs() + 1, -(q[..., 0].abs() + 1))  # |q_t . w| >= 1000
    sat = O.gsa_layer(geo, q, x.k, x.v, big, gate_per="token")
    sign = (q[:, :, 0].double().numpy() > 0).astype(np.float64)
    close(sat["g_rows"], sign, tol=1e-9, what="token gate saturates with sign(q_t . w)")


def all_pins(fixture_path):
    return {
        "block_structure": lambda: pin_block_structure(fixture_path),
        "pool_ramp": pin_pool_ramp,
        "dense_sdpa": pin_dense_matches_sdpa,
        "compressed_p1": pin_compressed_is_dense_at_pool_1,
        "selected_kall": pin_selected_is_dense_at_k_all,
        "layer_dense_limit": pin_layer_is_dense_at_pool_1_k_all,
        "constant_v": pin_constant_values,
        "zero_q": pin_zero_queries,
        "gate_limits": pin_gate_limits,
        "planted_topk": pin_planted_top_k,
        "bruteforce_layer": pin_bruteforce_layer,
        "bruteforce_dense": pin_bruteforce_dense,
        "frame_permutation": pin_frame_permutation,
        "row_subset": pin_row_subset,
        "frame_attention": pin_frame_attention,
        "dense_key_slices": pin_dense_key_slices,
        "sga": pin_sga,
        "reference_one_frame": pin_reference_one_frame,
        "reference_k_all": pin_reference_k_all,
        "reference_bruteforce": pin_reference_bruteforce,
        "split_layer": pin_split_layer,
        "split_dense": pin_split_dense,
        "split_sga": pin_split_sga,
        "variant_readings": pin_variant_readings,
    }
