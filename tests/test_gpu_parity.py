"""CUDA path vs the float64 CPU oracle, through the C ABI (needs a B200).

Every step of the path is checked element by element on workloads the oracle
finishes in seconds (several tiles, ragged tails, partial edge blocks, K >= the
number of blocks, pool factors 1-4, no special tokens), and the whole layer on
sampled query rows of the 100-, 300- and 1000-frame workloads.
"""

import numpy as np
import pytest
import torch

import parity as PT
from oracle import gsa_oracle as O
from synthetic import WORKLOADS, Workload, generate
from synthetic.workloads import sample_rows

pytestmark = pytest.mark.gpu

CASES = {
    "tiny": WORKLOADS["tiny"],
    "small": WORKLOADS["small"],
    # pool 3 with ragged blocks in both directions, 2 specials per frame
    "p3_ragged": Workload("p3_ragged", 3, 2, 10, 11, 2, 64, 3, 5, 7, "gaussian"),
    # pool 1 (every block one patch), no specials, T not a multiple of 64
    "p1_nospecial": Workload("p1_nospecial", 2, 0, 5, 7, 2, 64, 1, 6, 8, "gaussian"),
    # K larger than the number of blocks: every block kept, -1 padding
    "k_all": Workload("k_all", 2, 3, 6, 7, 3, 64, 4, 128, 9, "gaussian"),
    # pool 2, one head, single special
    "p2_onehead": Workload("p2_onehead", 4, 1, 9, 9, 1, 64, 2, 7, 10, "gaussian"),
    # one VGGT-shaped frame
    "one_frame": Workload("one_frame", 1, 5, 37, 37, 4, 64, 4, 16, 11, "gaussian"),
    # nine tokens: a single, mostly empty 128-row query tile and key tile
    "nine_tokens": Workload("nine_tokens", 1, 3, 2, 3, 2, 64, 2, 2, 12, "gaussian"),
    # reference-frame keep (frame 0 whole + camera tokens; frame 0 not ranked)
    "ref_small": WORKLOADS["small"].with_(name="ref_small", keep=1),
    "ref_p3_ragged": Workload("ref_p3_ragged", 3, 2, 10, 11, 2, 64, 3, 5, 7, "gaussian", keep=1),
    # one frame: nothing to rank (K_eff = 0), the kept set is the whole frame
    "ref_one_frame": Workload("ref_one_frame", 1, 5, 37, 37, 4, 64, 4, 16, 11, "gaussian", keep=1),
    # no specials: the kept set is frame 0's patches alone
    "ref_nospecial": Workload("ref_nospecial", 3, 0, 9, 10, 2, 64, 2, 6, 13, "gaussian", keep=1),
    # test-time K = 128 (above the fused kernel's heap): two ranking passes in
    # gsa_forward, the split scorer in the stage calls
    "k128_small": WORKLOADS["small"].with_(name="k128_small", top_k=128),
    # an uneven second pass (64 + 36) and the reference keep with K = 128
    "k100_small": WORKLOADS["small"].with_(name="k100_small", top_k=100),
    "ref_k128": Workload("ref_k128", 4, 5, 37, 37, 2, 64, 4, 128, 14, "gaussian", keep=1),
}

_cache = {}


def _dev(x):
    return (x.q.cuda(), x.k.cuda(), x.v.cuda(), x.w.cuda())


def case(name, n_split=1):
    key = (name, n_split)
    if key not in _cache:
        import sparse_global_attention_view_b200 as G
        wl = CASES[name]
        x = generate(wl)
        geo = O.geometry_of(wl)
        shape = G.Shape.of(wl)
        q, k, v, w = _dev(x)
        st = PT.Stages(shape, q, k, v, w, n_split).run()
        res = O.gsa_layer(geo, x.q, x.k, x.v, x.w, sel_override=st.sel_by_entry())
        _cache[key] = (x, geo, shape, st, res)
    return _cache[key]


NAMES = list(CASES)


def _bf16_rn(x: np.ndarray) -> np.ndarray:
    """float64 values rounded once to bf16 (8 significant bits), nearest-even,
    returned as float64."""
    x = np.asarray(x, dtype=np.float64)
    mant, e = np.frexp(x)  # x = mant * 2^e, 0.5 <= |mant| < 1
    return np.ldexp(np.round(mant * 256.0) / 256.0, e)  # np.round: half to even


def assert_bf16_of_mean(gpu: torch.Tensor, mean64: np.ndarray, what: str) -> None:
    """The GPU's bf16 means must be the round-to-nearest-even bf16 of the exact
    (float64) mean, bit for bit.  The one allowed exception: the GPU forms the
    mean in fp32 before rounding to bf16, so a value may instead be the bf16 of
    that fp32 mean (or of its fp32 neighbours) where this differs from the exact
    one -- a double-rounding case; those cases are counted and must stay rare."""
    g = gpu.cpu().double().numpy()
    m = np.asarray(mean64, dtype=np.float64)
    exact = _bf16_rn(m)
    f32 = m.astype(np.float32)
    via = [_bf16_rn(f32.astype(np.float64)),
           _bf16_rn(np.nextafter(f32, np.float32(np.inf)).astype(np.float64)),
           _bf16_rn(np.nextafter(f32, np.float32(-np.inf)).astype(np.float64))]
    ok = g == exact
    for v in via:
        ok |= g == v
    assert ok.all(), f"{what}: {int((~ok).sum())} bf16 means are neither the rounded exact mean nor a double rounding of it"
    frac = float((g != exact).mean()) if g.size else 0.0
    assert frac < 1e-3, f"{what}: {frac:.2e} of the bf16 means differ from the once-rounded exact mean"


@pytest.mark.parametrize("name", NAMES)
def test_pool(name):
    x, geo, shape, st, res = case(name)
    np.testing.assert_allclose(st.qc32.cpu().double().numpy(), res["qc"], rtol=1e-6, atol=1e-7)
    np.testing.assert_allclose(st.kc32.cpu().double().numpy(), res["kc"], rtol=1e-6, atol=1e-7)
    # bf16 means: the nearest-even bf16 of the exact mean, bit for bit
    assert_bf16_of_mean(st.vc, res["vc"], f"{name} vc")
    assert_bf16_of_mean(st.qc, res["qc"], f"{name} qc")
    assert_bf16_of_mean(st.kc, res["kc"], f"{name} kc")
    kept = geo.kept_tokens()
    if kept.size:
        kept = torch.as_tensor(np.array(kept))
        assert torch.equal(st.ks.cpu(), x.k[kept].permute(1, 0, 2))
        assert torch.equal(st.vs.cpu(), x.v[kept].permute(1, 0, 2))
    else:
        assert st.ks is None


@pytest.mark.parametrize("name", NAMES)
def test_compressed_attention(name):
    x, geo, shape, st, res = case(name)
    assert PT.zeros_fail(res["o_cmp"])
    PT.assert_close(st.oc, res["o_cmp"], f"{name} o_cmp")


@pytest.mark.parametrize("name", NAMES)
def test_top_k_selection(name):
    x, geo, shape, st, res = case(name)
    PT.assert_selection(res, name)
    sel = st.sel_by_entry()
    assert (sel[:, :, geo.K_eff:] == -1).all()
    chosen = sel[:, :, :geo.K_eff]
    assert (chosen >= 0).all() and (chosen < geo.NB).all()
    assert (np.diff(chosen, axis=-1) > 0).all(), "ids must be strictly ascending"


@pytest.mark.parametrize("name", ["small", "p3_ragged"])
def test_split_candidates_merge_to_same_selection(name):
    # n_split > 1 runs the fp32 block scorer over slices of the block range;
    # merging 2 or 3 slice lists must give the same selection
    a = case(name, 2)[3].sel.cpu()
    b = case(name, 3)[3].sel.cpu()
    assert torch.equal(a, b)


@pytest.mark.parametrize("name", ["small", "p3_ragged", "tiny"])
def test_sliced_block_scorer_is_valid(name):
    x, geo, shape, st, res = case(name, 3)
    PT.assert_selection(res, f"{name} (3 slices)")
    PT.assert_close(st.oc, res["o_cmp"], f"{name} o_cmp (warp-MMA path)")


@pytest.mark.parametrize("name", NAMES)
def test_selected_attention(name):
    x, geo, shape, st, res = case(name)
    assert PT.zeros_fail(res["o_sel"])
    PT.assert_close(st.o_sel, res["o_sel"], f"{name} o_sel")
    assert torch.isfinite(st.lse).all()


@pytest.mark.parametrize("name", NAMES)
def test_gate_combine(name):
    x, geo, shape, st, res = case(name)
    assert PT.zeros_fail(res["out"])
    PT.assert_close(st.out, res["out"], f"{name} out (stages)")


@pytest.mark.parametrize("name", NAMES)
def test_forward(name):
    import sparse_global_attention_view_b200 as G
    x, geo, shape, st, res = case(name)
    layer = G.GsaLayer(shape)
    out1 = torch.full_like(st.q, float("nan"))
    layer(st.q, st.k, st.v, st.w, out1)
    out2 = layer(st.q, st.k, st.v, st.w)
    torch.cuda.synchronize()
    G.check_device_error(layer.ws)
    assert torch.equal(out1, out2), "forward must be deterministic"
    sel_fwd = G.workspace_view(layer.ws, shape, "sel").permute(1, 0, 2).contiguous().cpu().numpy()
    if not np.array_equal(sel_fwd, st.sel_by_entry()):
        # K > 64: gsa_forward ranks on the tensor cores in two passes, the
        # stage call with an fp32 scorer; both are top-K up to the tie window
        # but may differ inside it, so the oracle takes the forward's own set
        res = O.gsa_layer(geo, x.q, x.k, x.v, x.w, sel_override=sel_fwd)
        PT.assert_selection(res, f"{name} forward selection")
    PT.assert_close(out1, res["out"], f"{name} out (forward)")


@pytest.mark.parametrize("name", ["small", "p3_ragged", "ref_small", "k128_small", "one_frame"])
def test_forward_work_order(name):
    # the selection branch's (head, entry) pairs: a permutation of all pairs,
    # grouped by head and by the grid position of each row's best block, and
    # that best block is the row's top pair (exact where the oracle's first and
    # second scores differ by >= 1e-3; a selected block scoring within the
    # window of the top elsewhere)
    import sparse_global_attention_view_b200 as G
    x, geo, shape, st, res = case(name)
    layer = G.GsaLayer(shape)
    layer(st.q, st.k, st.v, st.w)
    torch.cuda.synchronize()
    G.check_device_error(layer.ws)
    order = G.workspace_view(layer.ws, shape, "order").cpu().numpy().astype(np.int64)
    best = G.workspace_view(layer.ws, shape, "best").cpu().numpy().astype(np.int64)  # [H, Tc]
    n = geo.H * geo.Tc
    assert np.array_equal(np.sort(order), np.arange(n)), "order must be a permutation of the pairs"
    h_of = order // geo.Tc
    bk = np.where(best.ravel()[order] >= 0, best.ravel()[order] % geo.Bf, 0)
    key = h_of * geo.Bf + bk
    assert (np.diff(key) >= 0).all(), "pairs must be grouped by (head, best block position)"
    sel = G.workspace_view(layer.ws, shape, "sel").permute(1, 0, 2).cpu().numpy()
    guide = res["guide"][..., geo.B0:]  # [Tc, H, candidates]
    bt = best.T  # [Tc, H]
    if geo.K_eff == 0:
        assert (bt == -1).all()
        return
    assert ((bt[..., None] == sel) | (bt[..., None] < 0)).any(-1).all(), "the best block must be selected"
    top2 = np.sort(guide, axis=-1)[..., -2:] if guide.shape[-1] > 1 else np.concatenate([guide, guide - 1], -1)
    got = np.take_along_axis(guide, (bt - geo.B0)[..., None], -1)[..., 0]
    assert (got >= top2[..., 1] - PT.TIE_WINDOW).all(), "best block must score within the window of the top"
    clear = (top2[..., 1] - top2[..., 0]) >= PT.TIE_WINDOW
    want = np.argmax(guide, axis=-1) + geo.B0
    assert (bt[clear] == want[clear]).all(), "best block must be the top pair where it is clear"


@pytest.mark.parametrize("name", ["k128_small", "k100_small", "ref_k128", "k_all", "ref_small", "small"])
def test_forward_selection(name):
    # the selection gsa_forward itself made (for K > 64: two ranking passes of
    # the fused kernel and their union) must be the oracle's top-K up to the
    # tie window, and the layer output must match the oracle evaluated with it
    import sparse_global_attention_view_b200 as G
    x, geo, shape, st, res = case(name)
    layer = G.GsaLayer(shape)
    out = torch.full_like(st.q, float("nan"))
    layer(st.q, st.k, st.v, st.w, out)
    torch.cuda.synchronize()
    G.check_device_error(layer.ws)
    sel = G.workspace_view(layer.ws, shape, "sel").permute(1, 0, 2).contiguous().cpu().numpy()
    rows = sample_rows(geo.T, 2048, seed=6, forced=PT.forced_rows(geo))
    ref = O.gsa_layer(geo, x.q, x.k, x.v, x.w, rows=rows, sel_override=sel)
    PT.assert_selection(ref, f"{name} forward selection")
    assert (sel[:, :, geo.K_eff:] == -1).all()
    chosen = sel[:, :, :geo.K_eff]
    assert (np.diff(chosen, axis=-1) > 0).all(), "ids must be strictly ascending"
    PT.assert_close(out[torch.as_tensor(rows).cuda()], ref["out"], f"{name} forward out")


@pytest.mark.parametrize("name", ["tiny", "p3_ragged", "p1_nospecial", "k_all", "p2_onehead", "nine_tokens"])
def test_dense_full(name):
    import sparse_global_attention_view_b200 as G
    x, geo, shape, st, res = case(name)
    out = torch.full_like(st.q, float("nan"))
    G.dense_global_attn(shape, st.q, st.k, st.v, out, st.ws)
    ref = O.dense_attention(geo, x.q, x.k, x.v)
    assert PT.zeros_fail(ref)
    PT.assert_close(out, ref, f"{name} dense")


@pytest.mark.parametrize("name", ["tiny", "p3_ragged", "p2_onehead", "nine_tokens", "one_frame"])
def test_frame_attention_full(name):
    import sparse_global_attention_view_b200 as G
    x, geo, shape, st, res = case(name)
    out = torch.full_like(st.q, float("nan"))
    G.frame_attn(shape, st.q, st.k, st.v, out, st.ws)
    ref = O.frame_attention(geo, x.q, x.k, x.v)
    assert PT.zeros_fail(ref)
    PT.assert_close(out, ref, f"{name} frame attention")


@pytest.mark.parametrize("name", ["small"])
def test_frame_attention_sampled(name):
    import sparse_global_attention_view_b200 as G
    x, geo, shape, st, res = case(name)
    out = torch.full_like(st.q, float("nan"))
    G.frame_attn(shape, st.q, st.k, st.v, out, st.ws)
    rows = sample_rows(geo.T, 512, seed=4, forced=PT.forced_rows(geo))
    PT.assert_close(out[torch.as_tensor(rows).cuda()], O.frame_attention(geo, x.q, x.k, x.v, rows=rows),
                    f"{name} frame attention sampled")
    assert not torch.isnan(out).any()


SGA_CASES = [("tiny", 2, 2), ("tiny", 1, 1), ("p3_ragged", 3, 2), ("p2_onehead", 2, 3),
             ("nine_tokens", 2, 2), ("one_frame", 4, 4), ("ref_nospecial", 3, 3), ("k_all", 9, 9)]


@pytest.mark.parametrize("name,sh,sw", SGA_CASES)
def test_sga_full(name, sh, sw):
    import sparse_global_attention_view_b200 as G
    x, geo, shape, st, res = case(name)
    ws = G.new_sga_workspace(shape, sh, sw)
    out = torch.full_like(st.q, float("nan"))
    G.sga_attn(shape, sh, sw, st.q, st.k, st.v, out, ws)
    torch.cuda.synchronize()
    G.check_device_error(ws)
    ref = O.sga_attention(geo, x.q, x.k, x.v, sh, sw)
    assert PT.zeros_fail(ref)
    PT.assert_close(out, ref, f"{name} sga {sh}x{sw}")
    if (sh, sw) == (1, 1):
        PT.assert_close(out, O.dense_attention(geo, x.q, x.k, x.v), f"{name} sga 1x1 vs dense")


def test_sga_workspace_too_small():
    import sparse_global_attention_view_b200 as G
    x, geo, shape, st, res = case("tiny")
    need = G.sga_workspace_size(shape, 2, 2)
    ws = G.new_workspace(None)  # header only
    assert ws.numel() < need
    out = torch.empty_like(st.q)
    with pytest.raises(G.GsaError):
        G.sga_attn(shape, 2, 2, st.q, st.k, st.v, out, ws)


@pytest.mark.parametrize("name", ["tiny", "p3_ragged", "nine_tokens"])
def test_dense_warp_mma_baseline(name):
    import sparse_global_attention_view_b200 as G
    x, geo, shape, st, res = case(name)
    out = torch.full_like(st.q, float("nan"))
    G.dense_global_attn_mma(shape, st.q, st.k, st.v, out, st.ws)
    PT.assert_close(out, O.dense_attention(geo, x.q, x.k, x.v), f"{name} dense (mma.sync)")


@pytest.mark.parametrize("name", ["small", "one_frame"])
def test_dense_sampled(name):
    import sparse_global_attention_view_b200 as G
    x, geo, shape, st, res = case(name)
    out = torch.full_like(st.q, float("nan"))
    G.dense_global_attn(shape, st.q, st.k, st.v, out, st.ws)
    rows = sample_rows(geo.T, 384, seed=1, forced=PT.forced_rows(geo))
    ref = O.dense_attention(geo, x.q, x.k, x.v, rows=rows)
    PT.assert_close(out[torch.as_tensor(rows).cuda()], ref, f"{name} dense sampled")
    assert not torch.isnan(out).any()


# ---- the 100, 300 and 1000-frame workloads on sampled rows -----------------

# 4096 sampled query rows (plus the forced edge / special rows) on each
BIG = {"medium": 4096, "large": 4096, "pages": 4096}
BIG_VARIANTS = {
    # reference-frame keep, and test-time K = 128, on the 100-frame workload
    "medium_ref": (WORKLOADS["medium"].with_(name="medium_ref", keep=1), 1024),
    "medium_k128": (WORKLOADS["medium"].with_(name="medium_k128", top_k=128), 1024),
}


def _big(name):
    if name in BIG_VARIANTS:
        return BIG_VARIANTS[name]
    return WORKLOADS[name], BIG[name]


@pytest.mark.parametrize("name", list(BIG) + list(BIG_VARIANTS))
def test_big_workload_sampled(name):
    import sparse_global_attention_view_b200 as G
    wl, n_rows = _big(name)
    x = generate(wl)
    geo = O.geometry_of(wl)
    shape = G.Shape.of(wl)
    q, k, v, w = _dev(x)
    st = PT.Stages(shape, q, k, v, w).run()
    layer = G.GsaLayer(shape)
    out = torch.full_like(q, float("nan"))
    layer(q, k, v, w, out)
    torch.cuda.synchronize()
    G.check_device_error(layer.ws)
    assert not torch.isnan(out).any()
    rows = sample_rows(geo.T, n_rows, seed=2, forced=PT.forced_rows(geo))
    res = O.gsa_layer(geo, x.q, x.k, x.v, x.w, rows=rows, sel_override=st.sel_by_entry())
    PT.assert_selection(res, name)
    idx = torch.as_tensor(rows).cuda()
    ent = torch.as_tensor(res["entries"]).cuda()
    PT.assert_close(st.oc[ent], res["o_cmp"], f"{name} o_cmp")
    PT.assert_close(st.o_sel[idx], res["o_sel"], f"{name} o_sel")
    sel_fwd = G.workspace_view(layer.ws, shape, "sel").permute(1, 0, 2).contiguous().cpu().numpy()
    if not np.array_equal(sel_fwd, st.sel_by_entry()):
        # K > 64: the forward's two tensor-core ranking passes and the stage
        # call's fp32 scorer may pick differently inside the tie window
        res = O.gsa_layer(geo, x.q, x.k, x.v, x.w, rows=rows, sel_override=sel_fwd)
        PT.assert_selection(res, f"{name} forward selection")
    PT.assert_close(out[idx], res["out"], f"{name} out")
    del st, layer
    torch.cuda.empty_cache()


DENSE_ROWS = {"medium": 1024, "large": 512, "pages": 128}


@pytest.mark.parametrize("name", list(DENSE_ROWS))
def test_big_dense_sampled(name):
    import sparse_global_attention_view_b200 as G
    wl = WORKLOADS[name]
    x = generate(wl)
    geo = O.geometry_of(wl)
    shape = G.Shape.of(wl)
    q, k, v, w = _dev(x)
    ws = G.new_workspace(None)
    out = torch.full_like(q, float("nan"))
    G.dense_global_attn(shape, q, k, v, out, ws)
    torch.cuda.synchronize()
    G.check_device_error(ws)
    assert not torch.isnan(out).any()
    rows = sample_rows(geo.T, DENSE_ROWS[name], seed=3, forced=PT.forced_rows(geo))
    ref = O.dense_attention(geo, x.q, x.k, x.v, rows=rows)
    PT.assert_close(out[torch.as_tensor(rows).cuda()], ref, f"{name} dense sampled")
    del q, k, v, out
    torch.cuda.empty_cache()


SGA_BIG = {"small": (4, 4, 512), "medium": (4, 4, 1024), "pages": (8, 8, 256)}


@pytest.mark.parametrize("name", list(SGA_BIG))
def test_big_sga_sampled(name):
    import sparse_global_attention_view_b200 as G
    sh, sw, n_rows = SGA_BIG[name]
    wl = WORKLOADS[name]
    x = generate(wl)
    geo = O.geometry_of(wl)
    shape = G.Shape.of(wl)
    q, k, v, w = _dev(x)
    ws = G.new_sga_workspace(shape, sh, sw)
    out = torch.full_like(q, float("nan"))
    G.sga_attn(shape, sh, sw, q, k, v, out, ws)
    torch.cuda.synchronize()
    G.check_device_error(ws)
    assert not torch.isnan(out).any()
    rows = sample_rows(geo.T, n_rows, seed=5, forced=PT.forced_rows(geo))
    ref = O.sga_attention(geo, x.q, x.k, x.v, sh, sw, rows=rows)
    PT.assert_close(out[torch.as_tensor(rows).cuda()], ref, f"{name} sga {sh}x{sw} sampled")
    del q, k, v, out, ws
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name,h0,h1", [("small", 4, 9), ("ref_small", 0, 8), ("k128_small", 11, 16)])
def test_head_slice_matches_full_layer(name, h0, h1):
    # head-parallel ranks run gsa_forward on their own heads only: heads are
    # independent in every step, so a slice of heads gives exactly those
    # heads of the full layer
    import sparse_global_attention_view_b200 as G
    x, geo, shape, st, res = case(name)
    full = G.GsaLayer(shape)(st.q, st.k, st.v, st.w)
    wl = CASES[name].with_(n_heads=h1 - h0)
    part_shape = G.Shape.of(wl)
    sl = lambda t: t[:, h0:h1].contiguous()  # noqa: E731
    part = G.GsaLayer(part_shape)(sl(st.q), sl(st.k), sl(st.v), st.w[h0:h1].contiguous())
    torch.cuda.synchronize()
    assert torch.equal(part, full[:, h0:h1]), "a head slice must reproduce those heads bit for bit"


def test_softmax_fma_exp2_error_bound():
    # the attention softmax takes a quarter of its exponentials as 2^x by
    # range reduction and a cubic on the FMA pipe; its stated bound is a
    # relative error below 7.5e-5 on [-125, 0] (the clamp at -125 included),
    # checked against the exact 2^x in float64 on a dense grid, the integers
    # and half-integers (the reduction's edges) and random points
    import sparse_global_attention_view_b200 as G
    grid = np.linspace(-125.0, 0.0, 1 << 20)
    edges = np.concatenate([np.arange(-125, 1, dtype=np.float64), np.arange(-124.5, 0, 1.0)])
    edges = np.concatenate([edges, np.nextafter(edges, -np.inf), np.nextafter(edges, np.inf)])
    rnd = np.random.default_rng(7).uniform(-125.0, 0.0, 1 << 18)
    x = np.concatenate([grid, edges, rnd]).astype(np.float32)
    x = x[(x >= -125.0) & (x <= 0.0)]
    xd = torch.from_numpy(x).cuda()
    y = torch.empty_like(xd)
    G.selftest_exp2(xd, y)
    torch.cuda.synchronize()
    got = y.cpu().numpy().astype(np.float64)
    exact = np.exp2(x.astype(np.float64))
    rel = np.abs(got - exact) / exact
    assert np.isfinite(got).all()
    assert rel.max() < 7.5e-5, f"max relative error {rel.max():.3e} at x = {x[rel.argmax()]}"
    # an odd count leaves the last element paired with nothing
    y3 = torch.full((3,), float("nan"), device="cuda")
    G.selftest_exp2(xd[:3].contiguous(), y3)
    torch.cuda.synchronize()
    assert torch.equal(y3, y[:3])


@pytest.mark.parametrize("name", ["small", "p3_ragged", "p1_nospecial", "p2_onehead", "one_frame", "ref_small",
                                  "ref_p3_ragged"])
def test_selection_is_the_exact_top_k_of_the_kernels_own_logits(name):
    # gsa_guide_logits dumps the logits the fused kernel ranks (tf32 products
    # of the fp32 means).  They must lie within tf32 rounding of the exact
    # products, and the kernel's selection must be exactly the top-K of them
    # (score descending, lower id on ties): no tie window is needed here.
    import sparse_global_attention_view_b200 as G
    x, geo, shape, st, res = case(name)
    if shape.top_k > 64:
        pytest.skip("two ranking passes")
    z = G.derive(shape)
    logits = torch.full((shape.n_heads, z.Tc, z.Tc), float("nan"), device="cuda")
    G.guide_logits(shape, st.qc32, st.kc32, st.vc, 0, z.Tc, logits, st.ws)
    torch.cuda.synchronize()
    G.check_device_error(st.ws)
    lg = logits.permute(1, 0, 2).double().cpu().numpy()  # [Tc, H, Tc]
    assert np.isfinite(lg).all()
    q64 = st.qc32.double().cpu()
    k64 = st.kc32.double().cpu()
    exact = torch.einsum("ahd,chd->ahc", q64, k64).numpy()
    mag = torch.einsum("ahd,chd->ahc", q64.abs(), k64.abs()).numpy()
    # tf32 keeps 10 explicit mantissa bits of each operand: below 2^-10
    # relative per factor even if truncated, so below 2^-9 per product, plus
    # the fp32 accumulation over 64 terms
    assert (np.abs(lg - exact) <= 2.0 ** -8 * mag + 1e-6).all(), f"{name}: logits beyond tf32 rounding"
    own = O.top_k_blocks(geo, O.guide_scores(geo, lg))
    assert np.array_equal(st.sel_by_entry(), own), f"{name}: selection is not the top-K of the kernel's logits"
    # a row range runs only its CTAs and gives the same values
    if z.Tc > 140:
        part = torch.full((shape.n_heads, 9, z.Tc), float("nan"), device="cuda")
        G.guide_logits(shape, st.qc32, st.kc32, st.vc, 131, 9, part, st.ws)
        torch.cuda.synchronize()
        assert torch.equal(part, logits[:, 131:140]), f"{name}: row range differs"


def test_guide_logits_rejects_bad_row_ranges():
    import sparse_global_attention_view_b200 as G
    x, geo, shape, st, res = case("small")
    z = G.derive(shape)
    for row0, n in ((-1, 4), (0, 0), (z.Tc - 3, 4)):
        out = torch.empty((shape.n_heads, n, z.Tc), device="cuda")
        with pytest.raises(G.GsaError):
            G.guide_logits(shape, st.qc32, st.kc32, st.vc, row0, n, out, st.ws)


def test_exact_ties_go_to_the_lower_block_id():
    # every frame a copy of frame 0: the blocks at one grid position in the
    # six frames have identical pooled keys, so each query's scores tie exactly
    # in groups of six and the K-th place falls inside a tie; the fused
    # kernel must keep the lower block ids of a tie, as the oracle's ranking
    # by (score descending, id ascending) does
    import sparse_global_attention_view_b200 as G
    wl = Workload("ties", 6, 2, 9, 10, 2, 64, 3, 7, 21, "gaussian")
    x = generate(wl)
    L = wl.n_special + wl.hp * wl.wp
    for t in (x.q, x.k, x.v):
        f = t.view(wl.n_frames, L, wl.n_heads, wl.head_dim)
        f[1:] = f[0]
    geo = O.geometry_of(wl)
    shape = G.Shape.of(wl)
    q, k, v, w = _dev(x)
    st = PT.Stages(shape, q, k, v, w, 1).run()
    z = G.derive(shape)
    logits = torch.full((shape.n_heads, z.Tc, z.Tc), float("nan"), device="cuda")
    G.guide_logits(shape, st.qc32, st.kc32, st.vc, 0, z.Tc, logits, st.ws)
    torch.cuda.synchronize()
    G.check_device_error(st.ws)
    guide = O.guide_scores(geo, logits.permute(1, 0, 2).double().cpu().numpy())
    srt = -np.sort(-guide, axis=-1)
    assert (srt[..., geo.K_eff - 1] == srt[..., geo.K_eff]).mean() > 0.5, "the K-th place should fall in a tie"
    own = O.top_k_blocks(geo, guide)
    assert np.array_equal(st.sel_by_entry(), own), "ties must go to the lower block id"
    # the whole layer's selection (gsa_forward) as well
    layer = G.GsaLayer(shape)
    layer(q, k, v, w)
    torch.cuda.synchronize()
    fwd = G.workspace_view(layer.ws, shape, "sel").permute(1, 0, 2).cpu().numpy()
    assert np.array_equal(fwd, own)
