"""The bounded-wait timeout path on a B200, through the C ABI.

Every in-kernel wait of one pipeline role on another is bounded; a run whose
wait limit (gsa_shape.wait_limit_ns) is far shorter than a copy or a product
takes must give up, record GSA_ERR_TIMEOUT in the error word, drain its own
copies and products, free its tensor memory and return -- without trapping, so
that the next call on the same context is correct.  Nothing here faults or
hangs a GPU: the waits that run out are ordinary waits with a short limit.
"""

import dataclasses

import numpy as np
import pytest
import torch

import parity as PT
from oracle import gsa_oracle as O
from synthetic import WORKLOADS, generate

pytestmark = pytest.mark.gpu

SHORT_NS = 1  # far below the latency of any TMA copy or tensor-core product


def _inputs(name):
    import sparse_global_attention_view_b200 as G
    wl = WORKLOADS[name]
    x = generate(wl)
    return x, O.geometry_of(wl), G.Shape.of(wl), [t.cuda() for t in (x.q, x.k, x.v, x.w)]


def _expect_timeout(fn):
    import sparse_global_attention_view_b200 as G
    with pytest.raises(G.GsaError) as e:
        fn()
    assert e.value.status == 5, f"expected GSA_ERR_TIMEOUT, got {e.value}"


def test_dense_attention_wait_runs_out_then_recovers():
    import sparse_global_attention_view_b200 as G
    x, geo, shape, (q, k, v, w) = _inputs("tiny")
    short = dataclasses.replace(shape, wait_limit_ns=SHORT_NS)
    ws = G.new_workspace(None)
    out = torch.empty_like(q)
    G.dense_global_attn(short, q, k, v, out, ws)
    _expect_timeout(lambda: G.check_device_error(ws))
    G.check_device_error(ws)  # read and cleared: clean now
    out = torch.full_like(q, float("nan"))
    G.dense_global_attn(shape, q, k, v, out, ws)
    G.check_device_error(ws)
    PT.assert_close(out, O.dense_attention(geo, x.q, x.k, x.v), "dense after a timed-out call")


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_layer_wait_runs_out_then_recovers(name):
    import sparse_global_attention_view_b200 as G
    x, geo, shape, (q, k, v, w) = _inputs(name)
    short = dataclasses.replace(shape, wait_limit_ns=SHORT_NS)
    ws = G.new_workspace(shape)
    out = torch.empty_like(q)
    G.forward(short, q, k, v, w, out, ws)
    _expect_timeout(lambda: G.check_device_error(ws))
    layer = G.GsaLayer(shape)
    out = torch.full_like(q, float("nan"))
    layer(q, k, v, w, out)
    G.check_device_error(layer.ws)
    sel = G.workspace_view(layer.ws, shape, "sel").permute(1, 0, 2).contiguous().cpu().numpy()
    rows = np.arange(geo.T) if geo.T <= 2048 else np.sort(np.random.default_rng(3).choice(geo.T, 2048, replace=False))
    res = O.gsa_layer(geo, x.q, x.k, x.v, x.w, rows=rows, sel_override=sel)
    PT.assert_selection(res, f"{name} after a timed-out call")
    PT.assert_close(out[torch.as_tensor(rows).cuda()], res["out"], f"{name} after a timed-out call")


def test_noalloc_error_word_reports_the_timeout():
    import sparse_global_attention_view_b200 as G
    x, geo, shape, (q, k, v, w) = _inputs("tiny")
    short = dataclasses.replace(shape, wait_limit_ns=SHORT_NS)
    out = torch.empty_like(q)
    G.forward_noalloc(short, q, k, v, w, out)
    _expect_timeout(lambda: G.noalloc_check_device_error())
    out = torch.full_like(q, float("nan"))
    G.forward_noalloc(shape, q, k, v, w, out)
    G.noalloc_check_device_error()
    layer = G.GsaLayer(shape)
    PT.assert_close(out, layer(q, k, v, w).double().cpu().numpy(), "no-alloc after a timed-out call")
