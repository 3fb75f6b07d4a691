"""gsa_forward_noalloc against gsa_forward, through the C ABI (needs a B200).

Some callers cannot allocate device memory: a host application whose memory
manager owns all of the GPU's memory, or a latency-critical loop where a
cudaMalloc would synchronise the device.  gsa_forward_noalloc serves them from
a fixed device array inside the library instead of a caller workspace.  Here
its output must match the workspace entry point's within the parity
tolerances, on two calls in a row with different inputs (the second call runs
on the scratch the first one left behind).

This file sorts last so that a run stopping at its first failure has already
run every other test; it also passes on its own in a fresh process.
"""

import pytest
import torch

import parity as PT
from synthetic import WORKLOADS, generate

pytestmark = pytest.mark.gpu


def _device_inputs(wl):
    x = generate(wl)
    return [t.cuda() for t in (x.q, x.k, x.v, x.w)]


# Tiny, and the VGGT token layout (37x37 patches + 5 special tokens, 16
# heads) at 4 frames, the largest frame count whose workspace fits the array.
CASES = {"tiny": WORKLOADS["tiny"],
         "vggt_4_frames": WORKLOADS["small"].with_(name="vggt_4_frames", n_frames=4)}


@pytest.mark.parametrize("name", list(CASES))
def test_noalloc_matches_workspace_forward_on_two_calls(name):
    import sparse_global_attention_view_b200 as G
    from sparse_global_attention_view_b200._lib import NOALLOC_SCRATCH_BYTES

    wl = CASES[name]
    shape = G.Shape.of(wl)
    assert G.workspace_size(shape) <= NOALLOC_SCRATCH_BYTES
    layer = G.GsaLayer(shape)
    for call, seed in enumerate((wl.seed, wl.seed + 17)):
        q, k, v, w = _device_inputs(wl.with_(seed=seed))
        ref = layer(q, k, v, w)
        out = torch.full_like(q, float("nan"))
        G.forward_noalloc(shape, q, k, v, w, out)
        torch.cuda.synchronize()
        G.check_device_error(layer.ws)       # the workspace call
        G.noalloc_check_device_error()       # the no-alloc call's own error word
        PT.assert_close(out, ref.double().cpu().numpy(), f"{name} noalloc call {call + 1}")
