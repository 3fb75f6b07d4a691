"""The seeded input generators: reproducible, independent of how frames are
chunked over threads, and with the structure the workload statement describes
(patch (r, c) of frame f shows latent ((r + dy_f) * 64 + c + dx_f) mod 4096)."""

import numpy as np
import torch

from synthetic import WORKLOADS, generate
from synthetic import workloads as W


def test_scene_is_reproducible_and_independent_of_threads():
    wl = WORKLOADS["small"].with_(n_frames=3)
    a = W.scene_inputs(wl, threads=1)
    b = W.scene_inputs(wl, threads=3)
    for t in ("q", "k", "v", "w"):
        assert torch.equal(getattr(a, t), getattr(b, t))
    c = W.scene_inputs(wl.with_(seed=wl.seed + 1), threads=1)
    assert not torch.equal(a.q, c.q)


def test_scene_same_latent_tokens_align():
    # two frames see the same latent where their shifted grid positions agree;
    # without noise (sigma 0; at 0.3 per dimension the noise norm is ~10x the
    # unit latent's) their keys are then equal up to bf16 rounding
    wl = WORKLOADS["small"].with_(n_frames=4, sigma=0.0)
    x = generate(wl)
    rng = np.random.default_rng(wl.seed)
    W._unit_rows(rng, W.LATENT_ROWS, W.LATENT_DIM)  # the latent table, drawn first
    shifts = rng.integers(0, W.MAX_SHIFT, size=(wl.n_frames, 2))
    L, S = wl.tokens_per_frame, wl.n_special
    k = x.k.float().reshape(x.k.shape[0], -1)
    k = k / k.norm(dim=1, keepdim=True)
    same, other = [], []
    (dy0, dx0), (dy1, dx1) = shifts[0], shifts[1]
    for r in range(10, 20):
        for c in range(10, 20):
            r1, c1 = r + dy0 - dy1, c + dx0 - dx1  # frame 1's position of frame 0's latent
            t0 = S + r * wl.wp + c
            t1 = L + S + r1 * wl.wp + c1
            same.append(float(k[t0] @ k[t1]))
            other.append(float(k[t0] @ k[L + S + ((r + 7) % wl.hp) * wl.wp + (c + 11) % wl.wp]))
    assert min(same) > 0.999 and max(abs(v) for v in other) < 0.3


def test_gaussian_draws():
    x = generate("tiny")
    for t in (x.q, x.k, x.v):
        f = t.float()
        assert abs(float(f.mean())) < 0.02 and abs(float(f.std()) - 1.0) < 0.02
    assert abs(float(x.w.std()) - 1 / 8) < 0.04  # 128 draws
    assert x.q.shape == (512, 2, 64) and x.q.dtype == torch.bfloat16
