"""The five seeded workloads and their generators.

Two generators:

* ``gaussian_inputs`` -- Q, K, V i.i.d. N(0, 1), drawn in the order Q, K, V,
  then the per-head gate vectors w ~ N(0, 1/64).
* ``scene_inputs`` -- a synthetic multi-view scene.  A table of 4096 unit
  latent vectors in R^1024 stands for the surface points of one scene; every
  frame sees a window of it shifted by (dy_f, dx_f) in [0, 8)^2, so patch
  (r, c) of frame f shows latent ((r + dy_f) * 64 + (c + dx_f)) mod 4096.  Each
  token is its latent plus N(0, sigma^2) noise per dimension; special tokens
  take a fresh unit latent of their own.  Q, K and V are Gaussian projections
  1024 -> H x 64 with entries N(0, (1/32)^2).  An optional second, disjoint
  latent table feeds a seeded 20% of the frames ("unrelated views").

Random draws come from ``numpy.random.default_rng`` (PCG64), so the same seed
gives the same tensors on every machine.  The draw order of the main stream is
fixed: latent table, second table (if any), shifts, picked frames (if any),
special-token latents, W_q, W_k, W_v, gate vectors.  Noise for frame f comes
from its own stream ``default_rng([seed, f])`` so frames can be generated in
any chunking with identical results.
"""

from __future__ import annotations

import dataclasses
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    n_frames: int
    n_special: int
    hp: int
    wp: int
    n_heads: int
    head_dim: int
    pool: int
    top_k: int
    seed: int
    kind: str  # "gaussian" | "scene"
    sigma: float = 0.3
    second_table_frac: float = 0.0
    # always-kept set of the selection branch (a layer option, not an input
    # property): 0 every special token, 1 frame 0 whole + each camera token
    keep: int = 0

    @property
    def tokens_per_frame(self) -> int:
        return self.n_special + self.hp * self.wp

    @property
    def n_tokens(self) -> int:
        return self.n_frames * self.tokens_per_frame

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS: dict[str, Workload] = {
    # N=2 frames, 16x16 grid, no special tokens, 2 heads, pool 4, top-K 4.
    "tiny": Workload("tiny", 2, 0, 16, 16, 2, 64, 4, 4, 0, "gaussian"),
    # VGGT-shaped: 37x37 patches + 5 special tokens per frame, 16 heads.
    "small": Workload("small", 8, 5, 37, 37, 16, 64, 4, 16, 1, "scene"),
    "medium": Workload("medium", 100, 5, 37, 37, 16, 64, 4, 32, 2, "scene"),
    "large": Workload("large", 300, 5, 37, 37, 16, 64, 4, 32, 3, "scene",
                      sigma=0.5, second_table_frac=0.2),
    "pages": Workload("pages", 1000, 5, 37, 37, 16, 64, 4, 64, 4, "scene"),
}


@dataclasses.dataclass
class Inputs:
    """Host tensors of one workload: bf16 [T, H, D] and fp32 gate vectors [H, D]."""

    workload: Workload
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    w: torch.Tensor


def _to_bf16(a: np.ndarray) -> torch.Tensor:
    # torch's float32 -> bfloat16 conversion rounds to nearest even.
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def gaussian_inputs(wl: Workload) -> Inputs:
    rng = np.random.default_rng(wl.seed)
    shape = (wl.n_tokens, wl.n_heads, wl.head_dim)
    q = _to_bf16(rng.standard_normal(shape))
    k = _to_bf16(rng.standard_normal(shape))
    v = _to_bf16(rng.standard_normal(shape))
    w = torch.from_numpy((rng.standard_normal((wl.n_heads, wl.head_dim)) / 8.0).astype(np.float32))
    return Inputs(wl, q, k, v, w)


def _unit_rows(rng: np.random.Generator, n: int, dim: int) -> np.ndarray:
    x = rng.standard_normal((n, dim))
    x /= np.linalg.norm(x, axis=1, keepdims=True)
    return x.astype(np.float32)


LATENT_ROWS = 4096
LATENT_DIM = 1024
LATENT_GRID = 64
MAX_SHIFT = 8


def scene_inputs(wl: Workload, threads: int | None = None) -> Inputs:
    rng = np.random.default_rng(wl.seed)
    table = _unit_rows(rng, LATENT_ROWS, LATENT_DIM)
    table2 = _unit_rows(rng, LATENT_ROWS, LATENT_DIM) if wl.second_table_frac > 0 else None
    shifts = rng.integers(0, MAX_SHIFT, size=(wl.n_frames, 2))
    uses_second = np.zeros(wl.n_frames, dtype=bool)
    if table2 is not None:
        n_pick = int(round(wl.second_table_frac * wl.n_frames))
        uses_second[rng.permutation(wl.n_frames)[:n_pick]] = True
    special_lat = _unit_rows(rng, wl.n_frames * wl.n_special, LATENT_DIM).reshape(
        wl.n_frames, wl.n_special, LATENT_DIM)
    hd = wl.n_heads * wl.head_dim
    w_qkv = np.concatenate(
        [(rng.standard_normal((LATENT_DIM, hd)) / 32.0).astype(np.float32) for _ in range(3)], axis=1)
    w = torch.from_numpy((rng.standard_normal((wl.n_heads, wl.head_dim)) / 8.0).astype(np.float32))

    L = wl.tokens_per_frame
    T = wl.n_tokens
    q = torch.empty((T, wl.n_heads, wl.head_dim), dtype=torch.bfloat16)
    k = torch.empty_like(q)
    v = torch.empty_like(q)

    rr, cc = np.meshgrid(np.arange(wl.hp), np.arange(wl.wp), indexing="ij")
    rr = rr.reshape(-1)
    cc = cc.reshape(-1)

    def frame_latents(f: int) -> np.ndarray:
        src = table2 if uses_second[f] else table
        dy, dx = int(shifts[f, 0]), int(shifts[f, 1])
        idx = ((rr + dy) * LATENT_GRID + (cc + dx)) % LATENT_ROWS
        x = np.empty((L, LATENT_DIM), dtype=np.float32)
        x[: wl.n_special] = special_lat[f]
        x[wl.n_special:] = src[idx]
        noise = np.random.default_rng([wl.seed, f]).standard_normal((L, LATENT_DIM), dtype=np.float32)
        x += np.float32(wl.sigma) * noise
        return x

    chunk = max(1, min(wl.n_frames, 32))

    def do_chunk(f0: int) -> None:
        f1 = min(wl.n_frames, f0 + chunk)
        x = np.concatenate([frame_latents(f) for f in range(f0, f1)], axis=0)
        y = torch.from_numpy(x) @ torch.from_numpy(w_qkv)  # float32 [rows, 3*H*D]
        y = y.view(-1, 3, wl.n_heads, wl.head_dim).to(torch.bfloat16)
        t0, t1 = f0 * L, f1 * L
        q[t0:t1] = y[:, 0]
        k[t0:t1] = y[:, 1]
        v[t0:t1] = y[:, 2]

    starts = list(range(0, wl.n_frames, chunk))
    if threads is None:
        threads = max(1, min(len(starts), os.cpu_count() or 1, 16))
    if threads > 1:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(do_chunk, starts))
    else:
        for s in starts:
            do_chunk(s)
    return Inputs(wl, q, k, v, w)


def generate(wl: Workload | str, **kw) -> Inputs:
    if isinstance(wl, str):
        wl = WORKLOADS[wl]
    if wl.kind == "gaussian":
        return gaussian_inputs(wl)
    if wl.kind == "scene":
        if wl.n_heads * wl.head_dim != LATENT_DIM:
            raise ValueError("scene model projects 1024 -> H*D; needs H*D == 1024")
        return scene_inputs(wl, **kw)
    raise ValueError(f"unknown workload kind {wl.kind!r}")


def sample_rows(n_tokens: int, n_rows: int, seed: int, forced: list[int] | None = None) -> np.ndarray:
    """Seeded query-row sample: ``forced`` rows first, then uniform without replacement."""
    forced = sorted(set(int(t) for t in (forced or []) if 0 <= t < n_tokens))
    rest = n_rows - len(forced)
    rng = np.random.default_rng([seed, 99])
    if rest > 0:
        pool = np.setdiff1d(np.arange(n_tokens), np.asarray(forced, dtype=np.int64))
        pick = rng.choice(pool, size=min(rest, pool.size), replace=False)
        rows = np.concatenate([np.asarray(forced, dtype=np.int64), pick])
    else:
        rows = np.asarray(forced[:n_rows], dtype=np.int64)
    return np.sort(rows)

