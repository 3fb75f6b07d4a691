"""Thin Python binding of libgsa: torch tensors in, C-ABI calls out.

Every function here only checks tensor placement, dtype, contiguity and size,
turns tensors into device pointers and calls the entry point of the same name
in ``include/gsa.h``; all arithmetic runs in the library's CUDA kernels.  There
is no CPU fallback: a missing library or a CPU tensor raises.
"""

from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch

from ._lib import FORWARD_STEPS, GsaShape, GsaSizes, GsaWsOffsets, WS_HEADER_BYTES, check, load

BF16 = torch.bfloat16
F32 = torch.float32
I32 = torch.int32


@dataclass(frozen=True)
class Shape:
    """One layer call's sizes (``gsa_shape``)."""

    n_frames: int
    n_special: int
    hp: int
    wp: int
    n_heads: int
    head_dim: int = 64
    pool: int = 4
    top_k: int = 16
    scale: float = 0.0
    keep: int = 0  # 0: every special token always kept; 1: frame 0 + camera tokens
    wait_limit_ns: int = 0  # 0: default in-kernel wait limit (about 2 s); tiny values test the timeout path

    def c(self) -> GsaShape:
        return GsaShape(self.n_frames, self.n_special, self.hp, self.wp, self.n_heads,
                        self.head_dim, self.pool, self.top_k, float(self.scale), self.keep,
                        self.wait_limit_ns)

    @staticmethod
    def of(workload) -> "Shape":
        return Shape(workload.n_frames, workload.n_special, workload.hp, workload.wp,
                     workload.n_heads, workload.head_dim, workload.pool, workload.top_k,
                     keep=getattr(workload, "keep", 0))


def derive(shape: Shape) -> GsaSizes:
    z = GsaSizes()
    check(load().gsa_derive(ctypes.byref(shape.c()), ctypes.byref(z)), "gsa_derive")
    return z


def workspace_size(shape: Shape) -> int:
    n = ctypes.c_size_t()
    check(load().gsa_workspace_size(ctypes.byref(shape.c()), ctypes.byref(n)), "gsa_workspace_size")
    return n.value


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t, dtype, numel, name, optional=False):
    if t is None:
        if optional:
            return None
        raise ValueError(f"{name} is required")
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if numel is not None and t.numel() != numel:
        raise ValueError(f"{name} has {t.numel()} elements, expected {numel}")
    return ctypes.c_void_p(t.data_ptr())


def _ws(ws, min_bytes=WS_HEADER_BYTES):
    if not isinstance(ws, torch.Tensor) or not ws.is_cuda or not ws.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    if ws.numel() * ws.element_size() < min_bytes:
        raise ValueError(f"workspace holds {ws.numel() * ws.element_size()} bytes, needs {min_bytes}")
    return ctypes.c_void_p(ws.data_ptr())


def new_workspace(shape: Shape | None = None, device="cuda", stream=None) -> torch.Tensor:
    """A zeroed workspace: the forward's size for ``shape``, else just the header."""
    n = workspace_size(shape) if shape is not None else WS_HEADER_BYTES
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    check(load().gsa_workspace_init(ctypes.c_void_p(ws.data_ptr()), _stream(stream)),
          "gsa_workspace_init")
    return ws


def pool_kv(shape, q, k, v, qc32, kc32, vc, qc=None, kc=None, ks=None, vs=None, ws=None, stream=None):
    z = derive(shape)
    tok = z.T * shape.n_heads * shape.head_dim
    ent = z.Tc * shape.n_heads * shape.head_dim
    spc = z.NK * shape.n_heads * shape.head_dim
    check(load().gsa_pool_kv(
        ctypes.byref(shape.c()), _ptr(q, BF16, tok, "q"), _ptr(k, BF16, tok, "k"), _ptr(v, BF16, tok, "v"),
        _ptr(qc32, F32, ent, "qc32"), _ptr(kc32, F32, ent, "kc32"), _ptr(vc, BF16, ent, "vc"),
        _ptr(qc, BF16, ent, "qc", True), _ptr(kc, BF16, ent, "kc", True),
        _ptr(ks, BF16, spc, "ks", True), _ptr(vs, BF16, spc, "vs", True), _ws(ws), _stream(stream)),
        "gsa_pool_kv")


def compressed_attn(shape, qc, kc, vc, qc32, kc32, oc, cand_score, cand_idx, n_split, ws, stream=None):
    z = derive(shape)
    ent = z.Tc * shape.n_heads * shape.head_dim
    cand = shape.n_heads * z.Tc * n_split * shape.top_k
    check(load().gsa_compressed_attn(
        ctypes.byref(shape.c()), _ptr(qc, BF16, ent, "qc"), _ptr(kc, BF16, ent, "kc"),
        _ptr(vc, BF16, ent, "vc"), _ptr(qc32, F32, ent, "qc32"), _ptr(kc32, F32, ent, "kc32"),
        _ptr(oc, F32, ent, "oc"), _ptr(cand_score, F32, cand, "cand_score"),
        _ptr(cand_idx, I32, cand, "cand_idx"), ctypes.c_int32(n_split), _ws(ws), _stream(stream)),
        "gsa_compressed_attn")


def topk_blocks(shape, cand_score, cand_idx, n_split, sel, ws, stream=None):
    z = derive(shape)
    cand = shape.n_heads * z.Tc * n_split * shape.top_k
    check(load().gsa_topk_blocks(
        ctypes.byref(shape.c()), _ptr(cand_score, F32, cand, "cand_score"),
        _ptr(cand_idx, I32, cand, "cand_idx"), ctypes.c_int32(n_split),
        _ptr(sel, I32, shape.n_heads * z.Tc * shape.top_k, "sel"), _ws(ws), _stream(stream)),
        "gsa_topk_blocks")


def guide_logits(shape, qc32, kc32, vc, row0, n_rows, logits, ws, stream=None):
    """The fused kernel's own unscaled compressed logits for rows [row0, row0 + n_rows):
    logits [H][n_rows][Tc] fp32 (gsa_guide_logits)."""
    z = derive(shape)
    n = shape.n_heads * z.Tc * shape.head_dim
    check(load().gsa_guide_logits(
        ctypes.byref(shape.c()), _ptr(qc32, F32, n, "qc32"), _ptr(kc32, F32, n, "kc32"),
        _ptr(vc, BF16, n, "vc"), ctypes.c_int64(row0), ctypes.c_int32(n_rows),
        _ptr(logits, F32, shape.n_heads * n_rows * z.Tc, "logits"), _ws(ws), _stream(stream)),
        "gsa_guide_logits")


def selected_attn(shape, q, k, v, ks, vs, sel, o_sel, lse=None, ws=None, stream=None):
    z = derive(shape)
    tok = z.T * shape.n_heads * shape.head_dim
    spc = z.NK * shape.n_heads * shape.head_dim
    need_sp = z.NK > 0
    check(load().gsa_selected_attn(
        ctypes.byref(shape.c()), _ptr(q, BF16, tok, "q"), _ptr(k, BF16, tok, "k"), _ptr(v, BF16, tok, "v"),
        _ptr(ks, BF16, spc, "ks", not need_sp), _ptr(vs, BF16, spc, "vs", not need_sp),
        _ptr(sel, I32, shape.n_heads * z.Tc * shape.top_k, "sel"), _ptr(o_sel, BF16, tok, "o_sel"),
        _ptr(lse, F32, z.T * shape.n_heads, "lse", True), _ws(ws), _stream(stream)),
        "gsa_selected_attn")


def gate_combine(shape, qc32, w, oc, o_sel, out, ws, stream=None):
    z = derive(shape)
    tok = z.T * shape.n_heads * shape.head_dim
    ent = z.Tc * shape.n_heads * shape.head_dim
    check(load().gsa_gate_combine(
        ctypes.byref(shape.c()), _ptr(qc32, F32, ent, "qc32"),
        _ptr(w, F32, shape.n_heads * shape.head_dim, "w"), _ptr(oc, F32, ent, "oc"),
        _ptr(o_sel, BF16, tok, "o_sel"), _ptr(out, BF16, tok, "out"), _ws(ws), _stream(stream)),
        "gsa_gate_combine")


def dense_global_attn(shape, q, k, v, out, ws, stream=None):
    z = derive(shape)
    tok = z.T * shape.n_heads * shape.head_dim
    check(load().dense_global_attn(
        ctypes.byref(shape.c()), _ptr(q, BF16, tok, "q"), _ptr(k, BF16, tok, "k"), _ptr(v, BF16, tok, "v"),
        _ptr(out, BF16, tok, "out"), _ws(ws), _stream(stream)), "dense_global_attn")


def frame_attn(shape, q, k, v, out, ws, stream=None):
    """Attention of every token over the tokens of its own frame only."""
    z = derive(shape)
    tok = z.T * shape.n_heads * shape.head_dim
    check(load().frame_attn(
        ctypes.byref(shape.c()), _ptr(q, BF16, tok, "q"), _ptr(k, BF16, tok, "k"), _ptr(v, BF16, tok, "v"),
        _ptr(out, BF16, tok, "out"), _ws(ws), _stream(stream)), "frame_attn")


def sga_workspace_size(shape, sub_h: int, sub_w: int) -> int:
    n = ctypes.c_size_t()
    check(load().sga_workspace_size(ctypes.byref(shape.c()), ctypes.c_int32(sub_h), ctypes.c_int32(sub_w),
                                    ctypes.byref(n)), "sga_workspace_size")
    return n.value


def new_sga_workspace(shape, sub_h: int, sub_w: int, device=None, stream=None) -> torch.Tensor:
    """Zero-headed workspace for sga_attn."""
    ws = torch.empty(sga_workspace_size(shape, sub_h, sub_w), dtype=torch.uint8, device=device or "cuda")
    check(load().gsa_workspace_init(ctypes.c_void_p(ws.data_ptr()), _stream(stream)), "gsa_workspace_init")
    return ws


def sga_attn(shape, sub_h: int, sub_w: int, q, k, v, out, ws, stream=None):
    """Subsampled global attention (AVGGT SGA) over sub_h x sub_w windows."""
    z = derive(shape)
    tok = z.T * shape.n_heads * shape.head_dim
    check(load().sga_attn(
        ctypes.byref(shape.c()), ctypes.c_int32(sub_h), ctypes.c_int32(sub_w),
        _ptr(q, BF16, tok, "q"), _ptr(k, BF16, tok, "k"), _ptr(v, BF16, tok, "v"),
        _ptr(out, BF16, tok, "out"), _ws(ws), ctypes.c_size_t(ws.numel()), _stream(stream)), "sga_attn")


def dense_global_attn_mma(shape, q, k, v, out, ws, stream=None):
    """dense_global_attn on the warp-level mma.sync path (the measured baseline)."""
    z = derive(shape)
    tok = z.T * shape.n_heads * shape.head_dim
    check(load().dense_global_attn_mma(
        ctypes.byref(shape.c()), _ptr(q, BF16, tok, "q"), _ptr(k, BF16, tok, "k"), _ptr(v, BF16, tok, "v"),
        _ptr(out, BF16, tok, "out"), _ws(ws), _stream(stream)), "dense_global_attn_mma")


def forward(shape, q, k, v, w, out, ws, stream=None):
    z = derive(shape)
    tok = z.T * shape.n_heads * shape.head_dim
    need = workspace_size(shape)
    check(load().gsa_forward(
        ctypes.byref(shape.c()), _ptr(q, BF16, tok, "q"), _ptr(k, BF16, tok, "k"), _ptr(v, BF16, tok, "v"),
        _ptr(w, F32, shape.n_heads * shape.head_dim, "w"), _ptr(out, BF16, tok, "out"), _ws(ws, need),
        ctypes.c_size_t(ws.numel() * ws.element_size()), _stream(stream)), "gsa_forward")


def forward_noalloc(shape, q, k, v, w, out, stream=None) -> None:
    """``forward`` without a workspace: the intermediates use the library's
    fixed device array (for callers that cannot allocate; see gsa.h).  Calls
    on one device share that array, so they must not overlap on the GPU."""
    z = derive(shape)
    tok = z.T * shape.n_heads * shape.head_dim
    check(load().gsa_forward_noalloc(
        ctypes.byref(shape.c()), _ptr(q, BF16, tok, "q"), _ptr(k, BF16, tok, "k"), _ptr(v, BF16, tok, "v"),
        _ptr(w, F32, shape.n_heads * shape.head_dim, "w"), _ptr(out, BF16, tok, "out"), _stream(stream)),
        "gsa_forward_noalloc")


def noalloc_check_device_error(stream=None) -> None:
    """Synchronise, then read and clear the error word of the fixed array that
    ``forward_noalloc`` uses on the current device; raises on a device error."""
    check(load().gsa_noalloc_check_device_error(_stream(stream)), "gsa_noalloc_check_device_error")


def forward_timed(shape, q, k, v, w, out, ws, events, stream=None) -> int:
    """``forward`` recording ``events`` (len(FORWARD_STEPS) + 1 torch.cuda.Event
    with timing, already recorded once so their handles exist) between its
    kernels; returns the number of kernels enqueued."""
    z = derive(shape)
    tok = z.T * shape.n_heads * shape.head_dim
    need = workspace_size(shape)
    if len(events) != len(FORWARD_STEPS) + 1:
        raise ValueError(f"need {len(FORWARD_STEPS) + 1} events")
    handles = (ctypes.c_void_p * len(events))(*[ctypes.c_void_p(e.cuda_event) for e in events])
    n = ctypes.c_int32()
    check(load().gsa_forward_timed(
        ctypes.byref(shape.c()), _ptr(q, BF16, tok, "q"), _ptr(k, BF16, tok, "k"), _ptr(v, BF16, tok, "v"),
        _ptr(w, F32, shape.n_heads * shape.head_dim, "w"), _ptr(out, BF16, tok, "out"), _ws(ws, need),
        ctypes.c_size_t(ws.numel() * ws.element_size()), handles, ctypes.byref(n), _stream(stream)),
        "gsa_forward_timed")
    return n.value


def workspace_offsets(shape) -> GsaWsOffsets:
    o = GsaWsOffsets()
    check(load().gsa_workspace_offsets(ctypes.byref(shape.c()), ctypes.byref(o)), "gsa_workspace_offsets")
    return o


def workspace_view(ws, shape, name: str) -> torch.Tensor:
    """A typed view of one of gsa_forward's intermediates inside ``ws``."""
    z = derive(shape)
    o = workspace_offsets(shape)
    H, D, K = shape.n_heads, shape.head_dim, shape.top_k
    spec = {
        "qc32": (F32, (z.Tc, H, D)), "kc32": (F32, (z.Tc, H, D)), "vc": (BF16, (z.Tc, H, D)),
        "qc": (BF16, (z.Tc, H, D)), "kc": (BF16, (z.Tc, H, D)), "ks": (BF16, (H, z.NK, D)),
        "vs": (BF16, (H, z.NK, D)), "oc": (F32, (z.Tc, H, D)),
        "cand_score": (F32, (H, z.Tc, o.n_split, K)), "cand_idx": (I32, (H, z.Tc, o.n_split, K)),
        "sel": (I32, (H, z.Tc, K)),
        "o_spec": (F32, (z.T if z.NK else 0, H, D)), "lse_spec": (F32, (z.T if z.NK else 0, H)),
        "best": (I32, (H, z.Tc)), "order": (I32, (H * z.Tc,)),
    }[name]
    dtype, shp = spec
    n = 1
    for s in shp:
        n *= s
    off = getattr(o, name)
    nbytes = n * torch.tensor([], dtype=dtype).element_size()
    return ws[off:off + nbytes].view(dtype).view(shp)


def selftest_exp2(x, y, stream=None) -> None:
    """y[i] = the softmax's FMA-pipe 2^x[i] on the device (gsa_selftest_exp2); x, y cuda float32."""
    n = x.numel()
    check(load().gsa_selftest_exp2(_ptr(x, torch.float32, n, "x"), _ptr(y, torch.float32, n, "y"), n, _stream(stream)),
          "gsa_selftest_exp2")


def check_device_error(ws, stream=None) -> None:
    """Raise GsaError if a kernel set the workspace's error word (then cleared).
    A timeout's message carries where the first wait ran out (header words 1-2:
    the barrier's shared-memory address | 1, threadIdx.x << 8 | parity)."""
    p = _ws(ws)
    where = ""
    st = torch.cuda.current_stream() if stream is None else stream
    st.synchronize()
    hdr = ws[:12].view(torch.int32).cpu().tolist() if ws.numel() >= 12 else []
    if hdr and hdr[1] != 0:
        where = f" (first wait out: barrier smem 0x{hdr[1] & ~1:x}, thread {hdr[2] >> 8}, parity {hdr[2] & 255})"
    check(load().gsa_check_device_error(p, _stream(stream)), "gsa_check_device_error" + where)


class GsaLayer:
    """Convenience owner of a workspace for repeated ``forward`` calls of one shape."""

    def __init__(self, shape: Shape, device="cuda"):
        self.shape = shape
        self.sizes = derive(shape)
        self.ws = new_workspace(shape, device)

    def __call__(self, q, k, v, w, out=None, stream=None):
        if out is None:
            out = torch.empty_like(q)
        forward(self.shape, q, k, v, w, out, self.ws, stream)
        return out
