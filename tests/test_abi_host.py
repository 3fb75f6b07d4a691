"""The C-ABI library on the host: it loads without a GPU, exports every function
include/gsa.h declares, derives sizes like the oracle's geometry, and rejects
bad arguments before launching anything (all calls below fail validation, so
no CUDA work is attempted)."""

import ctypes
import os
import re
import subprocess

import pytest

from oracle import gsa_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gsa.h")


@pytest.fixture(scope="module")
def lib():
    from sparse_global_attention_view_b200 import build
    build.build()
    from sparse_global_attention_view_b200 import _lib
    return _lib.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w]*\s*\*?\s+\**([A-Za-z_]\w*)\s*\(", text, flags=re.M)
    return sorted(set(names))


def declared_arity():
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    text = re.sub(r"^\s*#.*$", "", text, flags=re.M)  # preprocessor lines
    out = {}
    for m in re.finditer(r"([A-Za-z_]\w*)\s*\(([^;{]*?)\)\s*;", text):
        args = m.group(2).strip()
        out[m.group(1)] = 0 if args in ("", "void") else args.count(",") + 1
    return out


def test_binding_arity_matches_header():
    from sparse_global_attention_view_b200 import _lib
    arity = declared_arity()
    for name in declared_functions():
        assert len(_lib.SIGNATURES[name]) == arity[name], name


def test_header_declares_the_path():
    names = declared_functions()
    for want in ("gsa_pool_kv", "gsa_compressed_attn", "gsa_topk_blocks", "gsa_selected_attn",
                 "gsa_gate_combine", "dense_global_attn", "gsa_forward", "gsa_derive",
                 "gsa_workspace_size", "gsa_check_device_error", "gsa_status_string"):
        assert want in names


def test_every_declared_symbol_is_exported(lib):
    from sparse_global_attention_view_b200 import _lib
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for name in declared_functions():
        assert name in exported, name
        assert hasattr(lib, name)
        assert name in _lib.SIGNATURES, f"binding lacks {name}"


def shape(**kw):
    from sparse_global_attention_view_b200 import Shape
    base = dict(n_frames=3, n_special=5, hp=37, wp=37, n_heads=16, head_dim=64, pool=4, top_k=16)
    base.update(kw)
    return Shape(**base)


@pytest.mark.parametrize("kw", [
    dict(), dict(n_special=0, hp=16, wp=16, n_heads=2, top_k=4), dict(pool=1, hp=5, wp=7),
    dict(pool=3, hp=10, wp=11, n_special=1), dict(top_k=128, n_frames=1), dict(pool=2, hp=1, wp=9),
    dict(keep=1), dict(keep=1, n_frames=1), dict(keep=1, n_special=0, top_k=128),
    dict(keep=1, n_frames=40, top_k=128, pool=1, hp=3, wp=3)])
def test_derive_matches_oracle_geometry(lib, kw):
    from sparse_global_attention_view_b200 import derive
    s = shape(**kw)
    z = derive(s)
    g = O.Geometry(N=s.n_frames, S=s.n_special, Hp=s.hp, Wp=s.wp, H=s.n_heads, D=64, P=s.pool, K=s.top_k,
                   keep="reference" if s.keep == 1 else "specials")
    assert (z.T, z.Tc, z.NB, z.NS, z.L, z.E, z.Bh, z.Bw, z.Bf, z.K_eff) == \
        (g.T, g.Tc, g.NB, g.NS, g.L, g.E, g.Bh, g.Bw, g.Bf, g.K_eff)
    assert (z.NK, z.B0) == (g.kept_tokens().size, g.B0)


def test_workspace_size_grows_with_frames(lib):
    from sparse_global_attention_view_b200 import workspace_size
    a = workspace_size(shape(n_frames=2))
    b = workspace_size(shape(n_frames=20))
    assert 256 < a < b
    assert a % 256 == 0 and b % 256 == 0


@pytest.mark.parametrize("kw,status", [
    (dict(head_dim=32), 2), (dict(pool=5), 2), (dict(top_k=129), 2), (dict(n_heads=129), 2),
    (dict(n_frames=0), 1), (dict(hp=0), 1), (dict(top_k=0), 1), (dict(pool=0), 1),
    (dict(n_special=-1), 1), (dict(scale=-1.0), 1), (dict(scale=float("nan")), 1),
    (dict(keep=2), 1), (dict(keep=-1), 1),
    (dict(n_frames=2_000_000), 1)])
def test_bad_shapes_are_rejected(lib, kw, status):
    from sparse_global_attention_view_b200 import _lib
    z = _lib.GsaSizes()
    s = shape(**kw).c()
    assert lib.gsa_derive(ctypes.byref(s), ctypes.byref(z)) == status
    n = ctypes.c_size_t()
    assert lib.gsa_workspace_size(ctypes.byref(s), ctypes.byref(n)) == status


FAKE = 0x10000  # aligned, never dereferenced: every call below fails validation first


def test_null_and_misaligned_pointers_are_rejected(lib):
    s = shape().c()
    p = ctypes.c_void_p(FAKE)
    bad = ctypes.c_void_p(FAKE + 2)
    null = ctypes.c_void_p(0)
    st = ctypes.c_void_p(0)
    assert lib.gsa_forward(ctypes.byref(s), p, p, p, p, null, p, ctypes.c_size_t(1 << 40), st) == 1
    assert lib.gsa_forward(ctypes.byref(s), p, bad, p, p, p, p, ctypes.c_size_t(1 << 40), st) == 1
    assert lib.dense_global_attn(ctypes.byref(s), p, p, p, p, null, st) == 1
    assert lib.gsa_pool_kv(ctypes.byref(s), p, p, p, p, p, p, null, null, p, null, p, st) == 1
    assert lib.gsa_selected_attn(ctypes.byref(s), p, p, p, null, null, p, p, null, p, st) == 1
    assert lib.gsa_gate_combine(ctypes.byref(s), p, p, p, bad, p, p, st) == 1
    assert lib.gsa_topk_blocks(ctypes.byref(s), p, p, 0, p, p, st) == 1
    assert lib.gsa_topk_blocks(ctypes.byref(s), p, p, 200, p, p, st) == 1
    assert lib.gsa_compressed_attn(ctypes.byref(s), p, p, p, p, p, p, p, p, 65, p, st) == 1
    assert lib.gsa_check_device_error(null, st) == 1
    assert lib.gsa_workspace_init(bad, st) == 1
    assert lib.gsa_derive(None, None) == 1
    assert lib.gsa_selftest_exp2(null, p, 4, st) == 1
    assert lib.gsa_guide_logits(ctypes.byref(s), p, p, p, -1, 4, p, p, st) == 1
    assert lib.gsa_guide_logits(ctypes.byref(s), p, p, p, 0, 0, p, p, st) == 1
    assert lib.gsa_guide_logits(ctypes.byref(s), p, null, p, 0, 4, p, p, st) == 1
    assert lib.gsa_selftest_exp2(p, p, -1, st) == 1
    assert lib.frame_attn(ctypes.byref(s), p, p, bad, p, p, st) == 1
    assert lib.sga_attn(ctypes.byref(s), 2, 2, p, p, p, null, p, ctypes.c_size_t(1 << 40), st) == 1
    assert lib.sga_attn(ctypes.byref(s), 0, 2, p, p, p, p, p, ctypes.c_size_t(1 << 40), st) == 1
    assert lib.sga_attn(ctypes.byref(s), 2, -1, p, p, p, p, p, ctypes.c_size_t(1 << 40), st) == 1


def test_sga_workspace_size(lib):
    from sparse_global_attention_view_b200 import derive
    s = shape()
    n2, n4 = ctypes.c_size_t(), ctypes.c_size_t()
    assert lib.sga_workspace_size(ctypes.byref(s.c()), 2, 2, ctypes.byref(n2)) == 0
    assert lib.sga_workspace_size(ctypes.byref(s.c()), 4, 4, ctypes.byref(n4)) == 0
    assert n2.value > n4.value > 256 and n2.value % 256 == 0
    # the fp32 output over the kept keys dominates: T x H x 64 x 4 bytes at least
    z = derive(s)
    assert n4.value >= z.T * s.n_heads * 64 * 4
    assert lib.sga_workspace_size(ctypes.byref(s.c()), 0, 4, ctypes.byref(n4)) == 1
    assert lib.sga_workspace_size(ctypes.byref(s.c()), 4, 4, None) == 1
    p = ctypes.c_void_p(FAKE)
    assert lib.sga_attn(ctypes.byref(s.c()), 4, 4, p, p, p, p, p, ctypes.c_size_t(n4.value - 1),
                        ctypes.c_void_p(0)) == 3


def test_two_pass_workspace_is_larger(lib):
    # K in (64, 128] keeps two 64-wide selections and a 64-bit bound per row
    a, b = ctypes.c_size_t(), ctypes.c_size_t()
    assert lib.gsa_workspace_size(ctypes.byref(shape(top_k=64).c()), ctypes.byref(a)) == 0
    assert lib.gsa_workspace_size(ctypes.byref(shape(top_k=65).c()), ctypes.byref(b)) == 0
    assert b.value > a.value


def test_small_workspace_is_rejected(lib):
    s = shape().c()
    p = ctypes.c_void_p(FAKE)
    n = ctypes.c_size_t()
    assert lib.gsa_workspace_size(ctypes.byref(s), ctypes.byref(n)) == 0
    assert lib.gsa_forward(ctypes.byref(s), p, p, p, p, p, p, ctypes.c_size_t(n.value - 1),
                           ctypes.c_void_p(0)) == 3


def test_noalloc_rejects_shapes_beyond_its_scratch(lib):
    from sparse_global_attention_view_b200 import workspace_size
    from sparse_global_attention_view_b200._lib import NOALLOC_SCRATCH_BYTES
    big = shape(n_frames=100, top_k=32)
    assert workspace_size(big) > NOALLOC_SCRATCH_BYTES
    p = ctypes.c_void_p(FAKE)
    # rejected on the host before any CUDA call
    assert lib.gsa_forward_noalloc(ctypes.byref(big.c()), p, p, p, p, p, ctypes.c_void_p(0)) == 7
    assert b"noalloc" in lib.gsa_status_string(7)


def test_noalloc_limit_falls_between_four_and_five_vggt_frames(lib):
    """The fixed array holds the VGGT token layout (5 + 37x37 tokens per frame,
    16 heads, K = 16) up to 4 frames and no more: a layout change that moves
    this limit fails here, on the CPU."""
    from sparse_global_attention_view_b200 import workspace_size
    from sparse_global_attention_view_b200._lib import NOALLOC_SCRATCH_BYTES
    assert workspace_size(shape(n_frames=4, top_k=16)) <= NOALLOC_SCRATCH_BYTES
    assert workspace_size(shape(n_frames=5, top_k=16)) > NOALLOC_SCRATCH_BYTES


def test_negative_wait_limit_is_rejected(lib):
    import dataclasses
    s = dataclasses.replace(shape(), wait_limit_ns=-1)
    n = ctypes.c_size_t()
    assert lib.gsa_workspace_size(ctypes.byref(s.c()), ctypes.byref(n)) == 1


def test_status_strings(lib):
    for code in range(8):
        assert lib.gsa_status_string(code)
    assert b"unknown" in lib.gsa_status_string(99)


def test_python_binding_refuses_cpu_tensors(lib):
    import torch
    from sparse_global_attention_view_b200 import dense_global_attn
    s = shape(n_frames=1, n_special=0, hp=4, wp=4, n_heads=1, top_k=1)
    x = torch.zeros(16, 1, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        dense_global_attn(s, x, x, x, x, torch.zeros(256, dtype=torch.uint8))
