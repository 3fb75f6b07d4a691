"""ctypes view of libgsa.so (include/gsa.h).  Argument marshalling only."""

from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "lib", "libgsa.so")

c_i32 = ctypes.c_int32
c_f32 = ctypes.c_float
c_vp = ctypes.c_void_p
c_size = ctypes.c_size_t

GSA_OK = 0
STATUS_NAMES = {
    0: "GSA_OK",
    1: "GSA_ERR_INVALID_ARG",
    2: "GSA_ERR_UNSUPPORTED",
    3: "GSA_ERR_WORKSPACE",
    4: "GSA_ERR_CUDA",
    5: "GSA_ERR_TIMEOUT",
    6: "GSA_ERR_DEVICE_CHECK",
    7: "GSA_ERR_SCRATCH_LIMIT",
}
NOALLOC_SCRATCH_BYTES = 32 << 20
WS_HEADER_BYTES = 256


class GsaShape(ctypes.Structure):
    _fields_ = [
        ("n_frames", c_i32),
        ("n_special", c_i32),
        ("hp", c_i32),
        ("wp", c_i32),
        ("n_heads", c_i32),
        ("head_dim", c_i32),
        ("pool", c_i32),
        ("top_k", c_i32),
        ("scale", c_f32),
        ("keep", c_i32),
        ("wait_limit_ns", c_i32),
    ]


KEEP_SPECIALS = 0
KEEP_REFERENCE = 1


class GsaSizes(ctypes.Structure):
    _fields_ = [
        ("T", ctypes.c_int64),
        ("Tc", ctypes.c_int64),
        ("NB", ctypes.c_int64),
        ("NS", ctypes.c_int64),
        ("NK", ctypes.c_int64),
        ("B0", ctypes.c_int64),
        ("L", c_i32),
        ("E", c_i32),
        ("Bh", c_i32),
        ("Bw", c_i32),
        ("Bf", c_i32),
        ("K_eff", c_i32),
    ]


class GsaWsOffsets(ctypes.Structure):
    _fields_ = [(n, c_size) for n in ("qc32", "kc32", "vc", "qc", "kc", "ks", "vs", "oc",
                                      "cand_score", "cand_idx", "sel", "o_spec", "lse_spec",
                                      "total")] + [("n_split", c_i32), ("best", c_size), ("order", c_size)]


FORWARD_STEPS = ("pool", "compressed_attn", "block_scores", "topk_merge", "kept_attn", "selected_gate")

P_SHAPE = ctypes.POINTER(GsaShape)

# name -> argument types (all return gsa_status, an int, except gsa_status_string)
SIGNATURES = {
    "gsa_derive": [P_SHAPE, ctypes.POINTER(GsaSizes)],
    "gsa_workspace_size": [P_SHAPE, ctypes.POINTER(c_size)],
    "gsa_workspace_init": [c_vp, c_vp],
    "gsa_pool_kv": [P_SHAPE] + [c_vp] * 12,
    "gsa_compressed_attn": [P_SHAPE] + [c_vp] * 8 + [c_i32, c_vp, c_vp],
    "gsa_topk_blocks": [P_SHAPE, c_vp, c_vp, c_i32, c_vp, c_vp, c_vp],
    "gsa_guide_logits": [P_SHAPE, c_vp, c_vp, c_vp, ctypes.c_int64, c_i32, c_vp, c_vp, c_vp],
    "gsa_selected_attn": [P_SHAPE] + [c_vp] * 10,
    "gsa_gate_combine": [P_SHAPE] + [c_vp] * 7,
    "dense_global_attn": [P_SHAPE] + [c_vp] * 6,
    "dense_global_attn_mma": [P_SHAPE] + [c_vp] * 6,
    "frame_attn": [P_SHAPE] + [c_vp] * 6,
    "sga_workspace_size": [P_SHAPE, c_i32, c_i32, ctypes.POINTER(c_size)],
    "sga_attn": [P_SHAPE, c_i32, c_i32] + [c_vp] * 5 + [c_size, c_vp],
    "gsa_forward": [P_SHAPE] + [c_vp] * 6 + [c_size, c_vp],
    "gsa_forward_timed": [P_SHAPE] + [c_vp] * 6 + [c_size, c_vp, ctypes.POINTER(c_i32), c_vp],
    "gsa_workspace_offsets": [P_SHAPE, ctypes.POINTER(GsaWsOffsets)],
    "gsa_forward_noalloc": [P_SHAPE] + [c_vp] * 6,
    "gsa_noalloc_check_device_error": [c_vp],
    "gsa_check_device_error": [c_vp, c_vp],
    "gsa_selftest_exp2": [c_vp, c_vp, ctypes.c_int64, c_vp],
    "gsa_status_string": [c_i32],
    "gsa_last_cuda_error": [],
    "gsa_cuda_error_name": [c_i32],
}

_lib = None


def load() -> ctypes.CDLL:
    """Load libgsa.so; raises if it has not been built (there is no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m sparse_global_attention_view_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, args in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = ctypes.c_char_p if name in ("gsa_status_string", "gsa_cuda_error_name") else ctypes.c_int
        _lib = lib
    return _lib


class GsaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        lib = load()
        text = lib.gsa_status_string(status).decode()
        if status == 4:  # GSA_ERR_CUDA: name the CUDA error behind it
            code = lib.gsa_last_cuda_error()
            text += f": {lib.gsa_cuda_error_name(code).decode()} ({code})"
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)} ({text})")


def check(status: int, where: str) -> None:
    if status != GSA_OK:
        raise GsaError(status, where)
