"""Plant plausible mistakes in the oracle (on the CPU) and check the pins catch each.

A pin set that still passes with a dropped term, a wrong sign or index, or a
swapped operand would not be worth much; every mutation below must make at
least one pin in ``pins.py`` fail.
"""

import os
import sys
import warnings

import numpy as np
import pytest
import torch

import pins
from oracle import gsa_oracle as O

FIXTURE = os.path.join(os.path.dirname(__file__), "golden", "block_structure_37x37_p4.txt")


def _pool_full_denominator(geo, X, frames_per_chunk=None):
    out = _orig["pool"](geo, X, frames_per_chunk)
    # re-weight every block entry as if it always held P*P patches
    for f in range(geo.N):
        for br in range(geo.Bh):
            for bc in range(geo.Bw):
                rows, cols = geo.block_rows_cols(br, bc)
                out[f * geo.E + geo.S + br * geo.Bw + bc] *= len(rows) * len(cols) / (geo.P * geo.P)
    return out


def _compressed_values_are_keys(geo, Qc_rows, Kc, Vc):
    return _orig["compressed_attention"](geo, Qc_rows, Kc, Kc)


def _top_k_ties_high(geo, guide):
    rows, H, NB = guide.shape
    sel = np.full((rows, H, geo.K), -1, dtype=np.int64)
    ids = np.arange(NB)
    for a in range(rows):
        for h in range(H):
            order = np.lexsort((-ids, -guide[a, h]))
            sel[a, h, :geo.K_eff] = np.sort(order[:geo.K_eff])
    return sel


def _kept_nothing(self):
    return np.zeros(0, dtype=np.int64)


def _kept_twice(self):
    once = _orig["Geometry.kept_tokens"](self)
    return np.concatenate([once, once])


def _selected_keys_drop_last_block(geo, sel_row):
    chosen = [b for b in sel_row if b >= 0][:-1]
    return _orig["selected_keys"](geo, np.asarray(chosen, dtype=np.int64))


def _combine_swapped(g, o_cmp_up, o_sel):
    return _orig["combine"](g, o_sel, o_cmp_up)


def _combine_no_one_minus(g, o_cmp_up, o_sel):
    return g[..., None] * o_cmp_up + o_sel


def _guide_counts_specials(geo, logits):
    return logits[..., :geo.NB]


def _entry_of_token_shifted(self, t):
    f, i = divmod(int(t), self.L)
    if i < self.S:
        return f * self.E + i
    r, c = divmod(i - self.S, self.Wp)
    return f * self.E + self.S + (r // self.P) * self.Bw + min((c + 1) // self.P, self.Bw - 1)


def _block_rows_cols_short(self, br, bc):
    return (range(self.P * br, min(self.P * br + self.P, self.Hp - 1)) if br == self.Bh - 1
            else range(self.P * br, self.P * br + self.P),
            range(self.P * bc, min(self.P * bc + self.P, self.Wp)))


def _frame_attention_next_frame(geo, Q, K, V, rows=None):
    # attends to the following frame's tokens (wrong key range)
    rows = np.arange(geo.T) if rows is None else np.asarray(rows, dtype=np.int64)
    out = np.empty((rows.size, geo.H, geo.D))
    for n, t in enumerate(rows):
        f = (int(t) // geo.L + 1) % geo.N
        keys = slice(f * geo.L, (f + 1) * geo.L)
        out[n] = O.weighted_values(O.softmax(O.qk_logits(O.f64(Q, [t]), O.f64(K, keys), geo.sm_scale)),
                                   O.f64(V, keys))[0]
    return out


def _kept_all_specials_of_later_frames(self):
    # reference keep that also keeps the register tokens of frames 1..N-1
    if self.keep != "reference":
        return _orig["Geometry.kept_tokens"](self)
    later = [self.special_token(f, j) for f in range(1, self.N) for j in range(self.S)]
    return np.array(list(range(self.L)) + later, dtype=np.int64)


def _kept_camera_from_last_slot(self):
    if self.keep != "reference":
        return _orig["Geometry.kept_tokens"](self)
    cams = [self.special_token(f, self.S - 1) for f in range(1, self.N)] if self.S > 0 else []
    return np.array(list(range(self.L)) + cams, dtype=np.int64)


def _dense_sliced_drops_last_slice(geo, Q, K, V, rows=None, key_chunk=1 << 14, max_bytes=1 << 30):
    if geo.T <= key_chunk:
        return _orig["dense_attention"](geo, Q, K, V, rows, key_chunk, max_bytes)
    # the keys of the ragged last slice are lost
    rows = np.arange(geo.T) if rows is None else np.asarray(rows)
    n = (geo.T - 1) // key_chunk * key_chunk
    k, v = O.f64(K, slice(0, n)), O.f64(V, slice(0, n))
    return O.weighted_values(O.softmax(O.qk_logits(O.f64(Q, rows), k, geo.sm_scale)), v)


def _sga_centre_sample(geo, sub_h, sub_w):
    keep = np.zeros((geo.Hp, geo.Wp), dtype=bool)
    keep[sub_h // 2::sub_h, sub_w // 2::sub_w] = True
    return keep


def _sga_without_mean_pair(geo, Q, K, V, sub_h, sub_w, rows=None):
    # the dropped columns simply vanish: SGA with the mean pair's logit at -inf
    rows = np.arange(geo.T) if rows is None else np.asarray(rows, dtype=np.int64)
    kept = O.sga_key_tokens(geo, sub_h, sub_w)
    out = np.empty((rows.size, geo.H, geo.D))
    for i, t in enumerate(rows):
        keys = kept if t in set(kept.tolist()) else np.append(kept, t)
        s_ = O.qk_logits(O.f64(Q, [t]), O.f64(K, keys), geo.sm_scale)
        out[i] = O.weighted_values(O.softmax(s_), O.f64(V, keys))[0]
    return out


def _sga_diagonal_twice(geo, Q, K, V, sub_h, sub_w, rows=None):
    # the own key is added even when it is already a sampled key
    rows = np.arange(geo.T) if rows is None else np.asarray(rows, dtype=np.int64)
    kept = O.sga_key_tokens(geo, sub_h, sub_w)
    is_kept = np.zeros(geo.T, dtype=bool)
    is_kept[kept] = True
    dropped = np.flatnonzero(~is_kept)
    out = np.empty((rows.size, geo.H, geo.D))
    for i, t in enumerate(rows):
        keys = np.append(kept, t)
        k, v = O.f64(K, keys), O.f64(V, keys)
        if dropped.size:
            k = np.concatenate([k, O.f64(K, dropped).mean(axis=0, keepdims=True)])
            v = np.concatenate([v, O.f64(V, dropped).mean(axis=0, keepdims=True)])
        out[i] = O.weighted_values(O.softmax(O.qk_logits(O.f64(Q, [t]), k, geo.sm_scale)), v)[0]
    return out


def _gate_wrong_sign(geo, Qc_rows, w):
    return 1.0 - _orig["gate"](geo, Qc_rows, w)


def _fine_queries_against_fine_keys(geo, Q, Kc, Vc, rows):
    # the A1 variant attending to the unpooled keys and values instead
    r = np.asarray(rows, dtype=np.int64)
    q = O.f64(Q, r)
    return O.weighted_values(O.softmax(O.qk_logits(q, O.f64(Q, np.arange(geo.T)), geo.sm_scale)),
                             O.f64(Q, np.arange(geo.T)))


def _token_gate_from_pooled_query(geo, Q, rows, w):
    # the A10 variant falling back to the pooled query of the token's block
    r = np.asarray(rows, dtype=np.int64)
    qc = O.pool(geo, Q)
    return O.gate(geo, qc[[geo.entry_of_token(int(t)) for t in r]], w)


def _softmax_torch_wrong_axis(z, axis=-1):
    # the threaded (large-array) form normalises over the first axis
    z = np.asarray(z, dtype=np.float64)
    if z.size < O.CHUNKS.softmax_torch_elems:
        return _orig["softmax"](z, axis)
    t = torch.from_numpy(z)
    e = torch.exp(t - torch.amax(t, dim=0, keepdim=True))
    return (e / torch.sum(e, dim=0, keepdim=True)).numpy()


def _spans_mistake(caller, how):
    """spans() that, only when called from ``caller`` and only when the work is
    really split, drops the last slice or skips the first element of every
    slice after the first (an off-by-one at the boundaries)."""
    def mutated(n, step):
        out = _orig["spans"](n, step)
        if sys._getframe(1).f_code.co_name != caller or len(out) < 2:
            return out
        if how == "drop_last":
            return out[:-1]
        return [(a + (1 if i else 0), b) for i, (a, b) in enumerate(out)]
    return mutated


_orig = {n: getattr(O, n) for n in ("pool", "compressed_attention", "selected_keys", "combine", "gate",
                                     "dense_attention", "softmax", "spans")}
_orig["Geometry.kept_tokens"] = O.Geometry.kept_tokens

MUTATIONS = {
    "pool divides partial blocks by P*P": ("pool", _pool_full_denominator),
    "compressed branch multiplies by K instead of V": ("compressed_attention", _compressed_values_are_keys),
    "ties go to the higher block id": ("top_k_blocks", _top_k_ties_high),
    "selection drops the always-kept tokens": ("Geometry.kept_tokens", _kept_nothing),
    "selection lists the always-kept tokens twice": ("Geometry.kept_tokens", _kept_twice),
    "selection drops its last selected block": ("selected_keys", _selected_keys_drop_last_block),
    "gate weights the selection branch": ("combine", _combine_swapped),
    "combine drops the (1 - g) factor": ("combine", _combine_no_one_minus),
    "special entries ranked as candidates": ("guide_scores", _guide_counts_specials),
    "fine token up-sampled from the wrong block": ("Geometry.entry_of_token", _entry_of_token_shifted),
    "last block row loses a patch row": ("Geometry.block_rows_cols", _block_rows_cols_short),
    "gate sigmoid of -z": ("gate", _gate_wrong_sign),
    "softmax scale 1/D": ("Geometry.sm_scale", property(lambda self: 1.0 / self.D)),
    "frame attention over the next frame": ("frame_attention", _frame_attention_next_frame),
    "sliced dense attention drops the ragged last slice": ("dense_attention", _dense_sliced_drops_last_slice),
    "SGA samples the window centre": ("sga_sampled", _sga_centre_sample),
    "SGA drops the mean pair": ("sga_attention", _sga_without_mean_pair),
    "SGA lists a sampled own key twice": ("sga_attention", _sga_diagonal_twice),
    "reference keep still ranks frame 0's blocks": ("Geometry.B0", property(lambda self: 0)),
    "reference keep keeps every register token": ("Geometry.kept_tokens", _kept_all_specials_of_later_frames),
    "reference keep takes the camera from the last slot": ("Geometry.kept_tokens", _kept_camera_from_last_slot),
    "threaded softmax over the wrong axis": ("softmax", _softmax_torch_wrong_axis),
    "fine-query variant attends to fine keys": ("compressed_attention_fine", _fine_queries_against_fine_keys),
    "per-token gate variant uses the pooled query": ("gate_token", _token_gate_from_pooled_query),
}
# every split loop of the oracle, with each boundary mistake
for _fn in ("pool", "gsa_layer", "dense_attention", "sga_attention"):
    for _how, _what in (("drop_last", "drops its last slice"), ("skip", "skips a slice boundary")):
        MUTATIONS[f"{_fn} {_what} when split"] = ("spans", _spans_mistake(_fn, _how))


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutation_is_caught(name, monkeypatch):
    target, repl = MUTATIONS[name]
    if target.startswith("Geometry."):
        monkeypatch.setattr(O.Geometry, target.split(".", 1)[1], repl)
    else:
        monkeypatch.setattr(O, target, repl)
    failed = []
    warnings.simplefilter("ignore")
    for pin_name, fn in pins.all_pins(FIXTURE).items():
        try:
            fn()
        except Exception:  # a failed assertion, or the mutant breaking outright
            failed.append(pin_name)
    assert failed, f"no pin caught the planted mistake: {name}"
