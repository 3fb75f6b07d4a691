"""Pure-Python brute force of the GSA layer and dense attention, for tiny inputs.

Written separately from the oracle (no shared helpers, plain lists and
``math``) so that the oracle can be checked against it.  The layer follows the
Speed3R pages' technical summary, section 2.1: average-pool the patch grid of
every frame in P x P blocks (specials stay single entries), attend in the
pooled space, rank patch blocks by the pooled scores, attend over the chosen
blocks' tokens plus all special tokens, and mix with a sigmoid gate taken
from the pooled query.
"""

import math


def _dot(a, b):
    s = 0.0
    for x, y in zip(a, b):
        s += x * y
    return s


def _attend(q, keys, vals, scale):
    logits = [_dot(q, k) * scale for k in keys]
    top = max(logits)
    w = [math.exp(z - top) for z in logits]
    tot = sum(w)
    out = [0.0] * len(vals[0])
    for wi, v in zip(w, vals):
        for d in range(len(v)):
            out[d] += wi / tot * v[d]
    return out


def layout(N, S, Hp, Wp, P):
    """Per frame: special token ids, and the blocks as lists of token ids."""
    per = S + Hp * Wp
    frames = []
    for f in range(N):
        base = f * per
        specials = [base + j for j in range(S)]
        blocks = []
        for r0 in range(0, Hp, P):
            for c0 in range(0, Wp, P):
                toks = []
                for r in range(r0, min(r0 + P, Hp)):
                    for c in range(c0, min(c0 + P, Wp)):
                        toks.append(base + S + r * Wp + c)
                blocks.append(toks)
        frames.append((specials, blocks))
    return frames


def gsa_bruteforce(Q, K, V, w, N, S, Hp, Wp, P, topk, keep="specials"):
    """Q, K, V: nested lists [T][H][D] of floats; w: [H][D].  Returns dict.

    keep="specials": every special token is always attended to.
    keep="reference": every token of frame 0 and the first special token of
    each later frame are always attended to, and only the blocks of frames
    1..N-1 are ranked.
    """
    H = len(Q[0])
    D = len(Q[0][0])
    scale = 1.0 / math.sqrt(D)
    frames = layout(N, S, Hp, Wp, P)

    # compressed sequence: list of (token list, is_special); block ids in order
    entries = []
    block_entry = []
    block_tokens = []
    all_specials = []
    block_frame = []
    for f, (specials, blocks) in enumerate(frames):
        for t in specials:
            entries.append([t])
            all_specials.append(t)
        for toks in blocks:
            block_entry.append(len(entries))
            block_tokens.append(toks)
            block_frame.append(f)
            entries.append(toks)
    if keep == "specials":
        always = all_specials
        rankable = list(range(len(block_entry)))
    else:
        per = S + Hp * Wp
        always = list(range(per)) + [f * per for f in range(1, N) if S > 0]
        rankable = [beta for beta in range(len(block_entry)) if block_frame[beta] > 0]

    def mean_of(X, toks, h):
        return [sum(X[t][h][d] for t in toks) / len(toks) for d in range(D)]

    qc = [[mean_of(Q, toks, h) for h in range(H)] for toks in entries]
    kc = [[mean_of(K, toks, h) for h in range(H)] for toks in entries]
    vc = [[mean_of(V, toks, h) for h in range(H)] for toks in entries]

    n_e = len(entries)
    o_cmp = [[None] * H for _ in range(n_e)]
    sel = [[None] * H for _ in range(n_e)]
    for a in range(n_e):
        for h in range(H):
            o_cmp[a][h] = _attend(qc[a][h], [kc[b][h] for b in range(n_e)],
                                  [vc[b][h] for b in range(n_e)], scale)
            scored = []
            for beta in rankable:
                b = block_entry[beta]
                scored.append((-(_dot(qc[a][h], kc[b][h]) * scale), beta))
            scored.sort()
            chosen = sorted(beta for _, beta in scored[:min(topk, len(scored))])
            sel[a][h] = chosen

    token_entry = {}
    for a, toks in enumerate(entries):
        for t in toks:
            token_entry[t] = a

    T = len(Q)
    o_sel = [[None] * H for _ in range(T)]
    out = [[None] * H for _ in range(T)]
    gates = [[None] * H for _ in range(n_e)]
    for a in range(n_e):
        for h in range(H):
            z = _dot(qc[a][h], w[h])
            gates[a][h] = 1.0 / (1.0 + math.exp(-z))
    for t in range(T):
        a = token_entry[t]
        for h in range(H):
            keys = []
            for beta in sel[a][h]:
                keys.extend(block_tokens[beta])
            keys.extend(always)
            o_sel[t][h] = _attend(Q[t][h], [K[j][h] for j in keys], [V[j][h] for j in keys], scale)
            g = gates[a][h]
            out[t][h] = [g * x + (1.0 - g) * y for x, y in zip(o_cmp[a][h], o_sel[t][h])]
    return dict(o_cmp=o_cmp, sel=sel, o_sel=o_sel, out=out, g=gates, token_entry=token_entry)


def dense_bruteforce(Q, K, V):
    T = len(Q)
    H = len(Q[0])
    D = len(Q[0][0])
    scale = 1.0 / math.sqrt(D)
    return [[_attend(Q[t][h], [K[j][h] for j in range(T)], [V[j][h] for j in range(T)], scale)
             for h in range(H)] for t in range(T)]


def frame_bruteforce(Q, K, V, tokens_per_frame):
    """Attention of every token over the tokens of its own frame only."""
    T = len(Q)
    H = len(Q[0])
    D = len(Q[0][0])
    scale = 1.0 / math.sqrt(D)
    out = []
    for t in range(T):
        start = (t // tokens_per_frame) * tokens_per_frame
        keys = range(start, start + tokens_per_frame)
        out.append([_attend(Q[t][h], [K[j][h] for j in keys], [V[j][h] for j in keys], scale)
                    for h in range(H)])
    return out


def sga_bruteforce(Q, K, V, tokens_per_frame, n_special, hp, wp, sub_h, sub_w):
    """Subsampled global attention: keys are every special token and the patch
    at the top-left of every sub_h x sub_w window, plus the query's own token,
    plus one key/value pair holding the means over all other patch tokens."""
    T = len(Q)
    H = len(Q[0])
    D = len(Q[0][0])
    scale = 1.0 / math.sqrt(D)
    keep = set()
    for t in range(T):
        i = t % tokens_per_frame
        if i < n_special:
            keep.add(t)
        else:
            r, c = divmod(i - n_special, wp)
            if r % sub_h == 0 and c % sub_w == 0:
                keep.add(t)
    dropped = [t for t in range(T) if t not in keep]
    out = []
    for t in range(T):
        row = []
        for h in range(H):
            keys = [K[j][h] for j in sorted(keep)]
            vals = [V[j][h] for j in sorted(keep)]
            if t not in keep:
                keys.append(K[t][h])
                vals.append(V[t][h])
            if dropped:
                keys.append([sum(K[j][h][d] for j in dropped) / len(dropped) for d in range(D)])
                vals.append([sum(V[j][h][d] for j in dropped) / len(dropped) for d in range(D)])
            row.append(_attend(Q[t][h], keys, vals, scale))
        out.append(row)
    return out
