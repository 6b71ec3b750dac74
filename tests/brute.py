"""Exact brute force for tiny HISA cases (pure Python, rational arithmetic).

Independent of the C oracle: every value is a ``fractions.Fraction``, so the
pooled means, the indexer scores and every comparison are exact, and top-k
membership is decided by its definition (an item is kept iff fewer than k
items beat it) rather than by sorting.  Only for inputs of a few dozen
tokens.

Method: HISA (gptget.net summary, "Methodology"; Chinese summary, method
details): mean-pool (or max-pool) contiguous blocks of size B, score the representatives
with the indexer, keep the top-m blocks (own block forced, counted in m),
score the tokens of the kept blocks, keep the top-k tokens.
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np

from hisa_inputs import bf16_to_f32, e4m3_to_f32


def key_values(case_keys, key_scale, dtype, b, s):
    """Exact rational value of key row (b, s) as the indexer sees it."""
    if dtype == "bf16":
        return [Fraction(float(v)) for v in bf16_to_f32(case_keys[b, s])]
    vals = e4m3_to_f32(case_keys[b, s])
    sc = np.float32(key_scale[b, s])
    # numpy fp32 multiply: one round-to-nearest of the exact product
    return [Fraction(float(np.float32(v) * sc)) for v in vals]


def query_values(Q, w, i):
    q = [[Fraction(float(v)) for v in bf16_to_f32(Q[i, h])] for h in range(Q.shape[1])]
    ww = [Fraction(float(v)) for v in w[i]]
    return q, ww


def score(q, ww, x):
    tot = Fraction(0)
    for qh, wh in zip(q, ww):
        z = sum((a * b for a, b in zip(qh, x)), Fraction(0))
        if z > 0:
            tot += wh * z
    return tot


def beats(a, b):
    """(value, index) a ranks above b: larger value, or equal value and lower index."""
    return a[0] > b[0] or (a[0] == b[0] and a[1] < b[1])


def keep_by_definition(items, k):
    """items: list of (value, index).  Returns the set of indices kept."""
    kept = []
    for it in items:
        n_above = sum(1 for o in items if o is not it and beats(o, it))
        if n_above < k:
            kept.append(it[1])
    return sorted(kept)


def block_mean(keys, key_scale, dtype, b, B, j, n):
    s0, s1 = j * B, min((j + 1) * B, n)
    rows = [key_values(keys, key_scale, dtype, b, s) for s in range(s0, s1)]
    return [sum(col, Fraction(0)) / (s1 - s0) for col in zip(*rows)]


def block_max(keys, key_scale, dtype, b, B, j, n):
    s0, s1 = j * B, min((j + 1) * B, n)
    rows = [key_values(keys, key_scale, dtype, b, s) for s in range(s0, s1)]
    return [max(col) for col in zip(*rows)]


def hisa_row(keys, key_scale, dtype, Q, w, b, t, i, B, m, k, pool="mean"):
    q, ww = query_values(Q, w, i)
    n = t + 1
    nb = -(-n // B)
    rep = block_max if pool == "max" else block_mean
    S = [score(q, ww, rep(keys, key_scale, dtype, b, B, j, n)) for j in range(nb)]
    if nb <= m:
        chosen = list(range(nb))
    else:
        others = [(S[j], j) for j in range(nb - 1)]
        chosen = keep_by_definition(others, m - 1) + [nb - 1]
    cand = []
    for j in chosen:
        for s in range(j * B, min((j + 1) * B, n)):
            cand.append((score(q, ww, key_values(keys, key_scale, dtype, b, s)), s))
    kept = keep_by_definition(cand, k)
    val = {s: v for v, s in cand}
    return dict(idx=kept, scores=[val[s] for s in kept], blocks=chosen, block_scores=S)


def refine_row(keys, key_scale, dtype, Q, w, b, t, i, B, k, blocks):
    """Token-level refinement on a GIVEN list of block ids (any order, -1 for
    an empty entry): slot r * B + o holds the exact score of token
    blocks[r] * B + o when that token is visible (<= t), else None; idx is the
    top-k of the visible slots by definition (ties: lower token index)."""
    q, ww = query_values(Q, w, i)
    cand, items = [], []
    for j in blocks:
        for o in range(B):
            s = j * B + o
            if j >= 0 and s <= t:
                v = score(q, ww, key_values(keys, key_scale, dtype, b, s))
                cand.append(v)
                items.append((v, s))
            else:
                cand.append(None)
    kept = keep_by_definition(items, k)
    val = {s: v for v, s in items}
    return dict(idx=kept, scores=[val[s] for s in kept], cand=cand)


def flat_row(keys, key_scale, dtype, Q, w, b, t, i, k):
    q, ww = query_values(Q, w, i)
    cand = [(score(q, ww, key_values(keys, key_scale, dtype, b, s)), s) for s in range(t + 1)]
    kept = keep_by_definition(cand, k)
    val = {s: v for v, s in cand}
    return dict(idx=kept, scores=[val[s] for s in kept])


def tree_row(keys, key_scale, dtype, Q, w, b, t, i, B, bf, W, m, k, pool="mean"):
    """Three-level search by definition: superblocks of bf blocks (own + best
    W - 1), the visible blocks under them (own + best m - 1), their tokens."""
    q, ww = query_values(Q, w, i)
    n = t + 1
    nb = -(-n // B)
    B2 = B * bf
    ns = -(-n // B2)
    rep = block_max if pool == "max" else block_mean
    S2 = [score(q, ww, rep(keys, key_scale, dtype, b, B2, j, n)) for j in range(ns)]
    if ns <= W:
        skept = list(range(ns))
    else:
        skept = keep_by_definition([(S2[j], j) for j in range(ns - 1)], W - 1) + [ns - 1]
    cand = [j for s in skept for j in range(s * bf, min((s + 1) * bf, nb - 1))]
    S1 = {j: score(q, ww, rep(keys, key_scale, dtype, b, B, j, n)) for j in cand}
    if len(cand) + 1 <= m:
        chosen = sorted(cand) + [nb - 1]
    else:
        chosen = keep_by_definition([(S1[j], j) for j in cand], m - 1) + [nb - 1]
    toks = []
    for j in chosen:
        for s in range(j * B, min((j + 1) * B, n)):
            toks.append((score(q, ww, key_values(keys, key_scale, dtype, b, s)), s))
    kept = keep_by_definition(toks, k)
    val = {s: v for v, s in toks}
    return dict(idx=kept, scores=[val[s] for s in kept], sblocks=skept, blocks=sorted(chosen),
                counts=(ns, len(cand) + 1, len(chosen) * B))


def levels_row(keys, key_scale, dtype, Q, w, b, t, i, level_B, keep, k, pool="mean"):
    """Search of any depth by definition: level l (finest first) has units of
    level_B[l] tokens; from the coarsest level down, keep the own unit plus
    the best keep[l] - 1 candidates, the candidates being every visible unit
    at the top and the visible units inside the kept units one level up
    below it; then the top k tokens of the kept blocks."""
    q, ww = query_values(Q, w, i)
    n = t + 1
    rep = block_max if pool == "max" else block_mean
    nl = len(level_B)
    kept, counts = [None] * nl, [0] * (nl + 1)
    up = None
    for lv in range(nl - 1, -1, -1):
        U = level_B[lv]
        nu = -(-n // U)
        if up is None:
            cand = list(range(nu - 1))
        else:
            bf = level_B[lv + 1] // U
            cand = [j for p in up for j in range(p * bf, min((p + 1) * bf, nu - 1))]
        S = {j: score(q, ww, rep(keys, key_scale, dtype, b, U, j, n)) for j in cand}
        if len(cand) + 1 <= keep[lv]:
            chosen = sorted(cand) + [nu - 1]
        else:
            chosen = keep_by_definition([(S[j], j) for j in cand], keep[lv] - 1) + [nu - 1]
        kept[lv] = sorted(chosen)
        counts[lv] = len(cand) + 1
        up = kept[lv]
    B = level_B[0]
    toks = []
    for j in up:
        for s in range(j * B, min((j + 1) * B, n)):
            toks.append((score(q, ww, key_values(keys, key_scale, dtype, b, s)), s))
    counts[nl] = len(up) * B
    sel = keep_by_definition(toks, k)
    val = {s: v for v, s in toks}
    return dict(idx=sel, scores=[val[s] for s in sel], kept=kept, counts=tuple(counts))
