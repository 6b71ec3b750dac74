"""Parity rules between the CUDA path and the CPU oracle.

Scores: |gpu - oracle| <= 1e-3 * (1 + |oracle|) (fp32 accumulation against
double).  Index sets: equal, except that entries whose oracle scores lie
within that tolerance of the selection threshold may be swapped.  HISA has
two selections, so the rule is applied twice:

  blocks  the GPU's kept blocks against the oracle's block scores, at the
          (m-1)-th best non-own block (the own block is always kept);
  tokens  the GPU's kept tokens against the oracle's token scores computed
          on the GPU's OWN block set, at the k-th best candidate.
Without the second step one allowed block swap near the threshold would
change about B tokens and fail a correct kernel.
"""
from __future__ import annotations

import numpy as np


def tau(x):
    return 1e-3 * (1.0 + np.abs(x))


def check_selection(kept, cand_scores: dict, k: int, what: str = "tokens"):
    """kept: GPU output row (ascending ids, -1 tail); cand_scores: id -> oracle score."""
    kept = [int(v) for v in kept]
    valid = [v for v in kept if v >= 0]
    assert kept[len(valid):] == [-1] * (len(kept) - len(valid)), f"{what}: -1 not only at the tail"
    assert all(a < b for a, b in zip(valid, valid[1:])), f"{what}: not strictly ascending"
    assert all(v in cand_scores for v in valid), f"{what}: id outside the candidates"
    n = len(cand_scores)
    if k == 0:
        assert not valid, f"{what}: kept ids with k = 0"
        return 0
    assert len(valid) == min(k, n), f"{what}: kept {len(valid)} of {n}, want {min(k, n)}"
    if n <= k:
        return 0
    vals = np.sort(np.fromiter(cand_scores.values(), dtype=np.float64))[::-1]
    thr = vals[k - 1]
    t = tau(thr)
    must = [s for s, v in cand_scores.items() if v > thr + t]
    got = set(valid)
    missing = [s for s in must if s not in got]
    assert not missing, f"{what}: clearly-above-threshold ids missing: {missing[:5]} thr={thr}"
    low = [s for s in valid if cand_scores[s] < thr - t]
    assert not low, f"{what}: clearly-below-threshold ids kept: {low[:5]} thr={thr}"
    # number of swaps relative to the oracle's own exact choice
    order = sorted(cand_scores.items(), key=lambda kv: (-kv[1], kv[0]))[:k]
    return len(set(s for s, _ in order) - got)


def check_scores(idx_row, gpu_scores_row, cand_scores: dict, what="scores"):
    for s, g in zip(idx_row, gpu_scores_row):
        if s < 0:
            assert np.isnan(g), f"{what}: padding score not NaN"
            continue
        o = cand_scores[int(s)]
        assert abs(g - o) <= tau(o), f"{what}: id {s}: gpu {g} oracle {o}"


def hisa_row_check(i, gpu, ora_blocks, ref, B, m, k, t):
    """gpu: dict of numpy arrays (idx, scores, blocks, nblocks); ora_blocks: oracle
    select dict (block_scores); ref: oracle refine on the GPU's block set."""
    nb = t // B + 1
    nbk = int(gpu["nblocks"][i])
    gblocks = [int(v) for v in gpu["blocks"][i]]
    assert nbk == min(m, nb)
    assert gblocks[nbk - 1] == nb - 1, "own block missing"
    S = ora_blocks["block_scores"][i]
    others = {j: float(S[j]) for j in range(nb - 1)}
    swaps_b = check_selection(gblocks[:nbk - 1] + [-1] * (len(gblocks) - nbk + 1), others,
                              min(m - 1, nb - 1) if nb > m else nb - 1, "blocks")
    cand = {}
    cs = ref["cand_scores"][i]
    for r in range(nbk):
        for o in range(B):
            v = cs[r * B + o]
            if not np.isnan(v):
                cand[gblocks[r] * B + o] = float(v)
    swaps_t = check_selection(gpu["idx"][i], cand, k, "tokens")
    if gpu.get("scores") is not None:
        check_scores(gpu["idx"][i], gpu["scores"][i], cand)
    return swaps_b, swaps_t


def iou(a_row, b_row):
    a = set(int(v) for v in a_row if v >= 0)
    b = set(int(v) for v in b_row if v >= 0)
    if not a and not b:
        return 1.0
    return len(a & b) / len(a | b)
