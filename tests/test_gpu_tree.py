"""GPU parity of the three-level search (superblocks of bf blocks, then
blocks, then tokens) against the CPU oracle, with the tolerance rule applied
at every level on the GPU's own choices one level up."""
import numpy as np
import pytest
import torch

import oracle
from hisa_inputs import make_case
from tests.gpu_util import device_case, lib, queries, run_hisa
from tests.parity import check_scores, check_selection

pytestmark = pytest.mark.gpu


def run_tree(case, kv, bf, W, m, k, pool="mean"):
    h = lib()
    kv2 = h.superblock_index(kv, bf)
    h.hisa_pool_blocks(kv2)
    Q, w, qs, qp = queries(case)
    r = h.hisa_tree_select(kv, kv2, Q, w, qs, qp, W, m, k, inspect=True)
    torch.cuda.synchronize()
    assert kv.status_bits() == 0
    return {key: v.cpu().numpy() for key, v in r.items()}


def check_tree(case, g, bf, W, m, k, pool="mean"):
    """Three-level rule; returns the number of near-threshold swaps."""
    B, B2 = case.B, case.B * bf
    cache = oracle.Cache.of(case)
    Q, w, qs, qp = case.Q, case.w, case.q_seq, case.q_pos
    big = 1 << 12
    s2 = oracle.hisa_select(cache, Q, w, qs, qp, B2, 1, 1, pool=pool)["block_scores"]
    s1 = oracle.hisa_select(cache, Q, w, qs, qp, B, 1, 1, pool=pool)["block_scores"]
    ref = oracle.hisa_refine(cache, Q, w, qs, qp, B, k, g["blocks"], g["nblocks"])
    swaps = 0
    for i in range(case.n_q):
        t = int(qp[i])
        nb, ns = t // B + 1, t // B2 + 1
        # superblocks: own + best W - 1
        nsk = int(g["nsblocks"][i])
        sb = [int(v) for v in g["sblocks"][i]]
        assert nsk == min(W, ns) and ns - 1 in sb[:nsk]
        others = {j: float(s2[i, j]) for j in range(ns - 1)}
        kept_others = [v for v in sb[:nsk] if v != ns - 1]
        swaps += check_selection(kept_others + [-1] * (len(sb) - len(kept_others)), others,
                                 min(W - 1, ns - 1), "superblocks")
        # blocks: candidates under the GPU's superblocks, own + best m - 1
        cand = {j: float(s1[i, j]) for s in sb[:nsk] for j in range(s * bf, min((s + 1) * bf, nb - 1))}
        nbk = int(g["nblocks"][i])
        bl = [int(v) for v in g["blocks"][i]]
        assert nbk == min(m, len(cand) + 1) and bl[nbk - 1] == nb - 1
        swaps += check_selection(bl[:nbk - 1] + [-1] * (len(bl) - nbk + 1), cand,
                                 min(m - 1, len(cand)), "blocks")
        assert tuple(g["counts"][i]) == (ns, len(cand) + 1, nbk * B)
        # tokens on the GPU's blocks
        toks = {}
        for r in range(nbk):
            for o in range(B):
                v = ref["cand_scores"][i][r * B + o]
                if not np.isnan(v):
                    toks[bl[r] * B + o] = float(v)
        swaps += check_selection(g["idx"][i], toks, k, "tokens")
        check_scores(g["idx"][i], g["scores"][i], toks)
    return swaps


@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
@pytest.mark.parametrize("B,bf,W,m,k", [(128, 4, 6, 16, 512), (64, 8, 3, 12, 300), (16, 4, 5, 9, 100),
                                      (8, 16, 4, 20, 200)])
def test_tree_matches_oracle(dtype, B, bf, W, m, k):
    case = make_case(batch=3, L=[6000, 2500, 900], H=64 if B == 128 else 16, d=128, B=B, m=m, k=k,
                     dtype=dtype, seed=61 + B + bf,
                     positions=[np.array([0, B, 5999, 3000]), np.array([2499, 1000]), np.array([899])])
    kv = device_case(case)
    g = run_tree(case, kv, bf, W, m, k)
    assert check_tree(case, g, bf, W, m, k) <= 3


def test_tree_gathered_level_matches_oracle():
    """Kept superblocks of bf = 32 blocks covering under a quarter of the
    blocks: the level under them loads and scores only their children (runs
    of 32 representatives), d = 64; the counters report those children."""
    case = make_case(batch=2, L=[20000, 9000], H=16, d=64, B=16, m=12, k=150, seed=79,
                     positions=[np.array([19999, 12345, 40]), np.array([8999, 4096])])
    kv = device_case(case)
    g = run_tree(case, kv, 32, 8, 12, 150)
    assert check_tree(case, g, 32, 8, 12, 150) <= 3


def test_tree_max_pooling_matches_oracle():
    case = make_case(batch=2, L=[5000, 3000], H=32, d=128, B=64, m=10, k=256, seed=77,
                     positions=[np.array([4999, 2000]), np.array([2999, 64])])
    kv = device_case(case, pool="max")
    g = run_tree(case, kv, 4, 4, 10, 256, pool="max")
    assert check_tree(case, g, 4, 4, 10, 256, pool="max") <= 3


def test_tree_keeping_every_superblock_equals_hisa_select():
    case = make_case(batch=4, L=4096, H=64, d=128, B=128, m=8, k=400, seed=78)
    kv = device_case(case)
    g = run_tree(case, kv, 4, 8, 8, 400)            # 4096 / 512 = 8 superblocks: all kept
    h = run_hisa(case, kv)
    np.testing.assert_array_equal(g["idx"], h["idx"])
    np.testing.assert_array_equal(g["blocks"], h["blocks"])


def test_tree_after_appends_with_tail_repool():
    """Decode loop: append to the block index, re-pool the superblock index's
    trailing superblock, select; the superblock index must equal a re-pool."""
    h = lib()
    steps = 40
    case = make_case(batch=2, L=[3000, 1100], H=32, d=128, B=64, m=6, k=128, seed=79,
                     append_steps=steps, cap=3100)
    kv = device_case(case)
    kv2 = h.superblock_index(kv, 4)
    h.hisa_pool_blocks(kv2)
    for s in range(steps):
        h.hisa_append(kv, torch.from_numpy(case.append_keys[s].view(np.int16)).cuda())
        h.hisa_pool_tail(kv2)
    torch.cuda.synchronize()
    inc = kv2.pooled.clone()
    h.hisa_pool_blocks(kv2)
    torch.cuda.synchronize()
    for b, n in enumerate([3040, 1140]):
        nb2 = -(-n // 256)
        assert torch.equal(inc[b, :nb2], kv2.pooled[b, :nb2])
    assert kv.status_bits() == 0
