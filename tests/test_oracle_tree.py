"""Pins of the oracle's three-level search (superblocks of bf blocks, then
blocks, then tokens) to things other than itself: exact rational brute force
on tiny inputs, and the two identities that reduce it to the two-stage search
(every superblock kept; one block per superblock with W >= m)."""
import numpy as np
import pytest

import oracle
from hisa_inputs import make_case
from tests import brute


def _tree(c, bf, W, m, k, pool="mean"):
    return oracle.tree_select(oracle.Cache.of(c), c.Q, c.w, c.q_seq, c.q_pos, c.B, bf, W, m, k,
                              threads=2, pool=pool)


def _two_stage(c, m, k, pool="mean"):
    return oracle.hisa_select(oracle.Cache.of(c), c.Q, c.w, c.q_seq, c.q_pos, c.B, m, k,
                              threads=2, pool=pool)


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("pool", ["mean", "max"])
def test_tree_matches_exact_bruteforce(seed, pool):
    rng = np.random.default_rng(700 + seed)
    B = int(rng.choice([1, 2, 4]))
    bf = int(rng.choice([2, 3, 4]))
    L = int(rng.integers(6, 60))
    ns = -(-L // (B * bf))
    W = int(rng.integers(1, ns + 2))
    m = int(rng.integers(1, 2 * W * bf + 2))
    k = int(rng.integers(1, L + 4))
    dtype = "e4m3" if seed % 2 else "bf16"
    c = make_case(batch=2, L=L, H=int(rng.integers(1, 4)), d=int(rng.choice([4, 8])), B=B, m=m,
                  k=k, dtype=dtype, seed=800 + seed, positions=np.unique(rng.integers(0, L, size=3)))
    r = _tree(c, bf, W, m, k, pool)
    for i in range(c.n_q):
        ref = brute.tree_row(c.keys, c.key_scale, c.dtype, c.Q, c.w, int(c.q_seq[i]),
                             int(c.q_pos[i]), i, B, bf, W, m, k, pool)
        got = [x for x in r["idx"][i] if x >= 0]
        assert got == ref["idx"], (i, got, ref["idx"])
        np.testing.assert_allclose(r["score"][i][:len(got)], [float(v) for v in ref["scores"]],
                                   rtol=1e-12, atol=1e-15)
        assert list(r["sblocks"][i][:r["nsblocks"][i]]) == ref["sblocks"]
        assert list(r["blocks"][i][:r["nblocks"][i]]) == ref["blocks"]
        assert tuple(r["counts"][i]) == ref["counts"]


@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
def test_tree_keeping_every_superblock_is_the_two_stage_search(dtype):
    c = make_case(batch=2, L=900, H=4, d=16, B=16, m=9, k=60, dtype=dtype, seed=31,
                  positions=np.array([0, 15, 16, 500, 899]))
    r = _tree(c, bf=8, W=8, m=9, k=60)            # 900 / 128 -> at most 8 superblocks
    h = _two_stage(c, m=9, k=60)
    assert np.array_equal(r["idx"], h["idx"])
    assert np.array_equal(r["blocks"], h["blocks"])
    np.testing.assert_array_equal(r["score"], h["score"])


def test_tree_with_single_block_superblocks_is_the_two_stage_search():
    c = make_case(batch=1, L=700, H=3, d=8, B=32, m=5, k=40, seed=32,
                  positions=np.array([699, 350, 40]))
    r = _tree(c, bf=1, W=7, m=5, k=40)            # top-7 blocks contain the top-5
    h = _two_stage(c, m=5, k=40)
    assert np.array_equal(r["idx"], h["idx"])
    assert np.array_equal(r["blocks"], h["blocks"])


def test_tree_output_structure():
    c = make_case(batch=2, L=[1500, 800], H=4, d=16, B=16, m=6, k=70, seed=33,
                  positions=[np.array([1499, 64, 0]), np.array([799, 300])])
    r = _tree(c, bf=4, W=3, m=6, k=70)
    for i in range(c.n_q):
        t = int(c.q_pos[i])
        nb, ns = t // 16 + 1, t // 64 + 1
        sb = list(r["sblocks"][i][:r["nsblocks"][i]])
        bl = list(r["blocks"][i][:r["nblocks"][i]])
        assert ns - 1 in sb and nb - 1 in bl                   # own superblock and block kept
        assert all(j // 4 in sb for j in bl)                   # blocks under kept superblocks
        assert sb == sorted(sb) and bl == sorted(bl)
        v = [x for x in r["idx"][i] if x >= 0]
        assert v == sorted(v) and all(x <= t for x in v)
        assert all(x // 16 in bl for x in v)
