"""Pins of the oracle's search of any depth (units of growing size searched
from the coarsest level down, then tokens) to things other than itself:
exact rational brute force on tiny inputs, and the identities that reduce a
deeper search to a shallower one (every unit of the top level kept; a level
whose units equal the level below)."""
import numpy as np
import pytest

import oracle
from hisa_inputs import make_case
from tests import brute


def _levels(c, level_B, keep, k, pool="mean"):
    return oracle.levels_select(oracle.Cache.of(c), c.Q, c.w, c.q_seq, c.q_pos, level_B, keep, k,
                                threads=2, pool=pool)


@pytest.mark.parametrize("seed", range(8))
@pytest.mark.parametrize("pool", ["mean", "max"])
def test_levels_match_exact_bruteforce(seed, pool):
    rng = np.random.default_rng(900 + seed)
    n_levels = 1 + seed % 4
    level_B = [int(rng.choice([1, 2, 3]))]
    for _ in range(n_levels - 1):
        level_B.append(level_B[-1] * int(rng.choice([1, 2, 3])))
    L = int(rng.integers(8, 56))
    keep = [int(rng.integers(1, 6)) for _ in range(n_levels)]
    k = int(rng.integers(1, L + 3))
    dtype = "e4m3" if seed % 2 else "bf16"
    c = make_case(batch=2, L=L, H=int(rng.integers(1, 4)), d=int(rng.choice([4, 8])), B=level_B[0],
                  m=keep[0], k=k, dtype=dtype, seed=950 + seed,
                  positions=np.unique(rng.integers(0, L, size=3)))
    r = _levels(c, level_B, keep, k, pool)
    for i in range(c.n_q):
        ref = brute.levels_row(c.keys, c.key_scale, c.dtype, c.Q, c.w, int(c.q_seq[i]),
                               int(c.q_pos[i]), i, level_B, keep, k, pool)
        got = [x for x in r["idx"][i] if x >= 0]
        assert got == ref["idx"], (i, got, ref["idx"])
        np.testing.assert_allclose(r["score"][i][:len(got)], [float(v) for v in ref["scores"]],
                                   rtol=1e-12, atol=1e-15)
        for lv in range(n_levels):
            n = int(r["nkept"][i, lv])
            assert list(r["kept"][lv][i][:n]) == ref["kept"][lv], (i, lv)
            assert all(v == -1 for v in r["kept"][lv][i][n:])
        assert tuple(r["counts"][i]) == ref["counts"]


@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
def test_one_level_is_the_two_stage_search(dtype):
    c = make_case(batch=2, L=[700, 333], H=4, d=16, B=16, m=7, k=50, dtype=dtype, seed=41,
                  positions=[np.array([0, 15, 16, 699]), np.array([332, 100])])
    r = _levels(c, [16], [7], 50)
    h = oracle.hisa_select(oracle.Cache.of(c), c.Q, c.w, c.q_seq, c.q_pos, 16, 7, 50, threads=2)
    np.testing.assert_array_equal(r["idx"], h["idx"])
    np.testing.assert_array_equal(r["score"], h["score"])
    np.testing.assert_array_equal(r["kept"][0], h["blocks"])
    np.testing.assert_array_equal(r["nkept"][:, 0], h["nblocks"])
    np.testing.assert_array_equal(r["counts"], h["counts"])


def test_two_levels_are_the_three_level_search():
    c = make_case(batch=2, L=[1500, 800], H=4, d=16, B=16, m=6, k=70, seed=42,
                  positions=[np.array([1499, 64, 0]), np.array([799, 300])])
    r = _levels(c, [16, 64], [6, 3], 70)
    t = oracle.tree_select(oracle.Cache.of(c), c.Q, c.w, c.q_seq, c.q_pos, 16, 4, 3, 6, 70,
                           threads=2)
    np.testing.assert_array_equal(r["idx"], t["idx"])
    np.testing.assert_array_equal(r["score"], t["score"])
    np.testing.assert_array_equal(r["kept"][0], t["blocks"])
    np.testing.assert_array_equal(r["kept"][1], t["sblocks"])
    np.testing.assert_array_equal(r["counts"][:, [1, 0, 2]], t["counts"])


@pytest.mark.parametrize("pool", ["mean", "max"])
def test_keeping_every_top_unit_drops_the_top_level(pool):
    """With the top level's keep at least its unit count, every unit is kept
    and the levels below see every visible unit: the same as no top level."""
    c = make_case(batch=2, L=[3000, 1234], H=3, d=16, B=8, m=9, k=80, seed=43,
                  positions=[np.array([2999, 1024, 7]), np.array([1233, 640])])
    deep = _levels(c, [8, 32, 256, 1024], [9, 5, 6, 3], 80, pool)      # <= 3 units of 1024
    shallow = _levels(c, [8, 32, 256], [9, 5, 6], 80, pool)
    np.testing.assert_array_equal(deep["idx"], shallow["idx"])
    np.testing.assert_array_equal(deep["score"], shallow["score"])
    for lv in range(3):
        np.testing.assert_array_equal(deep["kept"][lv], shallow["kept"][lv])


def test_a_level_of_equal_units_reduces_to_the_smaller_keep():
    """Level 1 with units equal to level 0's: level 0's candidates are level
    1's kept units, scored the same, so keeping keep[0] <= keep[1] of them is
    keeping the best keep[0] overall."""
    c = make_case(batch=1, L=2000, H=3, d=8, B=16, m=6, k=60, seed=44,
                  positions=np.array([1999, 900, 40]))
    a = _levels(c, [16, 16, 128], [6, 10, 4], 60)
    b = _levels(c, [16, 128], [6, 4], 60)
    np.testing.assert_array_equal(a["idx"], b["idx"])
    np.testing.assert_array_equal(a["kept"][0], b["kept"][0])


def test_levels_output_structure():
    c = make_case(batch=2, L=[5000, 2100], H=4, d=16, B=8, m=8, k=90, seed=45,
                  positions=[np.array([4999, 64, 0, 2047]), np.array([2099, 777])])
    level_B, keep = [8, 32, 128, 512], [8, 6, 4, 3]
    r = _levels(c, level_B, keep, 90)
    for i in range(c.n_q):
        t = int(c.q_pos[i])
        kept = [list(r["kept"][lv][i][:r["nkept"][i, lv]]) for lv in range(4)]
        for lv in range(4):
            assert t // level_B[lv] in kept[lv]                             # own unit kept
            assert kept[lv] == sorted(set(kept[lv]))
            assert len(kept[lv]) == min(keep[lv], r["counts"][i, lv])
            if lv < 3:
                f = level_B[lv + 1] // level_B[lv]
                assert all(j // f in kept[lv + 1] for j in kept[lv])        # nested
        v = [x for x in r["idx"][i] if x >= 0]
        assert v == sorted(v) and all(x <= t for x in v)
        assert all(x // 8 in kept[0] for x in v)
        assert r["counts"][i, 4] == len(kept[0]) * 8


def test_levels_reject_bad_arguments():
    c = make_case(batch=1, L=100, H=2, d=8, B=4, m=3, k=5, seed=46)
    with pytest.raises(ValueError):
        _levels(c, [4, 6], [3, 2], 5)             # 6 is not a multiple of 4
    with pytest.raises(ValueError):
        _levels(c, [4, 8], [3, 0], 5)             # nothing kept
    with pytest.raises(ValueError):
        _levels(c, [2] * 9, [3] * 9, 5)           # more than eight levels
