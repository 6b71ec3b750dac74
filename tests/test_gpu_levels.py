"""GPU parity of the search of any depth (levels of growing units searched
from the coarsest down, then tokens) against the CPU oracle: the tolerance
rule applied at every level on the GPU's own choices one level up, and the
identities with the two-stage search, the three-level search and a
shallower search."""
import numpy as np
import pytest
import torch

import oracle
from hisa_inputs import make_case
from tests.gpu_util import device_case, lib, queries, run_hisa
from tests.parity import check_scores, check_selection

pytestmark = pytest.mark.gpu


def level_indexes(kv, level_B):
    """kv plus one index per coarser unit size, each pooled from the keys."""
    h = lib()
    kvs = [kv]
    for U in level_B[1:]:
        kl = h.superblock_index(kv, U // level_B[0])
        h.hisa_pool_blocks(kl)
        kvs.append(kl)
    return kvs


def run_levels(case, kvs, keep, k):
    h = lib()
    Q, w, qs, qp = queries(case)
    r = h.hisa_levels_select(kvs, Q, w, qs, qp, keep, k, inspect=True)
    torch.cuda.synchronize()
    assert kvs[0].status_bits() == 0
    return dict(idx=r["idx"].cpu().numpy(), scores=r["scores"].cpu().numpy(),
                kept=[t.cpu().numpy() for t in r["kept"]], nkept=[t.cpu().numpy() for t in r["nkept"]],
                counts=r["counts"].cpu().numpy())


def check_levels(case, g, level_B, keep, k, pool="mean"):
    """The rule at every level; returns the number of near-threshold swaps."""
    cache = oracle.Cache.of(case)
    Q, w, qs, qp = case.Q, case.w, case.q_seq, case.q_pos
    S = [oracle.hisa_select(cache, Q, w, qs, qp, U, 1, 1, pool=pool)["block_scores"] for U in level_B]
    B, nl = level_B[0], len(level_B)
    ref = oracle.hisa_refine(cache, Q, w, qs, qp, B, k, g["kept"][0], g["nkept"][0])
    swaps = 0
    for i in range(case.n_q):
        t = int(qp[i])
        up = None
        for lv in range(nl - 1, -1, -1):
            U = level_B[lv]
            nu = t // U + 1
            if up is None:
                ids = range(nu - 1)
            else:
                f = level_B[lv + 1] // U
                ids = [j for p in up for j in range(p * f, min((p + 1) * f, nu - 1))]
            cand = {j: float(S[lv][i, j]) for j in ids}
            n = int(g["nkept"][lv][i])
            row = [int(v) for v in g["kept"][lv][i]]
            assert n == min(keep[lv], len(cand) + 1) and row[n - 1] == nu - 1, (i, lv)
            swaps += check_selection(row[:n - 1] + [-1] * (len(row) - n + 1), cand,
                                     min(keep[lv] - 1, len(cand)), f"level {lv}")
            assert int(g["counts"][i, lv]) == len(cand) + 1, (i, lv)
            up = row[:n]
        assert int(g["counts"][i, nl]) == len(up) * B
        toks = {}
        for r, j in enumerate(up):
            for o in range(B):
                v = ref["cand_scores"][i][r * B + o]
                if not np.isnan(v):
                    toks[j * B + o] = float(v)
        swaps += check_selection(g["idx"][i], toks, k, "tokens")
        check_scores(g["idx"][i], g["scores"][i], toks)
    return swaps


# (B, level unit sizes, keep, k, H, d): both levels below the top gathered
# (branching factor 8); masked levels (branching factor 4); four block
# levels with a masked level between gathered ones
CASES = [
    ([16, 128, 1024], [12, 8, 4], 150, 16, 64),
    ([64, 256, 1024], [10, 6, 3], 300, 64, 128),
    ([8, 64, 512, 4096], [16, 12, 6, 3], 200, 16, 128),
]


@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
@pytest.mark.parametrize("level_B,keep,k,H,d", CASES)
def test_levels_match_oracle(dtype, level_B, keep, k, H, d):
    case = make_case(batch=2, L=[30000, 9000], H=H, d=d, B=level_B[0], m=keep[0], k=k, dtype=dtype,
                     seed=91 + level_B[1],
                     positions=[np.array([29999, 12345, 40, level_B[-1]]), np.array([8999, 4096])])
    kv = device_case(case)
    g = run_levels(case, level_indexes(kv, level_B), keep, k)
    assert check_levels(case, g, level_B, keep, k) <= 3


def test_levels_max_pooling_match_oracle():
    level_B, keep, k = [32, 256, 2048], [10, 6, 3], 200
    case = make_case(batch=2, L=[20000, 5000], H=32, d=128, B=32, m=10, k=k, seed=95,
                     positions=[np.array([19999, 7000]), np.array([4999, 64])])
    kv = device_case(case, pool="max")
    g = run_levels(case, level_indexes(kv, level_B), keep, k)
    assert check_levels(case, g, level_B, keep, k, pool="max") <= 3


def test_one_level_equals_hisa_select():
    case = make_case(batch=3, L=[5000, 2000, 700], H=64, d=128, B=64, m=9, k=256, seed=96)
    kv = device_case(case)
    g = run_levels(case, [kv], [9], 256)
    h = run_hisa(case, kv, m=9, k=256)
    np.testing.assert_array_equal(g["idx"], h["idx"])
    np.testing.assert_array_equal(g["scores"], h["scores"])
    np.testing.assert_array_equal(g["kept"][0], h["blocks"])
    np.testing.assert_array_equal(g["counts"], h["counts"])


@pytest.mark.parametrize("bf,W", [(4, 5), (32, 8)])
def test_two_levels_equal_tree_select(bf, W):
    """The three-level entry point and two levels here: the same kernels, the
    same results bit for bit (bf = 32 gathers the block level)."""
    case = make_case(batch=2, L=[20000, 9000], H=16, d=64, B=16, m=12, k=150, seed=97,
                     positions=[np.array([19999, 12345, 40]), np.array([8999, 4096])])
    kv = device_case(case)
    kvs = level_indexes(kv, [16, 16 * bf])
    g = run_levels(case, kvs, [12, W], 150)
    h = lib()
    Q, w, qs, qp = queries(case)
    t = h.hisa_tree_select(kv, kvs[1], Q, w, qs, qp, W, 12, 150, inspect=True)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(g["idx"], t["idx"].cpu().numpy())
    np.testing.assert_array_equal(g["scores"], t["scores"].cpu().numpy())
    np.testing.assert_array_equal(g["kept"][0], t["blocks"].cpu().numpy())
    np.testing.assert_array_equal(g["kept"][1], t["sblocks"].cpu().numpy())
    np.testing.assert_array_equal(g["counts"][:, [1, 0, 2]], t["counts"].cpu().numpy())


def test_keeping_every_top_unit_equals_fewer_levels():
    case = make_case(batch=2, L=[8000, 3000], H=32, d=128, B=32, m=10, k=200, seed=98)
    kv = device_case(case)
    kvs = level_indexes(kv, [32, 256, 8192])                  # at most one unit of 8192
    deep = run_levels(case, kvs, [10, 6, 2], 200)
    shallow = run_levels(case, kvs[:2], [10, 6], 200)
    np.testing.assert_array_equal(deep["idx"], shallow["idx"])
    np.testing.assert_array_equal(deep["kept"][0], shallow["kept"][0])
    np.testing.assert_array_equal(deep["kept"][1], shallow["kept"][1])
