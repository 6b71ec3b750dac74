"""Pins of the CPU oracle to things other than itself (no GPU needed).

* exact rational brute force on tiny inputs (tests/brute.py), with forced ties;
* closed-form block means (constant blocks, arithmetic progressions, the
  trailing partial block) and the B = 1 identity; the same for max pooling;
* closed-form indexer scores (one-hot queries and keys, w = 0, all-negative
  dot products, scaling w);
* structure: m >= #blocks makes HISA the flat scan; the tokens-scored count
  ceil(L/B) + min(m, nb) * B of the pages' O(L/B + mB) (golden fixture);
  causality, ascending output, -1 tail padding, own block always kept.
"""
import json
import os

import numpy as np
import pytest

import oracle
from hisa_inputs import bf16_bits, bf16_to_f32, e4m3_to_f32, make_case, quantize_e4m3_rows
from tests import brute

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def tiny(seed, dtype="bf16", L=40, B=4, m=3, k=7, H=3, d=8, batch=2, positions=None):
    return make_case(batch=batch, L=L, H=H, d=d, B=B, m=m, k=k, dtype=dtype, seed=seed,
                     positions=positions)


def oracle_select(c, m=None, k=None, pool="mean"):
    return oracle.hisa_select(oracle.Cache.of(c), c.Q, c.w, c.q_seq, c.q_pos, c.B,
                              m or c.m, k or c.k, threads=2, pool=pool)


# ----------------------------------------------------------------- pooling


def test_pool_constant_block_is_exact():
    d, B = 8, 16
    keys = np.zeros((1, 64, d), np.float32)
    for j in range(4):
        keys[0, j * B:(j + 1) * B] = 0.375 * (j + 1) - 1.0   # exact in bf16
    c = oracle.Cache(bf16_bits(keys), None, [64], "bf16")
    P = oracle.pool(c, B)
    for j in range(4):
        assert np.all(P[0, j] == 0.375 * (j + 1) - 1.0)


@pytest.mark.parametrize("L,B", [(64, 16), (61, 16), (37, 8), (5, 8)])
def test_pool_arithmetic_progression_closed_form(L, B):
    # key[s, e] = (s + e) / 16: exact in bf16 for s + e <= 256.
    d = 4
    s = np.arange(L)[:, None]
    e = np.arange(d)[None, :]
    keys = ((s + e) / 16.0).astype(np.float32)[None]
    c = oracle.Cache(bf16_bits(keys), None, [L], "bf16")
    P = oracle.pool(c, B)
    for j in range(-(-L // B)):
        s0, s1 = j * B, min((j + 1) * B, L)          # trailing block: valid tokens only
        expect = ((s0 + s1 - 1) / 2.0 + np.arange(d)) / 16.0
        np.testing.assert_allclose(P[0, j], expect, rtol=0, atol=1e-15)


@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
def test_pool_block_size_one_is_identity(dtype):
    c = tiny(11, dtype=dtype, L=33, B=1)
    P = oracle.pool(oracle.Cache.of(c), 1)
    if dtype == "bf16":
        expect = bf16_to_f32(c.keys)
    else:   # fp32 product of the e4m3 value and the token's scale, computed by numpy
        expect = (e4m3_to_f32(c.keys) * c.key_scale[..., None]).astype(np.float32)
    assert np.array_equal(P[:, :33], expect[:, :33].astype(np.float64))


@pytest.mark.parametrize("L,B", [(64, 16), (61, 16), (37, 8), (5, 8)])
def test_pool_max_of_a_progression_is_its_last_valid_key(L, B):
    # key[s, e] = (s + e) / 16 rises with s, except column 0 falls: its max is
    # the block's first key.  The trailing block stops at its last valid key.
    d = 4
    s = np.arange(L)[:, None]
    e = np.arange(d)[None, :]
    keys = ((s + e) / 16.0).astype(np.float32)
    keys[:, 0] = -keys[:, 0]
    c = oracle.Cache(bf16_bits(keys[None]), None, [L], "bf16")
    P = oracle.pool(c, B, mode="max")
    for j in range(-(-L // B)):
        s0, s1 = j * B, min((j + 1) * B, L)
        expect = ((s1 - 1) + np.arange(d)) / 16.0
        expect[0] = -s0 / 16.0
        np.testing.assert_array_equal(P[0, j], expect)


@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
def test_pool_max_block_size_one_is_identity(dtype):
    c = tiny(12, dtype=dtype, L=33, B=1)
    P = oracle.pool(oracle.Cache.of(c), 1, mode="max")
    assert np.array_equal(P[:, :33], oracle.pool(oracle.Cache.of(c), 1)[:, :33])


def test_pool_max_constant_block_and_sign():
    d, B = 8, 4
    keys = np.full((1, 8, d), -0.75, np.float32)
    keys[0, 5, 3] = 0.5
    c = oracle.Cache(bf16_bits(keys), None, [8], "bf16")
    P = oracle.pool(c, B, mode="max")
    assert np.all(P[0, 0] == -0.75)
    assert P[0, 1, 3] == 0.5 and np.all(np.delete(P[0, 1], 3) == -0.75)


def test_pool_leaves_blocks_past_len_untouched():
    c = tiny(3, L=40, B=8)
    P = oracle.pool(oracle.Cache(c.keys, None, [17, 40], "bf16"), 8)
    assert np.all(np.isnan(P[0, 3:]))        # blocks 3.. start at >= 24 > 17
    assert not np.any(np.isnan(P[0, :3]))


# ----------------------------------------------------------------- scoring


def _onehot_case():
    d, H, L = 8, 3, 12
    alpha = np.array([0.5, -0.25, 1.5], np.float32)      # head h looks at coordinate a_h
    a = np.array([1, 4, 6])
    Q = np.zeros((1, H, d), np.float32)
    Q[0, np.arange(H), a] = alpha
    beta = (np.arange(L) % 5 - 2).astype(np.float32) * 0.125
    b = np.arange(L) % d
    keys = np.zeros((1, L, d), np.float32)
    keys[0, np.arange(L), b] = beta
    w = np.array([[0.75, 2.0, 0.5]], np.float32)
    expect = np.zeros(L)
    for s in range(L):
        for h in range(H):
            z = alpha[h] * beta[s] if a[h] == b[s] else 0.0
            expect[s] += w[0, h] * max(z, 0.0)
    return keys, Q, w, expect


def test_score_one_hot_closed_form():
    keys, Q, w, expect = _onehot_case()
    L = keys.shape[1]
    c = oracle.Cache(bf16_bits(keys), None, [L], "bf16")
    r = oracle.flat_select(c, bf16_bits(Q), w, [0], [L - 1], k=L, want_all=True)
    assert np.array_equal(r["all_scores"][0, :L], expect)


def test_score_zero_weights_ties_go_to_lowest_index():
    c = tiny(5, L=30)
    w0 = np.zeros_like(c.w)
    r = oracle.flat_select(oracle.Cache.of(c), c.Q, w0, c.q_seq, c.q_pos, k=7)
    assert np.all(r["score"] == 0.0)
    assert np.array_equal(r["idx"], np.tile(np.arange(7), (c.n_q, 1)))


def test_score_all_negative_dots_give_zero():
    c = tiny(6, L=20)
    Qf = np.abs(bf16_to_f32(c.Q))
    keys = -np.abs(bf16_to_f32(c.keys))
    cc = oracle.Cache(bf16_bits(keys), None, c.lens, "bf16")
    r = oracle.flat_select(cc, bf16_bits(Qf), c.w, c.q_seq, c.q_pos, k=5, want_all=True)
    assert np.all(r["all_scores"][:, :20] == 0.0)


def test_score_doubling_weights_doubles_scores():
    c = tiny(7, L=50, B=8, m=3, k=9)
    a = oracle_select(c)
    c2 = tiny(7, L=50, B=8, m=3, k=9)
    c2.w = (c.w * 2).astype(np.float32)
    b = oracle_select(c2)
    assert np.array_equal(a["idx"], b["idx"])
    assert np.array_equal(a["blocks"], b["blocks"])
    np.testing.assert_allclose(b["score"], 2 * a["score"], rtol=1e-15)


# --------------------------------------------------------- exact brute force


def _check_against_brute(c, m, k, pool="mean"):
    r = oracle_select(c, m=m, k=k, pool=pool)
    f = oracle.flat_select(oracle.Cache.of(c), c.Q, c.w, c.q_seq, c.q_pos, k=k)
    for i in range(c.n_q):
        b, t = int(c.q_seq[i]), int(c.q_pos[i])
        ref = brute.hisa_row(c.keys, c.key_scale, c.dtype, c.Q, c.w, b, t, i, c.B, m, k, pool=pool)
        got = [x for x in r["idx"][i] if x >= 0]
        assert got == ref["idx"], (i, got, ref["idx"])
        assert list(r["idx"][i][len(got):]) == [-1] * (k - len(got))
        np.testing.assert_allclose(r["score"][i][:len(got)], [float(v) for v in ref["scores"]],
                                   rtol=1e-12, atol=1e-15)
        nb = int(r["nblocks"][i])
        assert list(r["blocks"][i][:nb]) == ref["blocks"]
        np.testing.assert_allclose(r["block_scores"][i][:len(ref["block_scores"])],
                                   [float(v) for v in ref["block_scores"]], rtol=1e-12, atol=1e-15)
        fref = brute.flat_row(c.keys, c.key_scale, c.dtype, c.Q, c.w, b, t, i, k)
        fgot = [x for x in f["idx"][i] if x >= 0]
        assert fgot == fref["idx"]


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
def test_oracle_matches_exact_bruteforce(seed, dtype):
    rng = np.random.default_rng(seed)
    B = int(rng.choice([1, 2, 4, 16]))
    L = int(rng.integers(5, 48))
    nb = -(-L // B)
    m = int(rng.integers(1, nb + 2))
    k = int(rng.integers(1, L + 6))
    pos = np.unique(rng.integers(0, L, size=3))
    c = make_case(batch=2, L=L, H=int(rng.integers(1, 4)), d=int(rng.choice([4, 8])), B=B, m=m,
                  k=k, dtype=dtype, seed=100 + seed, positions=pos)
    _check_against_brute(c, m, k)


@pytest.mark.parametrize("seed", range(4))
@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
def test_oracle_max_pooling_matches_exact_bruteforce(seed, dtype):
    rng = np.random.default_rng(50 + seed)
    B = int(rng.choice([2, 4, 16]))
    L = int(rng.integers(9, 48))
    nb = -(-L // B)
    m = int(rng.integers(1, nb + 1))
    k = int(rng.integers(1, L + 6))
    pos = np.unique(rng.integers(0, L, size=3))
    c = make_case(batch=2, L=L, H=int(rng.integers(1, 4)), d=int(rng.choice([4, 8])), B=B, m=m,
                  k=k, dtype=dtype, seed=150 + seed, positions=pos)
    _check_against_brute(c, m, k, pool="max")


@pytest.mark.parametrize("seed", range(3))
def test_oracle_forced_ties_match_bruteforce(seed):
    # duplicated key rows and duplicated whole blocks: exact score ties at
    # token and block level, which must resolve toward the lower index.
    c = tiny(200 + seed, L=32, B=4, m=3, k=6)
    c.keys[:, 9] = c.keys[:, 2]
    c.keys[:, 17] = c.keys[:, 2]
    c.keys[:, 20:24] = c.keys[:, 4:8]
    c.keys[:, 12:16] = c.keys[:, 4:8]
    _check_against_brute(c, 3, 6)
    _check_against_brute(c, 2, 3)


# -------------------------------------------------------------- structure


@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
def test_hisa_with_all_blocks_is_the_flat_scan(dtype):
    c = make_case(batch=2, L=700, H=4, d=16, B=32, m=22, k=50, dtype=dtype, seed=9,
                  positions=np.array([0, 31, 32, 400, 699]))
    r = oracle_select(c, m=22)       # 22 blocks cover the whole prefix
    f = oracle.flat_select(oracle.Cache.of(c), c.Q, c.w, c.q_seq, c.q_pos, k=50)
    assert np.array_equal(r["idx"], f["idx"])
    assert np.array_equal(np.nan_to_num(r["score"], nan=-7), np.nan_to_num(f["score"], nan=-7))


def test_tokens_scored_count_matches_golden():
    g = json.load(open(os.path.join(GOLDEN, "complexity_counts.json")))
    for case in g["cases"]:
        L, B, m = case["L"], case["B"], case["m"]
        nb = -(-L // B)
        assert nb == case["block_scores"]
        assert min(m, nb) * B == case["token_slots"]
    # and the oracle's own counters agree on a small case
    c = make_case(batch=1, L=100, H=2, d=8, B=16, m=64, k=10, seed=4)
    r = oracle_select(c)
    assert tuple(r["counts"][0]) == (7, 112)
    c = make_case(batch=1, L=300, H=2, d=8, B=16, m=5, k=10, seed=4)
    r = oracle_select(c)
    assert tuple(r["counts"][0]) == (19, 80)


def test_output_format_and_causality():
    c = make_case(batch=3, L=[200, 150, 97], H=3, d=16, B=16, m=4, k=40, seed=12,
                  positions=[np.array([0, 5, 16, 199]), np.array([100, 149]), np.array([96])])
    r = oracle_select(c)
    for i in range(c.n_q):
        t = c.q_pos[i]
        row = r["idx"][i]
        valid = row[row >= 0]
        assert np.all(row[len(valid):] == -1)
        assert np.all(np.diff(valid) > 0)
        assert np.all(valid <= t)
        assert len(valid) == min(c.k, t + 1, r["nblocks"][i] * c.B)
        nb = -(-(t + 1) // c.B)
        assert (nb - 1) in r["blocks"][i]          # own block kept
        assert r["nblocks"][i] == min(c.m, nb)


def test_refine_on_own_blocks_reproduces_select():
    c = make_case(batch=2, L=500, H=4, d=16, B=16, m=6, k=33, seed=21,
                  positions=np.array([77, 499]))
    r = oracle_select(c)
    rr = oracle.hisa_refine(oracle.Cache.of(c), c.Q, c.w, c.q_seq, c.q_pos, c.B, c.k,
                            r["blocks"], r["nblocks"])
    assert np.array_equal(r["idx"], rr["idx"])


def _given_block_sets(rng, nb_vis, nb_all, mm):
    """Block lists a refinement may be handed (distinct ids, as every caller
    gives): unsorted, with -1 entries, with blocks past the query position,
    with the own (partial) block anywhere."""
    own = nb_vis - 1
    sets = []
    perm = [int(j) for j in rng.permutation(nb_vis)[:mm]]
    if own not in perm:
        perm[-1] = own
    sets.append(perm)                                        # unsorted, own block inside
    holes = list(perm)
    holes[0] = -1
    if len(holes) > 2:
        holes[len(holes) // 2] = -1
    sets.append(holes)                                       # -1 entries between ids
    future = [int(j) for j in rng.choice(nb_all - 1, size=min(mm, nb_all - 1) - 1, replace=False)]
    future = [nb_all - 1] + future                           # wholly past t when t < its start
    sets.append(future)
    sets.append([own] + [-1] * (mm - 1))                     # only the partial own block
    return sets


@pytest.mark.parametrize("seed", range(5))
@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
def test_refine_matches_exact_bruteforce_on_given_blocks(seed, dtype):
    # Token-level refinement on a block set the oracle did not choose itself
    # (the GPU's blocks in the token half of the parity rule): per slot
    # r * B + o the exact score of token blocks[r] * B + o, NaN for -1
    # entries and tokens past t; idx the top-k of the visible slots.
    rng = np.random.default_rng(400 + seed)
    B = int(rng.choice([2, 4, 8]))
    L = int(rng.integers(3 * B + 1, 48))
    nb_all = -(-L // B)
    pos = np.unique(np.concatenate([rng.integers(B + 1, L, size=2), [L - 1]]))
    c = make_case(batch=2, L=L, H=int(rng.integers(1, 4)), d=int(rng.choice([4, 8])), B=B, m=3,
                  k=5, dtype=dtype, seed=450 + seed, positions=pos)
    cache = oracle.Cache.of(c)
    for i in range(c.n_q):
        b, t = int(c.q_seq[i]), int(c.q_pos[i])
        nb_vis = t // B + 1
        mm = int(rng.integers(2, nb_vis + 1)) if nb_vis > 1 else 1
        for blocks in _given_block_sets(rng, nb_vis, nb_all, max(mm, 2)):
            for k in (1, int(rng.integers(2, 3 * B)), L + 3):
                Qi, wi = c.Q[i:i + 1], c.w[i:i + 1]
                r = oracle.hisa_refine(cache, Qi, wi, c.q_seq[i:i + 1], c.q_pos[i:i + 1], B, k,
                                       np.array([blocks], np.int32), np.array([len(blocks)], np.int32),
                                       threads=1)
                ref = brute.refine_row(c.keys, c.key_scale, c.dtype, c.Q, c.w, b, t, i, B, k, blocks)
                cs = r["cand_scores"][0]
                assert cs.shape == (len(blocks) * B,)
                for slot, v in enumerate(ref["cand"]):
                    if v is None:
                        assert np.isnan(cs[slot]), (slot, blocks, t)
                    else:
                        assert abs(cs[slot] - float(v)) <= 1e-12 * (1 + abs(float(v))), (slot, blocks)
                got = [x for x in r["idx"][0] if x >= 0]
                assert got == ref["idx"], (blocks, t, k)
                assert list(r["idx"][0][len(got):]) == [-1] * (k - len(got))
                np.testing.assert_allclose(r["score"][0][:len(got)], [float(v) for v in ref["scores"]],
                                           rtol=1e-12, atol=1e-15)


def test_topk_f32_rule_by_definition():
    rng = np.random.default_rng(3)
    x = rng.integers(-3, 4, size=(20, 37)).astype(np.float32) * 0.5   # many ties
    x[0] = 0.0
    x[1, ::2] = -0.0
    for k in (1, 5, 37, 50):
        got = oracle.topk_f32(x, k)
        for r in range(x.shape[0]):
            items = [(float(v), s) for s, v in enumerate(x[r])]
            ref = brute.keep_by_definition(items, k)
            assert [v for v in got[r] if v >= 0] == ref


def test_e4m3_dequant_is_fp32_product():
    rng = np.random.default_rng(1)
    k32 = rng.standard_normal((1, 24, 8)).astype(np.float32)
    codes, scale = quantize_e4m3_rows(k32)
    c = oracle.Cache(codes, scale, [24], "e4m3")
    P = oracle.pool(c, 1)
    import torch
    ref = (torch.from_numpy(codes).view(torch.float8_e4m3fn).float()
           * torch.from_numpy(scale)[..., None]).numpy()
    assert np.array_equal(P[0, :24], ref[0].astype(np.float64))
