"""The oracle's pins catch plausible mistakes.

Each case copies the oracle source, plants one mistake (a dropped term, a
wrong sign or index, a reversed tie rule ...), builds the copy on the CPU and
checks that the exact brute force or a closed form rejects it.  The committed
oracle is never modified.
"""
import os

import numpy as np
import pytest

import oracle
from hisa_inputs import bf16_bits, make_case
from tests import attn_pins, brute

MUTANTS = {
    "relu_dropped": ("acc += w[h] * (z > 0.0 ? z : 0.0);", "acc += w[h] * z;"),
    "causal_off_by_one": ("if (blk[r] >= 0 && s <= t) {", "if (blk[r] >= 0 && s < t) {"),
    "ties_to_higher_index": ("return (a->i > b->i) - (a->i < b->i);",
                             "return (a->i < b->i) - (a->i > b->i);"),
    "mean_over_B_not_valid_count": ("mu[e] /= (double)(s1 - s0);", "mu[e] /= (double)B;"),
    "own_block_not_forced": ("chosen[J->m - 1] = (int32_t)(nb - 1);",
                             "chosen[J->m - 1] = (int32_t)items[J->m - 1].i;"),
    "first_head_dropped": ("for (int h = 0; h < H; ++h) {\n        double z",
                           "for (int h = 1; h < H; ++h) {\n        double z"),
    "query_stride_transposed": ("double z = dot(q + (size_t)h * d, x, d);",
                                "double z = dot(q + (size_t)h, x, d);"),
    "e4m3_bias_wrong": ("else v = ldexp(1.0 + m / 8.0, e - 7);",
                        "else v = ldexp(1.0 + m / 8.0, e - 8);"),
    "flat_misses_last_token": ("for (long s = 0; s <= t; ++s) {", "for (long s = 0; s < t; ++s) {"),
    "max_pool_takes_min": ("(s == s0 || tmp[e] > mu[e])", "(s == s0 || tmp[e] < mu[e])"),
    "tree_own_superblock_not_forced": ("skept[J->W - 1] = (int32_t)(ns - 1);",
                                       "skept[J->W - 1] = (int32_t)items[J->W - 1].i;"),
    "tree_children_skip_last": ("j < (long)(skept[r] + 1) * bf && j < nb - 1; ++j",
                                "j < (long)(skept[r] + 1) * bf - 1 && j < nb - 1; ++j"),
    "levels_own_unit_not_forced": ("cur[n_keep - 1] = (int32_t)(nu - 1);",
                                   "cur[n_keep - 1] = (int32_t)(nu - 2 > 0 ? nu - 2 : 0);"),
    "levels_children_skip_last": ("j < (long)(up[r] + 1) * bf && j < nu - 1; ++j",
                                  "j < (long)(up[r] + 1) * bf - 1 && j < nu - 1; ++j"),
    "levels_counts_miss_own_unit": ("J->counts[(size_t)i * (J->n_lv + 1) + l] = nc + 1;",
                                    "J->counts[(size_t)i * (J->n_lv + 1) + l] = nc;"),
    "refine_cand_layout_transposed": ("if (cand) cand[(size_t)r * J->B + o] = v;",
                                      "if (cand) cand[(size_t)o * J->mm + r] = v;"),
    "refine_skips_last_given_block": ("for (int r = 0; r < nblk; ++r) {",
                                      "for (int r = 0; r + 1 < nblk; ++r) {"),
    "attn_scale_dropped": ("a[j] = J->scale * z;", "a[j] = z;"),
    "attn_entries_past_len_kept": ("if (s < 0 || s >= n) { a[j] = NAN; continue; }",
                                   "if (s < 0) { a[j] = NAN; continue; }"),
    "attn_lse_without_max": ("J->lse[(size_t)i * J->Ha + h] = amax + log(sum);",
                             "J->lse[(size_t)i * J->Ha + h] = log(sum);"),
}


def _cases():
    out = []
    for seed, dtype in [(1, "bf16"), (2, "e4m3"), (3, "bf16"), (4, "e4m3")]:
        rng = np.random.default_rng(seed)
        B = [4, 8, 4, 2][seed - 1]
        L = [37, 45, 30, 21][seed - 1]
        c = make_case(batch=2, L=L, H=3, d=8, B=B, m=2 + seed % 2, k=5 + seed, dtype=dtype,
                      seed=300 + seed, positions=np.array([L - 1, L // 2, B + 1]))
        out.append(c)
    t = make_case(batch=1, L=32, H=3, d=8, B=4, m=3, k=6, seed=305)
    t.keys[:, 9] = t.keys[:, 2]
    t.keys[:, 20:24] = t.keys[:, 4:8]
    t.keys[:, 12:16] = t.keys[:, 4:8]
    out.append(t)
    return out


def _pool_closed_form_fails(lib) -> bool:
    L, B, d = 61, 16, 4                       # trailing block holds 13 tokens
    s = np.arange(L)[:, None]
    keys = ((s + np.arange(d)[None, :]) / 16.0).astype(np.float32)[None]
    P = oracle.pool(oracle.Cache(bf16_bits(keys), None, [L], "bf16"), B, lib=lib)
    for j in range(-(-L // B)):
        s0, s1 = j * B, min((j + 1) * B, L)
        if not np.allclose(P[0, j], ((s0 + s1 - 1) / 2.0 + np.arange(d)) / 16.0, rtol=0,
                           atol=1e-15):
            return True
    return False


def _refine_fails(lib) -> bool:
    c = make_case(batch=1, L=30, H=2, d=4, B=4, m=3, k=5, seed=313, positions=np.array([29, 17]))
    cache = oracle.Cache.of(c)
    given = [[2, -1, 7, 0], [4, 1, -1, 3]]       # row 0 (t = 29): own block 7 partial
    r = oracle.hisa_refine(cache, c.Q, c.w, c.q_seq, c.q_pos, c.B, 5, np.array(given, np.int32),
                           np.array([4, 4], np.int32), threads=1, lib=lib)
    for i in range(c.n_q):
        ref = brute.refine_row(c.keys, c.key_scale, c.dtype, c.Q, c.w, int(c.q_seq[i]),
                               int(c.q_pos[i]), i, c.B, 5, given[i])
        if [x for x in r["idx"][i] if x >= 0] != ref["idx"]:
            return True
        for slot, v in enumerate(ref["cand"]):
            got = r["cand_scores"][i][slot]
            if (v is None) != bool(np.isnan(got)):
                return True
            if v is not None and abs(got - float(v)) > 1e-12 * (1 + abs(float(v))):
                return True
    return False


def _detects(lib) -> bool:
    """True if some pin rejects the library `lib`."""
    if _pool_closed_form_fails(lib):
        return True
    if attn_pins.any_fails(lib):
        return True
    for c in _cases():
        cache = oracle.Cache.of(c)
        r = oracle.hisa_select(cache, c.Q, c.w, c.q_seq, c.q_pos, c.B, c.m, c.k, threads=1,
                               lib=lib)
        f = oracle.flat_select(cache, c.Q, c.w, c.q_seq, c.q_pos, c.k, threads=1, lib=lib)
        for i in range(c.n_q):
            b, t = int(c.q_seq[i]), int(c.q_pos[i])
            ref = brute.hisa_row(c.keys, c.key_scale, c.dtype, c.Q, c.w, b, t, i, c.B, c.m, c.k)
            got = [x for x in r["idx"][i] if x >= 0]
            if got != ref["idx"]:
                return True
            if not np.allclose(r["score"][i][:len(got)], [float(v) for v in ref["scores"]],
                               rtol=1e-12, atol=1e-15):
                return True
            fref = brute.flat_row(c.keys, c.key_scale, c.dtype, c.Q, c.w, b, t, i, c.k)
            if [x for x in f["idx"][i] if x >= 0] != fref["idx"]:
                return True
    # refinement on given block lists (unsorted, -1 entries, the partial own
    # block) against the exact brute force, candidate scores slot by slot
    if _refine_fails(lib):
        return True
    # max-pooled representatives against the exact brute force
    c = make_case(batch=1, L=24, H=2, d=4, B=4, m=2, k=5, seed=311, positions=np.array([23, 13]))
    cache = oracle.Cache.of(c)
    r = oracle.hisa_select(cache, c.Q, c.w, c.q_seq, c.q_pos, c.B, c.m, c.k, threads=1, lib=lib,
                           pool="max")
    for i in range(c.n_q):
        ref = brute.hisa_row(c.keys, c.key_scale, c.dtype, c.Q, c.w, int(c.q_seq[i]),
                             int(c.q_pos[i]), i, c.B, c.m, c.k, pool="max")
        if [float(x) for x in r["block_scores"][i][:len(ref["block_scores"])]] != \
                [float(v) for v in ref["block_scores"]]:
            return True
    # the three-level search against its brute force
    c = make_case(batch=1, L=45, H=2, d=4, B=2, m=4, k=6, seed=312, positions=np.array([44, 30, 9]))
    cache = oracle.Cache.of(c)
    r = oracle.tree_select(cache, c.Q, c.w, c.q_seq, c.q_pos, 2, 3, 2, 4, 6, threads=1, lib=lib)
    for i in range(c.n_q):
        ref = brute.tree_row(c.keys, c.key_scale, c.dtype, c.Q, c.w, int(c.q_seq[i]),
                             int(c.q_pos[i]), i, 2, 3, 2, 4, 6)
        if list(r["blocks"][i][:r["nblocks"][i]]) != ref["blocks"] or \
                [x for x in r["idx"][i] if x >= 0] != ref["idx"]:
            return True
    # the search of any depth against its brute force (kept units, counts, tokens)
    c = make_case(batch=1, L=50, H=2, d=4, B=2, m=3, k=6, seed=314, positions=np.array([49, 31, 8]))
    cache = oracle.Cache.of(c)
    level_B, keep = [2, 4, 12], [3, 2, 2]
    r = oracle.levels_select(cache, c.Q, c.w, c.q_seq, c.q_pos, level_B, keep, 6, threads=1, lib=lib)
    for i in range(c.n_q):
        ref = brute.levels_row(c.keys, c.key_scale, c.dtype, c.Q, c.w, int(c.q_seq[i]),
                               int(c.q_pos[i]), i, level_B, keep, 6)
        if [x for x in r["idx"][i] if x >= 0] != ref["idx"] or tuple(r["counts"][i]) != ref["counts"]:
            return True
        for lv in range(3):
            if list(r["kept"][lv][i][:r["nkept"][i, lv]]) != ref["kept"][lv]:
                return True
    return False


def test_unmutated_oracle_passes():
    assert not _detects(oracle.load())


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(oracle.SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not unique"
    path = tmp_path / "mutant.c"
    path.write_text(src.replace(old, new))
    lib = oracle.load(oracle.build(str(path), str(tmp_path / f"lib_{name}.so")))
    assert _detects(lib), f"planted mistake {name} went unnoticed"
