"""Shared helpers of the GPU parity tests: run the library on a seeded case and
bring the results back as numpy arrays."""
from __future__ import annotations

import numpy as np
import torch

import oracle


def lib():
    import hierarchical_top_indexer_b200 as h
    return h


def device_case(case, pool="mean"):
    h = lib()
    kv = h.KVCache.from_case(case, pool=pool)
    h.hisa_pool_blocks(kv)
    return kv


def queries(case):
    return (torch.from_numpy(case.Q.view(np.int16)).view(torch.bfloat16).cuda(),
            torch.from_numpy(case.w).cuda(), torch.from_numpy(case.q_seq).cuda(),
            torch.from_numpy(case.q_pos).cuda())


def run_hisa(case, kv, m=None, k=None, q_pos_null=False):
    h = lib()
    Q, w, qs, qp = queries(case)
    r = h.hisa_select_inspect(kv, Q, w, qs, None if q_pos_null else qp, m or case.m, k or case.k)
    torch.cuda.synchronize()
    return {key: v.cpu().numpy() for key, v in r.items()}


def run_flat(case, kv, k=None):
    h = lib()
    Q, w, qs, qp = queries(case)
    idx, sc = h.dsa_flat_select(kv, Q, w, qs, qp, k or case.k, want_scores=True)
    torch.cuda.synchronize()
    return dict(idx=idx.cpu().numpy(), scores=sc.cpu().numpy())


def oracle_rows(case, rows):
    """Sub-select query rows (for oracles on large cases)."""
    rows = np.asarray(rows)
    return (case.Q[rows], case.w[rows], case.q_seq[rows], case.q_pos[rows])


def check_hisa(case, gpu, rows=None, threads=None, m=None, k=None, pool="mean"):
    """Apply the two-level parity rule to the GPU result on the given rows."""
    from tests.parity import hisa_row_check
    m = m or case.m
    k = k or case.k
    rows = np.arange(case.n_q) if rows is None else np.asarray(rows)
    cache = oracle.Cache.of(case)
    Q, w, qs, qp = oracle_rows(case, rows)
    ora = oracle.hisa_select(cache, Q, w, qs, qp, case.B, m, k, threads=threads, pool=pool)
    mm = gpu["blocks"].shape[1]
    ref = oracle.hisa_refine(cache, Q, w, qs, qp, case.B, k, gpu["blocks"][rows],
                             gpu["nblocks"][rows], threads=threads)
    swaps = []
    sub = {key: v[rows] for key, v in gpu.items()}
    for r, i in enumerate(rows):
        swaps.append(hisa_row_check(r, sub, ora, ref, case.B, m, k, int(case.q_pos[i])))
    return ora, swaps


def check_flat(case, gpu, rows=None, threads=None, k=None):
    from tests.parity import check_scores, check_selection
    k = k or case.k
    rows = np.arange(case.n_q) if rows is None else np.asarray(rows)
    cache = oracle.Cache.of(case)
    Q, w, qs, qp = oracle_rows(case, rows)
    ora = oracle.flat_select(cache, Q, w, qs, qp, k, want_all=True, threads=threads)
    swaps = []
    for r, i in enumerate(rows):
        t = int(case.q_pos[i])
        cand = {s: float(ora["all_scores"][r, s]) for s in range(t + 1)}
        swaps.append(check_selection(gpu["idx"][i], cand, k, "flat tokens"))
        check_scores(gpu["idx"][i], gpu["scores"][i], cand, "flat scores")
    return ora, swaps
