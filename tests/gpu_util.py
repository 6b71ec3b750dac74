"""Shared helpers of the GPU parity tests: run the library on a seeded case and
bring the results back as numpy arrays."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from hisa_inputs import bf16_bits


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


def pooled_tol(case, ora_pooled, B):
    """|delta| <= 1e-5 * (|mu| + mean|v|) per element: the fp32 sum of n <= B
    terms is within about n * 2^-24 * sum|v| of the exact sum."""
    from hisa_inputs import bf16_to_f32, e4m3_to_f32
    if case.dtype == "bf16":
        v = np.abs(bf16_to_f32(case.keys).astype(np.float64))
    else:
        v = np.abs((e4m3_to_f32(case.keys) * case.key_scale[..., None]).astype(np.float64))
    mav = np.zeros_like(ora_pooled)
    for b in range(case.batch):
        n = int(case.lens[b])
        for j in range(-(-n // B)):
            mav[b, j] = v[b, j * B:min((j + 1) * B, n)].mean(0)
    return 1e-5 * (np.abs(ora_pooled) + mav)


def check_pooled(case, kv):
    B = case.B
    got = kv.pooled.cpu().numpy().astype(np.float64)
    ora = oracle.pool(oracle.Cache.of(case), B)
    tol = pooled_tol(case, ora, B)
    for b in range(case.batch):
        nbv = -(-int(case.lens[b]) // B)
        d = np.abs(got[b, :nbv] - ora[b, :nbv])
        assert np.all(d <= tol[b, :nbv]), f"seq {b}: max excess {(d - tol[b, :nbv]).max()}"
    # hi/lo split of the fp32 mean
    hl = kv.pooled_hl.view(torch.int16).cpu().numpy().view(np.uint16).astype(np.uint32)
    hi = (hl[..., :case.d] << 16).view(np.float32)
    lo = (hl[..., case.d:] << 16).view(np.float32)
    g32 = kv.pooled.cpu().numpy()
    for b in range(case.batch):
        nbv = -(-int(case.lens[b]) // B)
        assert np.array_equal(bf16_bits(g32[b, :nbv]), hl[b, :nbv, :case.d].astype(np.uint16))
        assert np.array_equal(bf16_bits(g32[b, :nbv] - hi[b, :nbv]),
                              hl[b, :nbv, case.d:].astype(np.uint16))
        assert np.all(np.abs((hi + lo)[b, :nbv] - g32[b, :nbv]) <= 2.0 ** -15 * np.abs(g32[b, :nbv]) + 1e-30)
    return ora


class AppendRecorder:
    """Checks every append, not only the final state: after each hisa_append,
    `record(kv)` keeps a copy of each sequence's trailing block (the block
    that holds key len - 1: its pooled and pooled_hl rows and its valid key
    count).  `verify(kv)` then pools each recorded block from scratch in a
    separate cache (one sequence per record, the block's keys taken from the
    final cache: an append never rewrites an earlier key) and requires
    (1) the incremental rows to equal that re-pool bit for bit, and (2) the
    re-pooled means to match the oracle's within the pooled tolerance."""

    def __init__(self):
        self.seq, self.blk, self.cnt, self.rows, self.hl = [], [], [], [], []

    def record(self, kv):
        n = kv.len.to(torch.int64)
        j = torch.div(n - 1, kv.B, rounding_mode="floor")
        b = torch.arange(kv.batch, device=n.device)
        self.seq.append(b)
        self.blk.append(j)
        self.cnt.append(n - j * kv.B)
        self.rows.append(kv.pooled[b, j].clone())
        self.hl.append(kv.pooled_hl[b, j].clone())

    def verify(self, kv, pool="mean"):
        from types import SimpleNamespace
        h = lib()
        seq = torch.cat(self.seq).cpu().numpy()
        blk = torch.cat(self.blk).cpu().numpy()
        cnt = torch.cat(self.cnt).cpu().numpy()
        R, B, d = len(seq), kv.B, kv.d
        assert np.all((cnt >= 1) & (cnt <= B))
        kk = kv.keys.view(torch.int16 if kv.dtype == "bf16" else torch.uint8).cpu().numpy()
        keys = np.zeros((R, B, d), kk.dtype)
        scale = np.ones((R, B), np.float32) if kv.dtype == "e4m3" else None
        sc_all = kv.key_scale.cpu().numpy() if kv.dtype == "e4m3" else None
        for r in range(R):
            s0 = int(blk[r]) * B
            keys[r, :cnt[r]] = kk[seq[r], s0:s0 + cnt[r]]
            if scale is not None:
                scale[r, :cnt[r]] = sc_all[seq[r], s0:s0 + cnt[r]]
        fresh = h.KVCache(R, B, d, B, kv.dtype, device=kv.device, pool=pool)
        fresh.load(torch.from_numpy(keys), torch.from_numpy(cnt.astype(np.int32)),
                   None if scale is None else torch.from_numpy(scale))
        h.hisa_pool_blocks(fresh)
        torch.cuda.synchronize()
        inc = torch.cat(self.rows)
        inc_hl = torch.cat(self.hl)
        bad = [r for r in range(R) if not torch.equal(inc[r], fresh.pooled[r, 0])
               or not torch.equal(inc_hl[r], fresh.pooled_hl[r, 0])]
        assert not bad, f"{len(bad)} of {R} appends differ from a re-pool (first: record {bad[0]})"
        if pool == "mean":
            case = SimpleNamespace(keys=keys.view(np.uint16) if kv.dtype == "bf16" else keys,
                                   key_scale=scale, lens=cnt.astype(np.int32), batch=R, d=d, B=B,
                                   dtype=kv.dtype)
            check_pooled(case, fresh)
        else:
            ora = oracle.pool(oracle.Cache(keys.view(np.uint16) if kv.dtype == "bf16" else keys, scale,
                                           cnt.astype(np.int32), kv.dtype), B, mode="max")
            assert np.array_equal(fresh.pooled.cpu().numpy()[:, 0].astype(np.float64), ora[:, 0])
        return R
