"""ctypes front end of the HISA CPU oracle (``hisa_oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, the package smoke check and the bench's
CPU-baseline leg use it; the product library never does.  It imports nothing
from the product package.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(_HERE, "hisa_oracle.c")
LIB = os.path.join(_HERE, "libhisa_oracle.so")

KEY_BF16, KEY_E4M3 = 0, 1


def build(src: str = SRC, out: str = LIB, extra_flags=()) -> str:
    """Compile the oracle with gcc (plain C, no fast-math)."""
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", *extra_flags,
           src, "-o", out, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def _stale() -> bool:
    return (not os.path.exists(LIB)) or os.path.getmtime(LIB) < os.path.getmtime(SRC)


_lib = None


def load(path: Optional[str] = None):
    """Load (building if needed) the oracle shared library."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    if _lib is None:
        if _stale():
            build()
        _lib = _bind(ctypes.CDLL(LIB))
    return _lib


def _bind(lib):
    P = ctypes.c_void_p
    I = ctypes.c_int
    lib.hisa_oracle_pool.argtypes = [P, P, I, I, I, I, I, I, P, P]
    lib.hisa_oracle_select.argtypes = [P, P, I, I, I, I, I, I, P, P, P, P, P, I, I, I, I, I,
                                       P, P, P, P, P, P]
    lib.hisa_oracle_refine.argtypes = [P, P, I, I, I, I, I, P, P, P, P, P, I, I, I, P, P, I, I,
                                       P, P, P]
    lib.hisa_oracle_flat.argtypes = [P, P, I, I, I, I, P, P, P, P, P, I, I, I, I, P, P, P]
    lib.hisa_oracle_topk_f32.argtypes = [P, I, I, I, P]
    lib.hisa_oracle_tree_select.argtypes = [P, P, I, I, I, I, I, I, I, P, P, P, P, P, I, I, I, I,
                                            I, I, P, P, P, P, P, P, P]
    lib.hisa_oracle_levels_select.argtypes = [P, P, I, I, I, I, I, P, P, I, P, P, P, P, P, I, I,
                                              I, I, P, P, P, P, P]
    lib.hisa_oracle_sparse_attn.argtypes = [P, I, P, P, P, I, I, I, P, P, I, I, ctypes.c_double, I,
                                            P, P]
    for f in ("hisa_oracle_pool", "hisa_oracle_select", "hisa_oracle_refine",
              "hisa_oracle_flat", "hisa_oracle_topk_f32", "hisa_oracle_tree_select",
              "hisa_oracle_levels_select", "hisa_oracle_sparse_attn"):
        getattr(lib, f).restype = I
    return lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def default_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


class Cache:
    """Key cache view: keys [batch, cap, d] (bf16 bits / e4m3 codes), scale, lens."""

    def __init__(self, keys, key_scale, lens, dtype: str):
        self.dtype = KEY_BF16 if dtype == "bf16" else KEY_E4M3
        self.keys = np.ascontiguousarray(keys)
        assert self.keys.dtype == (np.uint16 if self.dtype == KEY_BF16 else np.uint8)
        self.scale = _c(key_scale, np.float32) if self.dtype == KEY_E4M3 else None
        self.lens = _c(lens, np.int32)
        self.batch, self.cap, self.d = self.keys.shape

    @classmethod
    def of(cls, case, lens=None):
        return cls(case.keys, case.key_scale, case.lens if lens is None else lens, case.dtype)

    def args(self):
        return (_p(self.keys), _p(self.scale), self.dtype, self.batch, self.cap, self.d)


POOL_MODES = {"mean": 0, "max": 1}


def pool(cache: Cache, B: int, lib=None, mode: str = "mean") -> np.ndarray:
    """Cache-level block representatives [batch, ceil(cap/B), d]: means, or
    elementwise maxima with mode="max" (double; NaN where unpooled)."""
    lib = lib or load()
    nblk = -(-cache.cap // B)
    out = np.full((cache.batch, nblk, cache.d), np.nan)
    rc = lib.hisa_oracle_pool(*cache.args(), B, POOL_MODES[mode], _p(cache.lens), _p(out))
    if rc:
        raise ValueError(f"hisa_oracle_pool rc={rc}")
    return out


def _queries(Q, w, q_seq, q_pos):
    Q = _c(Q, np.uint16)
    w = _c(w, np.float32)
    q_seq = _c(q_seq, np.int32)
    q_pos = _c(q_pos, np.int32)
    n_q, H, _ = Q.shape
    return Q, w, q_seq, q_pos, n_q, H


def hisa_select(cache: Cache, Q, w, q_seq, q_pos, B: int, m: int, k: int,
                threads: Optional[int] = None, lib=None, pool: str = "mean") -> dict:
    """The two-stage HISA selection, step by step, for every query row
    (block representatives by mean or, with pool="max", elementwise max)."""
    lib = lib or load()
    Q, w, q_seq, q_pos, n_q, H = _queries(Q, w, q_seq, q_pos)
    nbmax = -(-cache.cap // B)
    idx = np.empty((n_q, k), np.int32)
    score = np.empty((n_q, k))
    blocks = np.empty((n_q, m), np.int32)
    nblocks = np.empty(n_q, np.int32)
    bscores = np.empty((n_q, nbmax))
    counts = np.empty((n_q, 2), np.int64)
    rc = lib.hisa_oracle_select(*cache.args(), B, POOL_MODES[pool], _p(cache.lens), _p(Q), _p(w),
                                _p(q_seq),
                                _p(q_pos), n_q, H, m, k, threads or default_threads(),
                                _p(idx), _p(score), _p(blocks), _p(nblocks), _p(bscores),
                                _p(counts))
    if rc:
        raise ValueError(f"hisa_oracle_select rc={rc}")
    return dict(idx=idx, score=score, blocks=blocks, nblocks=nblocks, block_scores=bscores,
                counts=counts)


def tree_select(cache: Cache, Q, w, q_seq, q_pos, B: int, bf: int, W: int, m: int, k: int,
                threads: Optional[int] = None, lib=None, pool: str = "mean") -> dict:
    """Three-level search: superblocks of bf blocks (own + best W - 1), then the
    blocks under them (own + best m - 1), then their tokens (top k)."""
    lib = lib or load()
    Q, w, q_seq, q_pos, n_q, H = _queries(Q, w, q_seq, q_pos)
    idx = np.empty((n_q, k), np.int32)
    score = np.empty((n_q, k))
    sblocks = np.empty((n_q, W), np.int32)
    nsblocks = np.empty(n_q, np.int32)
    blocks = np.empty((n_q, m), np.int32)
    nblocks = np.empty(n_q, np.int32)
    counts = np.empty((n_q, 3), np.int64)
    rc = lib.hisa_oracle_tree_select(*cache.args(), B, bf, POOL_MODES[pool], _p(cache.lens), _p(Q),
                                     _p(w), _p(q_seq), _p(q_pos), n_q, H, W, m, k,
                                     threads or default_threads(), _p(idx), _p(score), _p(sblocks),
                                     _p(nsblocks), _p(blocks), _p(nblocks), _p(counts))
    if rc:
        raise ValueError(f"hisa_oracle_tree_select rc={rc}")
    return dict(idx=idx, score=score, sblocks=sblocks, nsblocks=nsblocks, blocks=blocks,
                nblocks=nblocks, counts=counts)


def levels_select(cache: Cache, Q, w, q_seq, q_pos, level_B, keep, k: int,
                  threads: Optional[int] = None, lib=None, pool: str = "mean") -> dict:
    """Search of any depth.  Level l (finest first) groups the keys into units
    of level_B[l] tokens, each size a multiple of the one below; from the
    coarsest level down, the own unit plus the best keep[l] - 1 candidates
    (every visible unit at the top, the units inside the kept ones below)
    are kept; then the tokens of the kept level-0 blocks (top k).  kept[l] is
    [n_q, keep[l]] (ascending, -1 padded), nkept [n_q, levels], counts
    [n_q, levels + 1] (units scored per level, then token slots)."""
    lib = lib or load()
    Q, w, q_seq, q_pos, n_q, H = _queries(Q, w, q_seq, q_pos)
    nl = len(level_B)
    lb = np.ascontiguousarray(level_B, np.int32)
    kp = np.ascontiguousarray(keep, np.int32)
    idx = np.empty((n_q, k), np.int32)
    score = np.empty((n_q, k))
    kept = np.empty((n_q, int(kp.sum())), np.int32)
    nkept = np.empty((n_q, nl), np.int32)
    counts = np.empty((n_q, nl + 1), np.int64)
    rc = lib.hisa_oracle_levels_select(*cache.args(), nl, _p(lb), _p(kp), POOL_MODES[pool],
                                       _p(cache.lens), _p(Q), _p(w), _p(q_seq), _p(q_pos), n_q, H, k,
                                       threads or default_threads(), _p(idx), _p(score), _p(kept),
                                       _p(nkept), _p(counts))
    if rc:
        raise ValueError(f"hisa_oracle_levels_select rc={rc}")
    off = np.concatenate([[0], np.cumsum(kp)])
    return dict(idx=idx, score=score, kept=[kept[:, off[l]:off[l + 1]] for l in range(nl)],
                nkept=nkept, counts=counts)


def hisa_refine(cache: Cache, Q, w, q_seq, q_pos, B: int, k: int, blocks, nblocks,
                want_candidates: bool = True, threads: Optional[int] = None, lib=None) -> dict:
    """Token-level refinement (score + top-k) on a GIVEN block set per row."""
    lib = lib or load()
    Q, w, q_seq, q_pos, n_q, H = _queries(Q, w, q_seq, q_pos)
    blocks = _c(blocks, np.int32)
    nblocks = _c(nblocks, np.int32)
    mm = blocks.shape[1]
    idx = np.empty((n_q, k), np.int32)
    score = np.empty((n_q, k))
    cand = np.empty((n_q, mm * B)) if want_candidates else None
    rc = lib.hisa_oracle_refine(*cache.args(), B, _p(cache.lens), _p(Q), _p(w), _p(q_seq),
                                _p(q_pos), n_q, H, k, _p(blocks), _p(nblocks), mm,
                                threads or default_threads(), _p(idx), _p(score), _p(cand))
    if rc:
        raise ValueError(f"hisa_oracle_refine rc={rc}")
    return dict(idx=idx, score=score, cand_scores=cand)


def flat_select(cache: Cache, Q, w, q_seq, q_pos, k: int, want_all: bool = False,
                threads: Optional[int] = None, lib=None) -> dict:
    """The flat DSA scan: every visible token scored, top-k kept."""
    lib = lib or load()
    Q, w, q_seq, q_pos, n_q, H = _queries(Q, w, q_seq, q_pos)
    idx = np.empty((n_q, k), np.int32)
    score = np.empty((n_q, k))
    allv = np.empty((n_q, cache.cap)) if want_all else None
    rc = lib.hisa_oracle_flat(*cache.args(), _p(cache.lens), _p(Q), _p(w), _p(q_seq),
                              _p(q_pos), n_q, H, k, threads or default_threads(), _p(idx),
                              _p(score), _p(allv))
    if rc:
        raise ValueError(f"hisa_oracle_flat rc={rc}")
    return dict(idx=idx, score=score, all_scores=allv)


def topk_f32(x, k: int, lib=None) -> np.ndarray:
    """Selection rule on given fp32 rows: [rows, n] -> [rows, k] ascending indices, -1 pad."""
    lib = lib or load()
    x = _c(x, np.float32)
    rows, n = x.shape
    idx = np.empty((rows, k), np.int32)
    rc = lib.hisa_oracle_topk_f32(_p(x), rows, n, k, _p(idx))
    if rc:
        raise ValueError(f"hisa_oracle_topk_f32 rc={rc}")
    return idx


def sparse_attn(Qa, K, V, lens, q_seq, idx, scale: float, threads: Optional[int] = None,
                lib=None):
    """Attention of each query row over its selected entries (the plain
    definition, in double).  Qa [n_q, Ha, d], K, V [batch, cap, d] as bf16
    bits (uint16); idx [n_q, k] (-1 or >= len: skipped).  Returns (out
    [n_q, Ha, d], lse [n_q, Ha])."""
    lib = lib or load()
    Qa = _c(Qa, np.uint16)
    K = _c(K, np.uint16)
    V = _c(V, np.uint16)
    lens = _c(lens, np.int32)
    q_seq = _c(q_seq, np.int32)
    idx = _c(idx, np.int32)
    n_q, Ha, d = Qa.shape
    batch, cap, _ = K.shape
    k = idx.shape[1]
    out = np.empty((n_q, Ha, d))
    lse = np.empty((n_q, Ha))
    rc = lib.hisa_oracle_sparse_attn(_p(Qa), Ha, _p(K), _p(V), _p(lens), batch, cap, d, _p(q_seq),
                                     _p(idx), n_q, k, float(scale), threads or default_threads(),
                                     _p(out), _p(lse))
    if rc:
        raise ValueError(f"hisa_oracle_sparse_attn rc={rc}")
    return out, lse
