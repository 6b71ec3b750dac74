"""Seeded synthetic inputs for the HISA indexer.

This module only draws random numbers and stores them in the formats the
indexer consumes (bf16 bit patterns, OCP e4m3 bytes with a per-token fp32
scale, fp32 head weights, int32 positions).  It holds none of the indexer's
arithmetic: no pooling, no scoring, no selection.  Both the CPU oracle and the
CUDA library read their inputs from here, so it is the one thing they share.

Recipe (block-clustered keys, as the HISA workloads describe them):

* per sequence, block centres mu_j ~ N(0, 1) in R^d for every block of size B
  the cache can hold (appended rows continue the same clusters);
* token noise eps_s ~ N(0, 0.5^2);
* key k_s = (mu_{floor(s/B)} + eps_s) / sqrt(d), stored as bf16 (round to
  nearest even) or as e4m3 codes with scale = max|k_s| / 448 (scale 1 for an
  all-zero row, round to nearest even, saturating at 448);
* queries q ~ N(0, 1) / sqrt(d) as bf16, head weights w ~ U(0, 1) as fp32;
* draw order per case: all sequences' (mu, eps) in sequence order, then Q,
  then w, then the appended rows (noise, then their queries and weights).

Everything comes from one ``numpy.random.Generator(PCG64(seed))``.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np

SEED_BASE = 20260330
E4M3_MAX = 448.0

# --------------------------------------------------------------------------
# storage formats
# --------------------------------------------------------------------------


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit pattern, round to nearest, ties to even (finite input)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounded = u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return (rounded >> np.uint32(16)).astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit pattern -> the exact fp32 value."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def e4m3_codes(x: np.ndarray) -> np.ndarray:
    """fp32 -> OCP e4m3 (the 'fn' variant: no inf, max 448) byte codes.

    Round to nearest even on the e4m3 grid, saturating at +-448.  The grid
    spacing at binade E (|x| in [2^E, 2^(E+1)), E >= -6) is 2^(E-3); below
    2^-6 the subnormal spacing 2^-9 applies.  With r = rint(|x| / spacing) the
    code is ((E + 7) << 3) + r - 8, which also covers the carry into the next
    binade (r = 16) and the subnormal range (E = -6, r < 8).
    """
    x = np.asarray(x, dtype=np.float32)
    a = np.abs(x).astype(np.float32)
    _, e = np.frexp(a)                    # a = f * 2^e, f in [0.5, 1)
    E = np.maximum(e.astype(np.int32) - 1, -6)
    r = np.rint(np.ldexp(a, 3 - E)).astype(np.int32)   # exact scaling by 2^(3-E)
    code = ((E + 7) << 3) + r - 8
    code = np.where(a == 0, 0, code)
    code = np.minimum(code, 0x7E)          # saturate at 448
    sign = np.where(x < 0, 0x80, 0)
    return (code | sign).astype(np.uint8)


def e4m3_to_f32(codes: np.ndarray) -> np.ndarray:
    """e4m3 byte codes -> exact fp32 values (0x7F / 0xFF are NaN)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int32)
    s = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 15
    m = c & 7
    v = np.where(e == 0, np.ldexp(m.astype(np.float64), -9),
                 np.ldexp(1.0 + m / 8.0, e - 7))
    v = np.where((c & 0x7F) == 0x7F, np.nan, v)
    return (s * v).astype(np.float32)


def quantize_e4m3_rows(k: np.ndarray):
    """Per-token e4m3 quantisation: returns (codes [.., d] uint8, scale [..] fp32)."""
    k = np.asarray(k, dtype=np.float32)
    amax = np.max(np.abs(k), axis=-1)
    scale = (amax / np.float32(E4M3_MAX)).astype(np.float32)
    scale = np.where(amax == 0, np.float32(1.0), scale).astype(np.float32)
    codes = e4m3_codes(k / scale[..., None])
    return codes, scale


# --------------------------------------------------------------------------
# cases
# --------------------------------------------------------------------------


@dataclass
class Case:
    """One seeded workload.  Arrays are host numpy arrays, C-contiguous.

    keys      [batch, cap, d]  uint16 (bf16 bits) or uint8 (e4m3 codes)
    key_scale [batch, cap]     float32, only for e4m3 (else None)
    lens      [batch]          int32, valid prefix length per sequence
    Q         [n_q, H, d]      uint16 bf16 bits
    w         [n_q, H]         float32
    q_seq     [n_q]            int32 sequence of each query row
    q_pos     [n_q]            int32 causal position of each query row
    append_*  rows appended one step at a time (streaming decode)
    """
    name: str
    seed: int
    dtype: str
    batch: int
    cap: int
    d: int
    H: int
    B: int
    m: int
    k: int
    keys: np.ndarray
    key_scale: Optional[np.ndarray]
    lens: np.ndarray
    Q: np.ndarray
    w: np.ndarray
    q_seq: np.ndarray
    q_pos: np.ndarray
    append_keys: Optional[np.ndarray] = None      # [steps, batch, d]
    append_scale: Optional[np.ndarray] = None     # [steps, batch]
    append_Q: Optional[np.ndarray] = None         # [sets, batch, H, d] (step s: set s % sets)
    append_w: Optional[np.ndarray] = None         # [sets, batch, H]
    meta: dict = field(default_factory=dict)

    @property
    def n_q(self) -> int:
        return int(self.q_pos.shape[0])

    @property
    def nblk(self) -> int:
        return -(-self.cap // self.B)


def _store_keys(k32: np.ndarray, dtype: str):
    if dtype == "bf16":
        return bf16_bits(k32), None
    if dtype == "e4m3":
        return quantize_e4m3_rows(k32)
    raise ValueError(f"unknown key dtype {dtype!r}")


def make_case(*, batch: int, L, H: int, d: int, B: int, m: int, k: int,
              positions=None, dtype: str = "bf16", seed: int = SEED_BASE,
              cap: Optional[int] = None, append_steps: int = 0,
              cluster_B: Optional[int] = None, noise: float = 0.5,
              append_query_sets: Optional[int] = None, name: str = "case") -> Case:
    """Build a case.

    L          prefix length, an int or one int per sequence.
    positions  query positions: None -> one row per sequence at its last
               position; an int array -> the same positions in every
               sequence; a list of arrays -> per sequence.
    cluster_B  block size of the synthetic clusters (defaults to B).
    append_query_sets  number of per-step query sets drawn for the appended
               steps (default: one per step; step s uses set s % sets).
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    Ls = np.full(batch, L, dtype=np.int64) if np.isscalar(L) else np.asarray(L, dtype=np.int64)
    assert Ls.shape == (batch,)
    cap = int(cap if cap is not None else Ls.max() + append_steps)
    assert cap >= Ls.max() + append_steps
    cB = int(cluster_B or B)
    n_clusters = -(-cap // cB)
    inv_sqrt_d = np.float32(1.0 / np.sqrt(d))

    kdt = np.uint16 if dtype == "bf16" else np.uint8
    keys = np.zeros((batch, cap, d), dtype=kdt)
    key_scale = np.ones((batch, cap), dtype=np.float32) if dtype == "e4m3" else None
    mus = []
    for b in range(batch):
        mu = rng.standard_normal((n_clusters, d), dtype=np.float32)
        mus.append(mu)
        Lb = int(Ls[b])
        eps = rng.standard_normal((Lb, d), dtype=np.float32)
        eps *= np.float32(noise)
        eps += mu[np.arange(Lb) // cB]
        eps *= inv_sqrt_d
        codes, sc = _store_keys(eps, dtype)
        keys[b, :Lb] = codes
        if sc is not None:
            key_scale[b, :Lb] = sc
        del eps

    if positions is None:
        per_seq = [np.array([Ls[b] - 1]) for b in range(batch)]
    elif isinstance(positions, (list, tuple)):
        per_seq = [np.asarray(p) for p in positions]
    else:
        per_seq = [np.asarray(positions) for _ in range(batch)]
    q_seq = np.concatenate([np.full(len(p), b) for b, p in enumerate(per_seq)]).astype(np.int32)
    q_pos = np.concatenate(per_seq).astype(np.int32)
    for b, p in enumerate(per_seq):
        assert np.all((p >= 0) & (p < Ls[b])), "query position outside the prefix"
    n_q = len(q_pos)
    Q = bf16_bits(rng.standard_normal((n_q, H, d), dtype=np.float32) * inv_sqrt_d)
    w = rng.random((n_q, H), dtype=np.float32)

    case = Case(name=name, seed=seed, dtype=dtype, batch=batch, cap=cap, d=d, H=H,
                B=B, m=m, k=k, keys=keys, key_scale=key_scale,
                lens=Ls.astype(np.int32), Q=Q, w=w, q_seq=q_seq, q_pos=q_pos)

    if append_steps:
        ak = np.zeros((append_steps, batch, d), dtype=kdt)
        asc = np.ones((append_steps, batch), dtype=np.float32) if dtype == "e4m3" else None
        for b in range(batch):
            pos = Ls[b] + np.arange(append_steps)
            eps = rng.standard_normal((append_steps, d), dtype=np.float32)
            eps *= np.float32(noise)
            eps += mus[b][pos // cB]
            eps *= inv_sqrt_d
            codes, sc = _store_keys(eps, dtype)
            ak[:, b] = codes
            if sc is not None:
                asc[:, b] = sc
        case.append_keys = ak
        case.append_scale = asc
        nsets = append_steps if append_query_sets is None else min(append_query_sets, append_steps)
        case.append_Q = bf16_bits(
            rng.standard_normal((nsets, batch, H, d), dtype=np.float32) * inv_sqrt_d)
        case.append_w = rng.random((nsets, batch, H), dtype=np.float32)
    return case


# The five workloads: shapes and sizes of the pages' settings (32K-128K
# contexts, top-k 2048), scaled per the block-clustered recipe above.
CONFIGS = {
    0: dict(name="tiny-decode-2k", batch=1, L=2048, positions=np.arange(2032, 2048),
            H=4, d=64, B=64, m=8, k=128, dtype="bf16"),
    1: dict(name="decode-32k-b64", batch=64, L=32768, positions=None,
            H=64, d=128, B=128, m=64, k=2048, dtype="bf16"),
    2: dict(name="prefill-64k-chunk4096", batch=1, L=65536,
            positions=np.arange(65536 - 4096, 65536),
            H=64, d=128, B=128, m=64, k=2048, dtype="bf16"),
    3: dict(name="decode-128k-b32-e4m3", batch=32, L=131072, positions=None,
            H=64, d=128, B=128, m=128, k=2048, dtype="e4m3"),
    4: dict(name="stream-append-128k", batch=1, L=131072, positions=None,
            H=64, d=128, B=128, m=64, k=2048, dtype="bf16", append_steps=512),
}


def make_config(i: int, seed: Optional[int] = None, **overrides) -> Case:
    """Workload ``i`` (0..4) with seed SEED_BASE + i unless given."""
    spec = dict(CONFIGS[i])
    spec.update(overrides)
    return make_case(seed=SEED_BASE + i if seed is None else seed, **spec)
