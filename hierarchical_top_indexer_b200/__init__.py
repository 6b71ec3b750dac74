"""HISA hierarchical top-k indexer on B200 — Python binding of libhisa_b200.so.

Argument marshalling only: every step of the indexer runs in the library's
CUDA kernels (see include/hisa.h for the contract of each call).  PyTorch
provides device memory and the current CUDA stream.  There is no CPU or
PyTorch fallback: if the library is missing, importing this package fails.

    import hierarchical_top_indexer_b200 as hisa
    kv = hisa.KVCache(batch, cap, d=128, B=128, dtype="bf16")
    kv.load(keys_bf16, lens)             # host or device tensors
    hisa.hisa_pool_blocks(kv)
    idx = hisa.hisa_select(kv, Q, w, q_seq, q_pos, m=64, k=2048)

    # a deeper search: coarser indexes over the same keys, finest first
    kvs = [kv] + [hisa.superblock_index(kv, f) for f in (8, 64)]
    for c in kvs[1:]:
        hisa.hisa_pool_blocks(c)
    idx = hisa.hisa_levels_select(kvs, Q, w, q_seq, q_pos, keep=[64, 32, 8], k=2048)
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhisa_b200.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python hierarchical_top_indexer_b200/build.py` "
        "(there is no fallback implementation)")

_lib = ctypes.CDLL(LIB_PATH)

HISA_KEY_BF16, HISA_KEY_E4M3 = 0, 1
HISA_POOL_MEAN, HISA_POOL_MAX = 0, 1
HISA_OK, HISA_E_INVAL, HISA_E_UNSUPPORTED, HISA_E_WORKSPACE, HISA_E_CUDA = range(5)
HISA_E_SCRATCH_LIMIT = 5
HISA_STATIC_SCRATCH_BYTES = 8 << 20
HISA_DEV_BAD_QUERY, HISA_DEV_CAPACITY, HISA_DEV_BAD_LEN, HISA_DEV_TIMEOUT = 0x1, 0x2, 0x4, 0x8

EXPORTS = ("hisa_pool_blocks", "hisa_append", "hisa_select_workspace_bytes", "hisa_select",
           "hisa_decode_step_workspace_bytes", "hisa_decode_step",
           "hisa_select_inspect", "hisa_select_static", "hisa_tree_workspace_bytes",
           "hisa_tree_select", "hisa_pool_tail", "hisa_levels_workspace_bytes", "hisa_levels_select",
           "hisa_cp_workspace_bytes", "hisa_cp_blocks",
           "hisa_cp_tokens", "hisa_merge_topk", "hisa_sparse_attn_workspace_bytes", "hisa_sparse_attn",
           "dsa_flat_workspace_bytes", "dsa_flat_select", "hisa_topk_f32",
           "hisa_profile_enable", "hisa_profile_read", "hisa_status_string", "hisa_last_cuda_error",
           "hisa_selftest_wait")
PHASES = ("block_score", "block_select", "token_score", "token_select", "flat_score",
          "flat_select", "pool", "append", "topk", "qsplit", "merge", "attn")


class hisa_kv(ctypes.Structure):
    _fields_ = [("keys", ctypes.c_void_p), ("key_scale", ctypes.c_void_p),
                ("pooled", ctypes.c_void_p), ("pooled_hl", ctypes.c_void_p),
                ("len", ctypes.c_void_p), ("status", ctypes.c_void_p),
                ("batch", ctypes.c_int32), ("cap", ctypes.c_int32), ("d", ctypes.c_int32),
                ("B", ctypes.c_int32), ("dtype", ctypes.c_int32), ("pool", ctypes.c_int32)]


_P, _I, _Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
_KVP = ctypes.POINTER(hisa_kv)
_lib.hisa_pool_blocks.argtypes = [_KVP, _P]
_lib.hisa_append.argtypes = [_KVP, _P, _P, _P]
_lib.hisa_select_workspace_bytes.argtypes = [_KVP, _I, _I, _I, _I]
_lib.hisa_select_workspace_bytes.restype = _Z
_lib.hisa_select.argtypes = [_KVP, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P, _P, _Z, _P]
_lib.hisa_decode_step_workspace_bytes.argtypes = [_KVP, _I, _I, _I]
_lib.hisa_decode_step_workspace_bytes.restype = _Z
_lib.hisa_decode_step.argtypes = [_KVP, _P, _P, _P, _P, _I, _I, _I, _P, _P, _P, _Z, _P]
_lib.hisa_select_inspect.argtypes = [_KVP, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P, _P, _P, _P,
                                     _P, _Z, _P]
_lib.hisa_select_static.argtypes = [_KVP, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P, _P]
_lib.hisa_tree_workspace_bytes.argtypes = [_KVP, _KVP, _I, _I, _I, _I, _I]
_lib.hisa_tree_workspace_bytes.restype = _Z
_lib.hisa_tree_select.argtypes = [_KVP, _KVP, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P,
                                  _P, _P, _P, _Z, _P]
_lib.hisa_pool_tail.argtypes = [_KVP, _P]
_lib.hisa_levels_workspace_bytes.argtypes = [_P, _I, _P, _I, _I, _I]
_lib.hisa_levels_workspace_bytes.restype = _Z
_lib.hisa_levels_select.argtypes = [_P, _I, _P, _P, _P, _P, _P, _I, _I, _I, _P, _P, _P, _P, _P, _P, _Z,
                                    _P]
_lib.hisa_cp_workspace_bytes.argtypes = [_KVP, ctypes.c_int32, _I, _I, _I, _I]
_lib.hisa_cp_workspace_bytes.restype = _Z
_lib.hisa_cp_blocks.argtypes = [_KVP, ctypes.c_int32, _P, _P, _P, _P, _I, _I, _I, _P, _P, _P, _Z, _P]
_lib.hisa_cp_tokens.argtypes = [_KVP, ctypes.c_int32, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P, _P, _P,
                                _Z, _P]
_lib.hisa_merge_topk.argtypes = [_P, _P, _I, _I, _I, _I, _P, _P, _P]
_lib.hisa_sparse_attn_workspace_bytes.argtypes = [_I, _I]
_lib.hisa_sparse_attn_workspace_bytes.restype = _Z
_lib.hisa_sparse_attn.argtypes = [_P, _I, _P, _P, _P, _I, _I, _I, _P, _P, _I, _I, ctypes.c_float, _P, _P,
                                  _P, _P, _Z, _P]
_lib.dsa_flat_workspace_bytes.argtypes = [_KVP, _I, _I, _I]
_lib.dsa_flat_workspace_bytes.restype = _Z
_lib.dsa_flat_select.argtypes = [_KVP, _P, _P, _P, _P, _I, _I, _I, _P, _P, _P, _Z, _P]
_lib.hisa_topk_f32.argtypes = [_P, _I, _I, _I, _P, _P]
_lib.hisa_selftest_wait.argtypes = [_P, _P]
_lib.hisa_selftest_wait.restype = _I
_lib.hisa_profile_enable.argtypes = [_I]
_lib.hisa_profile_read.argtypes = [_P, _P, _I]
_lib.hisa_status_string.argtypes = [_I]
_lib.hisa_status_string.restype = ctypes.c_char_p
_lib.hisa_last_cuda_error.argtypes = []
_lib.hisa_last_cuda_error.restype = ctypes.c_char_p
for _f in ("hisa_pool_blocks", "hisa_append", "hisa_select", "hisa_decode_step", "hisa_select_inspect",
           "hisa_select_static",
           "hisa_tree_select", "hisa_pool_tail", "hisa_levels_select", "hisa_cp_blocks", "hisa_cp_tokens",
           "hisa_merge_topk",
           "hisa_sparse_attn", "dsa_flat_select", "hisa_topk_f32", "hisa_profile_enable", "hisa_profile_read"):
    getattr(_lib, _f).restype = _I


class HisaError(RuntimeError):
    def __init__(self, fn: str, code: int):
        msg = f"{fn}: {_lib.hisa_status_string(code).decode()} (code {code})"
        if code == HISA_E_CUDA:
            msg += f": {_lib.hisa_last_cuda_error().decode()}"
        super().__init__(msg)
        self.code = code


def _check(fn: str, code: int):
    if code != HISA_OK:
        raise HisaError(fn, code)


def lib():
    """The loaded ctypes library (for direct C-ABI calls)."""
    return _lib


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    assert t.is_contiguous(), "tensors passed to the library must be contiguous"
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dev(x, dtype, device):
    if isinstance(x, torch.Tensor) and x.dtype == dtype and x.is_cuda and x.is_contiguous() and \
            x.device.index == (device.index if device.index is not None else torch.cuda.current_device()):
        return x
    if not isinstance(x, torch.Tensor):
        x = torch.as_tensor(x)
    if x.dtype != dtype:
        x = x.view(dtype) if x.element_size() == torch.empty((), dtype=dtype).element_size() \
            else x.to(dtype)
    return x.to(device).contiguous()


class KVCache:
    """Device storage of the indexer keys and the block index (hisa_kv).
    pool="mean" or "max": how block representatives pool their keys."""

    def __init__(self, batch: int, cap: int, d: int, B: int, dtype: str = "bf16",
                 device="cuda", pool: str = "mean"):
        if pool not in ("mean", "max"):
            raise ValueError("pool must be 'mean' or 'max'")
        self.batch, self.cap, self.d, self.B = batch, cap, d, B
        self.dtype = dtype
        self.pool = pool
        self.device = torch.device(device)
        self.nblk = -(-cap // B)
        kdt = torch.bfloat16 if dtype == "bf16" else torch.uint8
        self.keys = torch.zeros((batch, cap, d), dtype=kdt, device=self.device)
        self.key_scale = (torch.ones((batch, cap), dtype=torch.float32, device=self.device)
                          if dtype == "e4m3" else None)
        self.pooled = torch.zeros((batch, self.nblk, d), dtype=torch.float32, device=self.device)
        self.pooled_hl = torch.zeros((batch, self.nblk, 2 * d), dtype=torch.bfloat16,
                                     device=self.device)
        self.len = torch.zeros(batch, dtype=torch.int32, device=self.device)
        self.status = torch.zeros(1, dtype=torch.int32, device=self.device)
        self._struct = hisa_kv(
            keys=self.keys.data_ptr(),
            key_scale=self.key_scale.data_ptr() if self.key_scale is not None else None,
            pooled=self.pooled.data_ptr(), pooled_hl=self.pooled_hl.data_ptr(),
            len=self.len.data_ptr(), status=self.status.data_ptr(), batch=batch, cap=cap, d=d,
            B=B, dtype=HISA_KEY_BF16 if dtype == "bf16" else HISA_KEY_E4M3,
            pool=HISA_POOL_MAX if pool == "max" else HISA_POOL_MEAN)

    @property
    def struct(self):
        return ctypes.byref(self._struct)

    def load(self, keys, lens, key_scale=None):
        """Copy keys [batch, <=cap, d] (bf16 bits / e4m3 codes), lens and scales in."""
        kdt = torch.bfloat16 if self.dtype == "bf16" else torch.uint8
        k = _dev(keys, kdt, self.device)
        self.keys[:, :k.shape[1]].copy_(k)
        self.len.copy_(_dev(lens, torch.int32, self.device))
        if self.dtype == "e4m3":
            sc = _dev(key_scale, torch.float32, self.device)
            self.key_scale[:, :sc.shape[1]].copy_(sc)
        return self

    @classmethod
    def from_case(cls, case, device="cuda", pool: str = "mean", B: Optional[int] = None):
        """A cache holding a seeded case's keys (block size B overrides the case's)."""
        kv = cls(case.batch, case.cap, case.d, B or case.B, case.dtype, device, pool)
        return kv.load(torch.from_numpy(case.keys), torch.from_numpy(case.lens),
                       None if case.key_scale is None else torch.from_numpy(case.key_scale))

    @classmethod
    def shard_of_case(cls, case, tok_off: int, cap: int, device="cuda", pool: str = "mean",
                      B: Optional[int] = None):
        """The context-parallel shard of a seeded case that holds global
        positions [tok_off, tok_off + cap) of every sequence."""
        kv = cls(case.batch, cap, case.d, B or case.B, case.dtype, device, pool)
        keys = torch.from_numpy(case.keys[:, tok_off:tok_off + cap])
        lens = torch.from_numpy(case.lens.astype("int64").clip(tok_off, tok_off + cap) - tok_off)
        sc = None if case.key_scale is None else torch.from_numpy(case.key_scale[:, tok_off:tok_off + cap])
        return kv.load(keys, lens.to(torch.int32), sc)

    def status_bits(self) -> int:
        return int(self.status.item()) & 0xFFFFFFFF

    def clear_status(self):
        self.status.zero_()


def hisa_pool_blocks(kv: KVCache, stream=None):
    _check("hisa_pool_blocks", _lib.hisa_pool_blocks(kv.struct, _stream(stream)))


def hisa_append(kv: KVCache, tok: torch.Tensor, tok_scale: Optional[torch.Tensor] = None,
                stream=None):
    _check("hisa_append", _lib.hisa_append(kv.struct, _ptr(tok), _ptr(tok_scale), _stream(stream)))


def _queries(kv, Q, w, q_seq, q_pos):
    dev = kv.keys.device
    Q = _dev(Q, torch.bfloat16, dev)
    w = _dev(w, torch.float32, dev)
    q_seq = _dev(q_seq, torch.int32, dev)
    q_pos = None if q_pos is None else _dev(q_pos, torch.int32, dev)
    return Q, w, q_seq, q_pos


def _check_ws(fn: str, kv, ws: Optional[torch.Tensor]):
    """A caller's workspace: its byte size is passed as numel(), so it must be
    a contiguous byte tensor on the cache's device."""
    if ws is not None and (ws.dtype != torch.uint8 or not ws.is_contiguous()
                           or ws.device != kv.keys.device):
        raise ValueError(f"{fn}: ws must be a contiguous uint8 tensor on {kv.keys.device}")


def hisa_select_workspace_bytes(kv: KVCache, n_q: int, H: int, m: int, k: int) -> int:
    return int(_lib.hisa_select_workspace_bytes(kv.struct, n_q, H, m, k))


def dsa_flat_workspace_bytes(kv: KVCache, n_q: int, H: int, k: int) -> int:
    return int(_lib.dsa_flat_workspace_bytes(kv.struct, n_q, H, k))


def workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """A caller-owned workspace buffer (256-byte aligned by the allocator)."""
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def hisa_select(kv: KVCache, Q, w, q_seq, q_pos, m: int, k: int, want_scores: bool = False,
                ws: Optional[torch.Tensor] = None, idx: Optional[torch.Tensor] = None,
                scores: Optional[torch.Tensor] = None, stream=None):
    """Two-stage HISA selection.  Returns idx [n_q, k] (and scores if asked)."""
    Q, w, q_seq, q_pos = _queries(kv, Q, w, q_seq, q_pos)
    n_q, H = Q.shape[0], Q.shape[1]
    if ws is None:
        ws = workspace(hisa_select_workspace_bytes(kv, n_q, H, m, k), kv.device)
    _check_out("hisa_select", kv, n_q, k, idx, scores)
    _check_ws("hisa_select", kv, ws)
    idx = torch.empty((n_q, k), dtype=torch.int32, device=kv.device) if idx is None else idx
    if want_scores and scores is None:
        scores = torch.empty((n_q, k), dtype=torch.float32, device=kv.device)
    _check("hisa_select", _lib.hisa_select(
        kv.struct, _ptr(Q), _ptr(w), _ptr(q_seq), _ptr(q_pos), n_q, H, m, k, _ptr(idx),
        _ptr(scores), _ptr(ws), ws.numel(), _stream(stream)))
    return (idx, scores) if want_scores else idx


def hisa_decode_step_workspace_bytes(kv: KVCache, H: int, m: int, k: int) -> int:
    return int(_lib.hisa_decode_step_workspace_bytes(kv.struct, H, m, k))


def hisa_decode_step(kv: KVCache, tok: torch.Tensor, Q, w, m: int, k: int,
                     tok_scale: Optional[torch.Tensor] = None, want_scores: bool = False,
                     ws: Optional[torch.Tensor] = None, idx: Optional[torch.Tensor] = None,
                     scores: Optional[torch.Tensor] = None, stream=None):
    """hisa_append(kv, tok) then hisa_select for every sequence's new last
    position (query row b = sequence b), in one call.  Returns idx [batch, k]
    (and scores if asked)."""
    fn = "hisa_decode_step"
    dev = kv.keys.device
    Q = _dev(Q, torch.bfloat16, dev)
    w = _dev(w, torch.float32, dev)
    n_q, H = kv.batch, Q.shape[1]
    if Q.dim() != 3 or Q.shape[0] != n_q or Q.shape[2] != kv.d or tuple(w.shape) != (n_q, H):
        raise ValueError(f"{fn}: Q must be [{n_q}, H, {kv.d}] and w [{n_q}, H]")
    tdt = torch.bfloat16 if kv.dtype == "bf16" else torch.uint8
    if tok.dtype not in (tdt, torch.int16) or not tok.is_contiguous() or tok.device != dev or \
            tok.numel() != n_q * kv.d:
        raise ValueError(f"{fn}: tok must be a contiguous [{n_q}, {kv.d}] {tdt} tensor on {dev}")
    if kv.dtype == "e4m3" and (tok_scale is None or tok_scale.dtype != torch.float32 or
                               tok_scale.numel() != n_q or tok_scale.device != dev):
        raise ValueError(f"{fn}: tok_scale must be fp32 [{n_q}] on {dev}")
    _check_out(fn, kv, n_q, k, idx, scores)
    _check_ws(fn, kv, ws)
    if ws is None:
        ws = workspace(hisa_decode_step_workspace_bytes(kv, H, m, k), dev)
    idx = torch.empty((n_q, k), dtype=torch.int32, device=dev) if idx is None else idx
    if want_scores and scores is None:
        scores = torch.empty((n_q, k), dtype=torch.float32, device=dev)
    _check(fn, _lib.hisa_decode_step(
        kv.struct, _ptr(tok), _ptr(tok_scale), _ptr(Q), _ptr(w), H, m, k, _ptr(idx), _ptr(scores),
        _ptr(ws), ws.numel(), _stream(stream)))
    return (idx, scores) if want_scores else idx


def hisa_select_inspect(kv: KVCache, Q, w, q_seq, q_pos, m: int, k: int, stream=None):
    """hisa_select plus kept blocks, their count and the per-row work counters."""
    Q, w, q_seq, q_pos = _queries(kv, Q, w, q_seq, q_pos)
    n_q, H = Q.shape[0], Q.shape[1]
    mm = min(m, kv.nblk)
    ws = workspace(hisa_select_workspace_bytes(kv, n_q, H, m, k), kv.device)
    idx = torch.empty((n_q, k), dtype=torch.int32, device=kv.device)
    scores = torch.empty((n_q, k), dtype=torch.float32, device=kv.device)
    blocks = torch.empty((n_q, mm), dtype=torch.int32, device=kv.device)
    nblocks = torch.empty(n_q, dtype=torch.int32, device=kv.device)
    counts = torch.empty((n_q, 2), dtype=torch.int64, device=kv.device)
    _check("hisa_select_inspect", _lib.hisa_select_inspect(
        kv.struct, _ptr(Q), _ptr(w), _ptr(q_seq), _ptr(q_pos), n_q, H, m, k, _ptr(idx),
        _ptr(scores), _ptr(blocks), _ptr(nblocks), _ptr(counts), _ptr(ws), ws.numel(),
        _stream(stream)))
    return dict(idx=idx, scores=scores, blocks=blocks, nblocks=nblocks, counts=counts)


def _same_device(t: torch.Tensor, kv: KVCache) -> bool:
    return t.device == kv.keys.device


def _check_out(fn: str, kv: KVCache, n_q: int, k: int, idx: Optional[torch.Tensor],
               scores: Optional[torch.Tensor]):
    """Caller-owned outputs: the library writes n_q * k entries to each, so a
    short or misplaced buffer must be refused here, before any launch."""
    for name, t, dt in (("idx", idx, torch.int32), ("scores", scores, torch.float32)):
        if t is None:
            continue
        if t.dtype != dt or not t.is_contiguous() or not _same_device(t, kv):
            raise ValueError(f"{fn}: {name} must be a contiguous {dt} tensor on {kv.keys.device}")
        if t.numel() < n_q * k:
            raise ValueError(f"{fn}: {name} holds {t.numel()} entries, needs n_q * k = {n_q * k}")


def hisa_select_static(kv: KVCache, Q: torch.Tensor, w: torch.Tensor, q_seq: torch.Tensor,
                       q_pos: Optional[torch.Tensor], m: int, k: int, idx: torch.Tensor,
                       scores: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """hisa_select with the library's fixed scratch array instead of a workspace.

    Every tensor must already be on the cache's device with its final dtype and
    layout (Q bf16 [n_q, H, d], w fp32 [n_q, H], q_seq / q_pos int32 [n_q], idx
    int32 and scores fp32 (or None) of at least n_q * k entries): this wrapper
    converts and allocates nothing, and neither does the library call.  It is
    also the only guard of those shapes, since the C call cannot see tensor
    sizes: anything else raises ValueError before the call.  Calls on one
    device share the scratch, so they must be ordered on one stream."""
    fn = "hisa_select_static"
    for name, t, dt in (("Q", Q, torch.bfloat16), ("w", w, torch.float32), ("q_seq", q_seq, torch.int32),
                        ("q_pos", q_pos, torch.int32)):
        if t is not None and (t.dtype != dt or not t.is_contiguous() or not _same_device(t, kv)):
            raise ValueError(f"{fn}: {name} must be a contiguous {dt} tensor on {kv.keys.device}")
    if Q.dim() != 3 or Q.shape[2] != kv.d:
        raise ValueError(f"{fn}: Q must be [n_q, H, {kv.d}], got {tuple(Q.shape)}")
    n_q, H = Q.shape[0], Q.shape[1]
    if tuple(w.shape) != (n_q, H):
        raise ValueError(f"{fn}: w must be [{n_q}, {H}], got {tuple(w.shape)}")
    for name, t in (("q_seq", q_seq), ("q_pos", q_pos)):
        if t is not None and t.numel() != n_q:
            raise ValueError(f"{fn}: {name} must hold n_q = {n_q} entries, got {t.numel()}")
    if idx is None:
        raise ValueError(f"{fn}: idx is required (the call allocates nothing)")
    _check_out(fn, kv, n_q, k, idx, scores)
    _check(fn, _lib.hisa_select_static(
        kv.struct, _ptr(Q), _ptr(w), _ptr(q_seq), _ptr(q_pos), n_q, H, m, k, _ptr(idx),
        _ptr(scores), _stream(stream)))
    return idx


def superblock_index(kv: KVCache, bf: int) -> KVCache:
    """A second index over kv's keys with superblocks of bf blocks (for
    hisa_tree_select); shares kv's keys, scales and lengths."""
    kv2 = KVCache.__new__(KVCache)
    kv2.batch, kv2.cap, kv2.d, kv2.B = kv.batch, kv.cap, kv.d, kv.B * bf
    kv2.dtype, kv2.device, kv2.pool = kv.dtype, kv.device, kv.pool
    kv2.nblk = -(-kv.cap // kv2.B)
    kv2.keys, kv2.key_scale, kv2.len, kv2.status = kv.keys, kv.key_scale, kv.len, kv.status
    kv2.pooled = torch.zeros((kv.batch, kv2.nblk, kv.d), dtype=torch.float32, device=kv.device)
    kv2.pooled_hl = torch.zeros((kv.batch, kv2.nblk, 2 * kv.d), dtype=torch.bfloat16, device=kv.device)
    kv2._struct = hisa_kv(keys=kv._struct.keys, key_scale=kv._struct.key_scale,
                          pooled=kv2.pooled.data_ptr(), pooled_hl=kv2.pooled_hl.data_ptr(),
                          len=kv._struct.len, status=kv._struct.status, batch=kv.batch, cap=kv.cap,
                          d=kv.d, B=kv2.B, dtype=kv._struct.dtype, pool=kv._struct.pool)
    return kv2


def hisa_pool_tail(kv: KVCache, stream=None):
    _check("hisa_pool_tail", _lib.hisa_pool_tail(kv.struct, _stream(stream)))


def hisa_tree_workspace_bytes(kv: KVCache, kv2: KVCache, n_q: int, H: int, W: int, m: int,
                              k: int) -> int:
    return int(_lib.hisa_tree_workspace_bytes(kv.struct, kv2.struct, n_q, H, W, m, k))


def hisa_tree_select(kv: KVCache, kv2: KVCache, Q, w, q_seq, q_pos, W: int, m: int, k: int,
                     inspect: bool = False, ws: Optional[torch.Tensor] = None,
                     idx: Optional[torch.Tensor] = None, stream=None):
    """Three-level search (superblocks of kv2, blocks of kv, tokens).  Returns
    idx [n_q, k], or with inspect=True a dict with scores, kept superblocks and
    blocks and the per-row work counters."""
    Q, w, q_seq, q_pos = _queries(kv, Q, w, q_seq, q_pos)
    n_q, H = Q.shape[0], Q.shape[1]
    dev = kv.keys.device
    _check_out("hisa_tree_select", kv, n_q, k, idx, None)
    _check_ws("hisa_tree_select", kv, ws)
    ws = workspace(hisa_tree_workspace_bytes(kv, kv2, n_q, H, W, m, k), dev) if ws is None else ws
    idx = torch.empty((n_q, k), dtype=torch.int32, device=dev) if idx is None else idx
    out = {}
    if inspect:
        out = dict(scores=torch.empty((n_q, k), dtype=torch.float32, device=dev),
                   sblocks=torch.empty((n_q, min(W, kv2.nblk)), dtype=torch.int32, device=dev),
                   nsblocks=torch.empty(n_q, dtype=torch.int32, device=dev),
                   blocks=torch.empty((n_q, min(m, kv.nblk)), dtype=torch.int32, device=dev),
                   nblocks=torch.empty(n_q, dtype=torch.int32, device=dev),
                   counts=torch.empty((n_q, 3), dtype=torch.int64, device=dev))
    g = lambda name: _ptr(out.get(name))
    _check("hisa_tree_select", _lib.hisa_tree_select(
        kv.struct, kv2.struct, _ptr(Q), _ptr(w), _ptr(q_seq), _ptr(q_pos), n_q, H, W, m, k,
        _ptr(idx), g("scores"), g("sblocks"), g("nsblocks"), g("blocks"), g("nblocks"),
        g("counts"), _ptr(ws), ws.numel(), _stream(stream)))
    if inspect:
        out["idx"] = idx
        return out
    return idx


def _levels_args(kvs, keep):
    """Host arrays of the level indexes and kept counts (kept alive by the caller)."""
    n = len(kvs)
    if n != len(keep):
        raise ValueError("hisa_levels_select: one keep count per level")
    arr = (_KVP * n)(*[ctypes.pointer(kv._struct) for kv in kvs])
    kp = (ctypes.c_int * n)(*[int(x) for x in keep])
    return n, arr, kp


def hisa_levels_workspace_bytes(kvs, keep, n_q: int, H: int, k: int) -> int:
    n, arr, kp = _levels_args(kvs, keep)
    return int(_lib.hisa_levels_workspace_bytes(ctypes.cast(arr, _P), n, ctypes.cast(kp, _P), n_q, H, k))


def hisa_levels_select(kvs, Q, w, q_seq, q_pos, keep, k: int, inspect: bool = False,
                       ws: Optional[torch.Tensor] = None, idx: Optional[torch.Tensor] = None,
                       stream=None):
    """Search of any depth.  kvs: indexes over the same keys, finest first
    (kvs[0] the block index, each unit size a multiple of the one below, the
    coarser ones made by superblock_index); keep[l]: units kept at level l.
    Returns idx [n_q, k], or with inspect=True a dict with scores, the kept
    units of every level (kept[l], nkept[l]) and the per-row work counters."""
    kv = kvs[0]
    Q, w, q_seq, q_pos = _queries(kv, Q, w, q_seq, q_pos)
    n_q, H = Q.shape[0], Q.shape[1]
    dev = kv.keys.device
    _check_out("hisa_levels_select", kv, n_q, k, idx, None)
    _check_ws("hisa_levels_select", kv, ws)
    n, arr, kp = _levels_args(kvs, keep)
    ws = workspace(hisa_levels_workspace_bytes(kvs, keep, n_q, H, k), dev) if ws is None else ws
    idx = torch.empty((n_q, k), dtype=torch.int32, device=dev) if idx is None else idx
    scores = kept = nkept = counts = None
    kept_p = nkept_p = None
    if inspect:
        scores = torch.empty((n_q, k), dtype=torch.float32, device=dev)
        kept = [torch.empty((n_q, min(int(keep[l]), kvs[l].nblk)), dtype=torch.int32, device=dev)
                for l in range(n)]
        nkept = [torch.empty(n_q, dtype=torch.int32, device=dev) for _ in range(n)]
        counts = torch.empty((n_q, n + 1), dtype=torch.int64, device=dev)
        kept_p = (_P * n)(*[t.data_ptr() for t in kept])
        nkept_p = (_P * n)(*[t.data_ptr() for t in nkept])
    _check("hisa_levels_select", _lib.hisa_levels_select(
        ctypes.cast(arr, _P), n, ctypes.cast(kp, _P), _ptr(Q), _ptr(w), _ptr(q_seq), _ptr(q_pos), n_q,
        H, k, _ptr(idx), _ptr(scores), ctypes.cast(kept_p, _P) if kept_p else None,
        ctypes.cast(nkept_p, _P) if nkept_p else None, _ptr(counts), _ptr(ws), ws.numel(),
        _stream(stream)))
    if inspect:
        return dict(idx=idx, scores=scores, kept=kept, nkept=nkept, counts=counts)
    return idx


def dsa_flat_select(kv: KVCache, Q, w, q_seq, q_pos, k: int, want_scores: bool = False,
                    ws: Optional[torch.Tensor] = None, idx: Optional[torch.Tensor] = None,
                    scores: Optional[torch.Tensor] = None, stream=None):
    """Flat indexer scan over every visible key.  Returns idx [n_q, k] (and scores)."""
    Q, w, q_seq, q_pos = _queries(kv, Q, w, q_seq, q_pos)
    n_q, H = Q.shape[0], Q.shape[1]
    need = dsa_flat_workspace_bytes(kv, n_q, H, k)
    ws = workspace(need, kv.device) if ws is None else ws
    _check_out("dsa_flat_select", kv, n_q, k, idx, scores)
    _check_ws("dsa_flat_select", kv, ws)
    idx = torch.empty((n_q, k), dtype=torch.int32, device=kv.device) if idx is None else idx
    if want_scores and scores is None:
        scores = torch.empty((n_q, k), dtype=torch.float32, device=kv.device)
    _check("dsa_flat_select", _lib.dsa_flat_select(
        kv.struct, _ptr(Q), _ptr(w), _ptr(q_seq), _ptr(q_pos), n_q, H, k, _ptr(idx),
        _ptr(scores), _ptr(ws), ws.numel(), _stream(stream)))
    return (idx, scores) if want_scores else idx


def hisa_topk_f32(x: torch.Tensor, k: int, stream=None) -> torch.Tensor:
    """Top-k selection rule on fp32 rows (ties: lower index; ascending output, -1 pad)."""
    x = x.to(torch.float32).contiguous()
    rows, n = x.shape
    idx = torch.empty((rows, k), dtype=torch.int32, device=x.device)
    _check("hisa_topk_f32", _lib.hisa_topk_f32(_ptr(x), rows, n, k, _ptr(idx), _stream(stream)))
    return idx


def hisa_cp_workspace_bytes(kv: KVCache, tok_off: int, n_q: int, H: int, m: int, k: int) -> int:
    return int(_lib.hisa_cp_workspace_bytes(kv.struct, tok_off, n_q, H, m, k))


def hisa_cp_blocks(kv: KVCache, tok_off: int, Q, w, q_seq, q_pos, m: int,
                   ws: Optional[torch.Tensor] = None, stream=None):
    """One shard's block candidates: (ids [n_q, m] global block ids, scores
    [n_q, m]); the own block, on the shard holding the query, scores +inf."""
    Q, w, q_seq, q_pos = _queries(kv, Q, w, q_seq, q_pos)
    n_q, H = Q.shape[0], Q.shape[1]
    _check_ws("hisa_cp_blocks", kv, ws)
    ws = workspace(hisa_cp_workspace_bytes(kv, tok_off, n_q, H, m, 1), kv.device) if ws is None else ws
    ids = torch.empty((n_q, m), dtype=torch.int32, device=kv.device)
    sc = torch.empty((n_q, m), dtype=torch.float32, device=kv.device)
    _check("hisa_cp_blocks", _lib.hisa_cp_blocks(
        kv.struct, tok_off, _ptr(Q), _ptr(w), _ptr(q_seq), _ptr(q_pos), n_q, H, m, _ptr(ids), _ptr(sc),
        _ptr(ws), ws.numel(), _stream(stream)))
    return ids, sc


def hisa_cp_tokens(kv: KVCache, tok_off: int, Q, w, q_seq, q_pos, m: int, k: int, kept: torch.Tensor,
                   ws: Optional[torch.Tensor] = None, stream=None):
    """One shard's token candidates under the merged kept blocks kept [n_q, m]:
    (idx [n_q, k] global token indices, scores [n_q, k])."""
    Q, w, q_seq, q_pos = _queries(kv, Q, w, q_seq, q_pos)
    n_q, H = Q.shape[0], Q.shape[1]
    _check_ws("hisa_cp_tokens", kv, ws)
    ws = workspace(hisa_cp_workspace_bytes(kv, tok_off, n_q, H, m, k), kv.device) if ws is None else ws
    kept = _dev(kept, torch.int32, kv.device)
    idx = torch.empty((n_q, k), dtype=torch.int32, device=kv.device)
    sc = torch.empty((n_q, k), dtype=torch.float32, device=kv.device)
    _check("hisa_cp_tokens", _lib.hisa_cp_tokens(
        kv.struct, tok_off, _ptr(Q), _ptr(w), _ptr(q_seq), _ptr(q_pos), n_q, H, m, k, _ptr(kept),
        _ptr(idx), _ptr(sc), _ptr(ws), ws.numel(), _stream(stream)))
    return idx, sc


def hisa_merge_topk(ids: torch.Tensor, scores: torch.Tensor, k: int, stream=None):
    """Top-k of the (id, score) lists ids / scores [lists, rows, n] per row,
    by (score desc, id asc): (idx [rows, k], scores [rows, k])."""
    ids = ids.to(torch.int32).contiguous()
    scores = scores.to(torch.float32).contiguous()
    lists, rows, n = ids.shape
    idx = torch.empty((rows, k), dtype=torch.int32, device=ids.device)
    sc = torch.empty((rows, k), dtype=torch.float32, device=ids.device)
    _check("hisa_merge_topk", _lib.hisa_merge_topk(_ptr(ids), _ptr(scores), lists, rows, n, k, _ptr(idx),
                                                   _ptr(sc), _stream(stream)))
    return idx, sc


def hisa_sparse_attn_workspace_bytes(n_q: int, k: int) -> int:
    return int(_lib.hisa_sparse_attn_workspace_bytes(n_q, k))


def hisa_sparse_attn(Qa: torch.Tensor, K: torch.Tensor, V: torch.Tensor, lens: torch.Tensor,
                     q_seq: torch.Tensor, idx: torch.Tensor, scale: Optional[float] = None,
                     ws: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                     lse: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None,
                     stream=None):
    """Attention of each query row over its selected tokens: Qa [n_q, Ha, 128]
    bf16 heads sharing the key and value heads K, V [batch, cap, 128] bf16;
    idx [n_q, k] (hisa_select's output).  Returns (out [n_q, Ha, 128] fp32,
    lse [n_q, Ha] fp32); `status` (int32 [1], device) collects device errors."""
    n_q, Ha, d = Qa.shape
    batch, cap, _ = K.shape
    k = idx.shape[1]
    dev = Qa.device
    scale = (1.0 / d ** 0.5) if scale is None else float(scale)
    ws = workspace(hisa_sparse_attn_workspace_bytes(n_q, k), dev) if ws is None else ws
    out = torch.empty((n_q, Ha, d), dtype=torch.float32, device=dev) if out is None else out
    lse = torch.empty((n_q, Ha), dtype=torch.float32, device=dev) if lse is None else lse
    status = torch.zeros(1, dtype=torch.int32, device=dev) if status is None else status
    _check("hisa_sparse_attn", _lib.hisa_sparse_attn(
        _ptr(Qa), Ha, _ptr(K), _ptr(V), _ptr(lens), batch, cap, d, _ptr(q_seq), _ptr(idx), n_q, k,
        scale, _ptr(out), _ptr(lse), _ptr(status), _ptr(ws), ws.numel(), _stream(stream)))
    return out, lse


def _gather_ranks(t: torch.Tensor, group=None) -> torch.Tensor:
    """[world, *t.shape]: every rank's t in rank order."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    if dist.get_backend(group) == "nccl":
        out = torch.empty((world,) + tuple(t.shape), dtype=t.dtype, device=t.device)
        dist.all_gather_into_tensor(out, t.contiguous(), group=group)
        return out
    parts = [torch.empty_like(t) for _ in range(world)]
    dist.all_gather(parts, t.contiguous(), group=group)
    return torch.stack(parts)


def hisa_cp_select(kv: KVCache, tok_off: int, Q, w, q_seq, q_pos, m: int, k: int, group=None,
                   ws: Optional[torch.Tensor] = None):
    """Context-parallel hisa_select on the current stream: this rank holds the
    shard at tok_off, the ranks of `group` hold ascending shards in rank
    order.  Every rank passes the same query rows (Q, w, q_seq, global q_pos)
    and the same m and k.  Two all-gathers of (id, score) pairs; the result
    (idx, scores) equals hisa_select's on the whole sequence, on every rank."""
    ids, sc = hisa_cp_blocks(kv, tok_off, Q, w, q_seq, q_pos, m, ws=ws)
    kept, _ = hisa_merge_topk(_gather_ranks(ids, group), _gather_ranks(sc, group), m)
    tid, tsc = hisa_cp_tokens(kv, tok_off, Q, w, q_seq, q_pos, m, k, kept, ws=ws)
    return hisa_merge_topk(_gather_ranks(tid, group), _gather_ranks(tsc, group), k)


def hisa_selftest_wait(status: torch.Tensor, stream=None):
    """Launch one warp whose bounded wait must run out and set HISA_DEV_TIMEOUT
    in `status` (int32 [1], device)."""
    _check("hisa_selftest_wait", _lib.hisa_selftest_wait(_ptr(status), _stream(stream)))


def hisa_profile_enable(on: bool = True):
    """Record CUDA events around every kernel the library launches."""
    _check("hisa_profile_enable", _lib.hisa_profile_enable(1 if on else 0))


def hisa_profile_read(reset: bool = True) -> dict:
    """{phase: (milliseconds, launches)} accumulated since the last reset."""
    ms = (ctypes.c_float * len(PHASES))()
    n = (ctypes.c_int * len(PHASES))()
    _check("hisa_profile_read", _lib.hisa_profile_read(ms, n, 1 if reset else 0))
    return {name: (float(ms[i]), int(n[i])) for i, name in enumerate(PHASES)}
