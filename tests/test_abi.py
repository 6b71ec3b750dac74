"""The C-ABI library builds, loads and exports what include/hisa.h declares,
and its host-side argument checks reject bad calls before touching a GPU."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hisa.h")


def build_module():
    """The build script, loaded by path (importing the package needs the library)."""
    import importlib.util
    path = os.path.join(ROOT, "hierarchical_top_indexer_b200", "build.py")
    spec = importlib.util.spec_from_file_location("hisa_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.fixture(scope="module")
def hisa():
    build = build_module()
    if build.stale():
        build.build()
    import hierarchical_top_indexer_b200 as h
    return h


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(\w+)\s*\(", text, flags=re.M)
    return sorted(set(n for n in names if n.startswith(("hisa_", "dsa_"))))


def test_header_declares_the_boundary():
    names = declared_functions()
    for fn in ("hisa_pool_blocks", "hisa_append", "hisa_select", "dsa_flat_select"):
        assert fn in names


def test_library_exports_every_declared_symbol(hisa):
    lib = ctypes.CDLL(hisa.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in hisa.h but not exported"
    assert set(hisa.EXPORTS) <= set(declared_functions())


def test_library_has_no_link_time_dependency_on_the_driver(hisa):
    # The driver API is reached through cudaGetDriverEntryPoint, so the
    # library loads on machines without libcuda (like this one).
    import subprocess
    out = subprocess.run(["ldd", hisa.LIB_PATH], capture_output=True, text=True).stdout
    assert "libcuda.so" not in out


def test_status_strings(hisa):
    lib = hisa.lib()
    assert lib.hisa_status_string(0) == b"ok"
    assert lib.hisa_status_string(3).startswith(b"workspace")
    assert lib.hisa_status_string(99) == b"unknown status"


def _kv(hisa, **over):
    fields = dict(keys=16, key_scale=None, pooled=32, pooled_hl=48, len=64, status=128,
                  batch=1, cap=1024, d=128, B=128, dtype=0)
    fields.update(over)
    return hisa.hisa_kv(**fields)


def test_argument_checks_reject_before_any_launch(hisa):
    lib = hisa.lib()
    kv = _kv(hisa)
    P = ctypes.c_void_p
    good = dict(Q=P(16), w=P(16), q_seq=P(16), idx=P(16))
    # NULL cache, bad sizes, missing pointers, unsupported d / B / H
    assert lib.hisa_pool_blocks(None, None) == hisa.HISA_E_INVAL
    assert lib.hisa_pool_blocks(ctypes.byref(_kv(hisa, batch=0)), None) == hisa.HISA_E_INVAL
    assert lib.hisa_pool_blocks(ctypes.byref(_kv(hisa, d=96)), None) == hisa.HISA_E_UNSUPPORTED
    assert lib.hisa_pool_blocks(ctypes.byref(_kv(hisa, dtype=1)), None) == hisa.HISA_E_INVAL
    assert lib.hisa_pool_blocks(ctypes.byref(_kv(hisa, keys=8)), None) == hisa.HISA_E_INVAL
    assert lib.hisa_append(ctypes.byref(kv), None, None, None) == hisa.HISA_E_INVAL

    def sel(kvp, n_q=4, H=64, m=8, k=16, ws=P(256), ws_bytes=1 << 30, **kw):
        a = dict(good)
        a.update(kw)
        return lib.hisa_select(kvp, a["Q"], a["w"], a["q_seq"], None, n_q, H, m, k, a["idx"],
                               None, ws, ws_bytes, None)

    assert sel(ctypes.byref(kv), k=0) == hisa.HISA_E_INVAL
    assert sel(ctypes.byref(kv), m=0) == hisa.HISA_E_INVAL
    assert sel(ctypes.byref(kv), H=129) == hisa.HISA_E_UNSUPPORTED
    assert sel(ctypes.byref(kv), H=0) == hisa.HISA_E_UNSUPPORTED
    assert sel(ctypes.byref(kv), n_q=-1) == hisa.HISA_E_INVAL
    assert sel(ctypes.byref(_kv(hisa, B=100))) == hisa.HISA_E_UNSUPPORTED
    assert sel(ctypes.byref(kv), Q=None) == hisa.HISA_E_INVAL
    assert sel(ctypes.byref(kv), Q=P(8)) == hisa.HISA_E_INVAL          # misaligned
    assert sel(ctypes.byref(kv), ws=None) == hisa.HISA_E_WORKSPACE
    assert sel(ctypes.byref(kv), ws=P(128)) == hisa.HISA_E_WORKSPACE   # not 256-aligned
    assert sel(ctypes.byref(kv), ws_bytes=16) == hisa.HISA_E_WORKSPACE
    assert sel(ctypes.byref(kv), n_q=0) == hisa.HISA_OK                # nothing to do
    assert lib.dsa_flat_select(ctypes.byref(kv), P(16), P(16), P(16), None, 4, 64, 0, P(16),
                               None, P(256), 1 << 30, None) == hisa.HISA_E_INVAL
    assert lib.hisa_topk_f32(None, 3, 10, 2, None, None) == hisa.HISA_E_INVAL
    assert lib.hisa_topk_f32(P(16), 0, 10, 2, P(16), None) == hisa.HISA_OK


def test_workspace_sizes(hisa):
    lib = hisa.lib()
    kv = _kv(hisa, cap=32768, B=128)
    ws = lib.hisa_select_workspace_bytes(ctypes.byref(kv), 64, 64, 64, 2048)
    # block keys 64x256x4 + blocks 64x64x4 + counts 64x4 + plan 64x16 + token keys 64x8192x4
    assert ws == 65536 + 16384 + 256 + 1024 + 2097152
    assert lib.dsa_flat_workspace_bytes(ctypes.byref(kv), 64, 64, 2048) == 64 * 32768 * 4
    assert lib.hisa_select_workspace_bytes(None, 1, 1, 1, 1) == 0


def test_static_scratch_entry_checks_before_setup(hisa):
    """hisa_select_static validates its arguments and its scratch limit on the
    host: bad calls return an error code without any CUDA call (none is
    possible on this machine)."""
    lib = hisa.lib()
    P = ctypes.c_void_p
    kv = _kv(hisa, cap=32768, B=128)

    def sel(n_q=64, m=64, k=2048, Q=P(16)):
        return lib.hisa_select_static(ctypes.byref(kv), Q, P(16), P(16), None, n_q, 64, m, k,
                                      P(16), None, None)

    assert sel(Q=None) == hisa.HISA_E_INVAL
    assert sel(m=0) == hisa.HISA_E_INVAL
    assert sel(k=0) == hisa.HISA_E_INVAL
    assert lib.hisa_select_static(None, P(16), P(16), P(16), None, 1, 64, 8, 16, P(16), None,
                                  None) == hisa.HISA_E_INVAL
    # 256 rows over 32K keys with B = 128, m = 64 need 8.65 MB > 8 MiB
    assert lib.hisa_select_workspace_bytes(ctypes.byref(kv), 256, 64, 64, 2048) > \
        hisa.HISA_STATIC_SCRATCH_BYTES
    assert sel(n_q=256) == hisa.HISA_E_SCRATCH_LIMIT
    assert lib.hisa_status_string(hisa.HISA_E_SCRATCH_LIMIT).startswith(b"call needs more")


def test_pool_mode_is_checked(hisa):
    lib = hisa.lib()
    assert lib.hisa_pool_blocks(ctypes.byref(_kv(hisa, pool=2)), None) == hisa.HISA_E_INVAL
    assert lib.hisa_pool_blocks(ctypes.byref(_kv(hisa, pool=-1)), None) == hisa.HISA_E_INVAL


def test_tree_index_must_share_the_keys(hisa):
    lib = hisa.lib()
    P = ctypes.c_void_p
    kv = _kv(hisa, cap=4096, B=128)
    good2 = _kv(hisa, cap=4096, B=512, pooled=64, pooled_hl=80)
    assert lib.hisa_tree_workspace_bytes(ctypes.byref(kv), ctypes.byref(good2), 4, 64, 2, 4, 64) > 0
    bad_b = _kv(hisa, cap=4096, B=200, pooled=64, pooled_hl=80)          # not a multiple of 128
    bad_keys = _kv(hisa, cap=4096, B=512, keys=32, pooled=64, pooled_hl=80)
    for bad in (bad_b, bad_keys):
        assert lib.hisa_tree_workspace_bytes(ctypes.byref(kv), ctypes.byref(bad), 4, 64, 2, 4, 64) == 0
        assert lib.hisa_tree_select(ctypes.byref(kv), ctypes.byref(bad), P(16), P(16), P(16), None,
                                    4, 64, 2, 4, 64, P(16), None, None, None, None, None, None,
                                    P(256), 1 << 30, None) == hisa.HISA_E_INVAL


def test_context_parallel_shard_checks(hisa):
    lib = hisa.lib()
    P = ctypes.c_void_p
    kv = _kv(hisa, cap=4096, B=128)
    assert lib.hisa_cp_workspace_bytes(ctypes.byref(kv), 8192, 4, 64, 8, 64) > 0
    # shard offsets and capacities on block boundaries only
    assert lib.hisa_cp_workspace_bytes(ctypes.byref(kv), 100, 4, 64, 8, 64) == 0
    assert lib.hisa_cp_workspace_bytes(ctypes.byref(kv), -128, 4, 64, 8, 64) == 0
    odd = _kv(hisa, cap=4000, B=128)
    assert lib.hisa_cp_workspace_bytes(ctypes.byref(odd), 0, 4, 64, 8, 64) == 0
    args = (P(16), P(16), P(16))
    # global query positions are required
    assert lib.hisa_cp_blocks(ctypes.byref(kv), 0, *args, None, 4, 64, 8, P(16), P(16), P(256), 1 << 30,
                              None) == hisa.HISA_E_INVAL
    assert lib.hisa_cp_blocks(ctypes.byref(kv), 100, *args, P(16), 4, 64, 8, P(16), P(16), P(256),
                              1 << 30, None) == hisa.HISA_E_INVAL
    assert lib.hisa_cp_blocks(ctypes.byref(kv), 0, *args, P(16), 4, 64, 0, P(16), P(16), P(256), 1 << 30,
                              None) == hisa.HISA_E_INVAL
    assert lib.hisa_cp_blocks(ctypes.byref(kv), 0, *args, P(16), 4, 64, 8, P(16), P(16), P(256), 16,
                              None) == hisa.HISA_E_WORKSPACE
    assert lib.hisa_cp_tokens(ctypes.byref(kv), 0, *args, P(16), 4, 64, 8, 64, None, P(16), P(16),
                              P(256), 1 << 30, None) == hisa.HISA_E_INVAL
    assert lib.hisa_cp_blocks(ctypes.byref(kv), 0, *args, P(16), 0, 64, 8, P(16), P(16), None, 0,
                              None) == hisa.HISA_OK


def test_merge_checks(hisa):
    lib = hisa.lib()
    P = ctypes.c_void_p
    assert lib.hisa_merge_topk(P(16), P(16), 0, 4, 8, 4, P(16), None, None) == hisa.HISA_E_INVAL
    assert lib.hisa_merge_topk(P(16), P(16), 2, 4, 8, 0, P(16), None, None) == hisa.HISA_E_INVAL
    assert lib.hisa_merge_topk(None, P(16), 2, 4, 8, 4, P(16), None, None) == hisa.HISA_E_INVAL
    assert lib.hisa_merge_topk(P(16), P(16), 4, 4, 8192, 4, P(16), None, None) == hisa.HISA_E_UNSUPPORTED
    assert lib.hisa_merge_topk(P(16), P(16), 2, 0, 8, 4, P(16), None, None) == hisa.HISA_OK


def test_sparse_attention_checks(hisa):
    lib = hisa.lib()
    P = ctypes.c_void_p
    ok = dict(Qa=P(16), Ha=128, Kc=P(16), Vc=P(16), len=P(16), batch=2, cap=64, d=128, q_seq=P(16),
              idx=P(16), n_q=4, k=32, scale=0.1, out=P(16), lse=None, status=P(16), ws=P(256),
              ws_bytes=1 << 30, stream=None)

    def call(**kw):
        a = dict(ok)
        a.update(kw)
        return lib.hisa_sparse_attn(*a.values())
    assert lib.hisa_sparse_attn_workspace_bytes(4, 32) > 0
    assert lib.hisa_sparse_attn_workspace_bytes(4, 0) == 0
    assert call(d=64) == hisa.HISA_E_UNSUPPORTED
    assert call(Ha=129) == hisa.HISA_E_UNSUPPORTED
    assert call(scale=0.0) == hisa.HISA_E_INVAL
    assert call(scale=float("inf")) == hisa.HISA_E_INVAL
    assert call(k=0) == hisa.HISA_E_INVAL
    assert call(idx=None) == hisa.HISA_E_INVAL
    assert call(out=P(20)) == hisa.HISA_E_INVAL              # output rows need 16-byte alignment
    assert call(ws_bytes=16) == hisa.HISA_E_WORKSPACE
    assert call(n_q=0, Qa=None) == hisa.HISA_OK


def test_decode_step_checks_before_any_launch(hisa):
    """hisa_decode_step rejects bad arguments on the host (no CUDA call is
    possible on this machine, so reaching one would return HISA_E_CUDA)."""
    lib = hisa.lib()
    P = ctypes.c_void_p
    kv = _kv(hisa, cap=32768, B=128)

    def step(kvp=ctypes.byref(kv), tok=P(16), tok_scale=None, Q=P(16), w=P(16), H=64, m=64, k=2048,
             idx=P(16), scores=None, ws=P(256), ws_bytes=1 << 30):
        return lib.hisa_decode_step(kvp, tok, tok_scale, Q, w, H, m, k, idx, scores, ws, ws_bytes, None)

    assert step(kvp=None) == hisa.HISA_E_INVAL
    assert step(tok=None) == hisa.HISA_E_INVAL
    assert step(tok=P(8)) == hisa.HISA_E_INVAL                      # misaligned key rows
    assert step(kvp=ctypes.byref(_kv(hisa, cap=32768, dtype=1, key_scale=16))) == hisa.HISA_E_INVAL  # e4m3 without scales
    assert step(Q=None) == hisa.HISA_E_INVAL
    assert step(idx=None) == hisa.HISA_E_INVAL
    assert step(scores=P(2)) == hisa.HISA_E_INVAL
    assert step(m=0) == hisa.HISA_E_INVAL
    assert step(k=0) == hisa.HISA_E_INVAL
    assert step(H=0) == hisa.HISA_E_UNSUPPORTED
    assert step(kvp=ctypes.byref(_kv(hisa, B=100))) == hisa.HISA_E_UNSUPPORTED
    assert step(ws=None) == hisa.HISA_E_WORKSPACE
    assert step(ws_bytes=16) == hisa.HISA_E_WORKSPACE
    need = lib.hisa_decode_step_workspace_bytes(ctypes.byref(kv), 64, 64, 2048)
    assert need == lib.hisa_select_workspace_bytes(ctypes.byref(kv), kv.batch, 64, 64, 2048) > 0


def test_levels_entry_checks_and_workspace(hisa):
    """hisa_levels_select refuses malformed level lists on the host, and its
    workspace is hisa_select's for one level and hisa_tree_select's for two."""
    lib = hisa.lib()
    P = ctypes.c_void_p
    KVP = ctypes.POINTER(hisa.hisa_kv)
    base = dict(cap=32768, B=128)
    kv0 = _kv(hisa, **base)
    kv1 = _kv(hisa, **dict(base, B=1024))
    kv2 = _kv(hisa, **dict(base, B=8192))

    def arrays(kvs, keep):
        arr = (KVP * len(kvs))(*[ctypes.pointer(k) for k in kvs])
        return arr, (ctypes.c_int * len(keep))(*keep)

    def sel(kvs, keep, n=None, n_q=4, ws=P(256), ws_bytes=1 << 30):
        arr, kp = arrays(kvs, keep)
        return lib.hisa_levels_select(ctypes.cast(arr, P), len(kvs) if n is None else n,
                                      ctypes.cast(kp, P), P(16), P(16), P(16), None, n_q, 64, 16,
                                      P(16), None, None, None, None, ws, ws_bytes, None)

    def wsb(kvs, keep, n_q=64):
        arr, kp = arrays(kvs, keep)
        return lib.hisa_levels_workspace_bytes(ctypes.cast(arr, P), len(kvs), ctypes.cast(kp, P),
                                               n_q, 64, 2048)

    assert sel([kv0, kv1], [8, 4], n=0) == hisa.HISA_E_INVAL
    assert sel([kv0] * 9, [8] * 9) == hisa.HISA_E_INVAL                      # above HISA_MAX_LEVELS
    assert sel([kv0, kv1], [8, 0]) == hisa.HISA_E_INVAL                      # nothing kept
    assert sel([kv0, _kv(hisa, **dict(base, B=1000))], [8, 4]) == hisa.HISA_E_INVAL   # not a multiple
    assert sel([kv0, _kv(hisa, **dict(base, B=1024, keys=32))], [8, 4]) == hisa.HISA_E_INVAL
    assert sel([kv0, kv1, _kv(hisa, **dict(base, B=512))], [8, 4, 2]) == hisa.HISA_E_INVAL
    big = dict(cap=1 << 22, B=16)
    assert sel([_kv(hisa, **big), _kv(hisa, **dict(big, B=64))], [8, 4]) == hisa.HISA_E_UNSUPPORTED
    assert sel([kv0, kv1, kv2], [8, 4, 2], ws_bytes=16) == hisa.HISA_E_WORKSPACE
    assert sel([kv0, kv1, kv2], [8, 4, 2], n_q=0) == hisa.HISA_OK
    assert wsb([kv0], [64]) == lib.hisa_select_workspace_bytes(ctypes.byref(kv0), 64, 64, 64, 2048)
    assert wsb([kv0, kv1], [64, 8]) == lib.hisa_tree_workspace_bytes(
        ctypes.byref(kv0), ctypes.byref(kv1), 64, 64, 8, 64, 2048)
    assert wsb([kv0, kv1, kv2], [64, 8, 2]) > wsb([kv0, kv1], [64, 8])
    assert wsb([kv0, kv1], [64, 0]) == 0
