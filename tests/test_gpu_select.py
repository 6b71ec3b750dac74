"""GPU parity of the selection path: the top-k rule, the flat scan and the
two-stage HISA selection, on sizes the oracle finishes in seconds."""
import numpy as np
import pytest
import torch

import oracle
from hisa_inputs import make_case
from tests.gpu_util import check_flat, check_hisa, device_case, lib, queries, run_flat, run_hisa

pytestmark = pytest.mark.gpu


# ----------------------------------------------------------- selection rule


@pytest.mark.parametrize("n,k", [(1, 1), (7, 3), (100, 100), (100, 150), (5000, 128),
                                 (16384, 2048), (16385, 2048), (70000, 2048), (131072, 4096)])
def test_topk_f32_is_exact(n, k):
    """Both sides decide on the same fp32 values: the result must be identical."""
    h = lib()
    rng = np.random.default_rng(n + k)
    rows = 6
    x = rng.standard_normal((rows, n)).astype(np.float32)
    x[1] = np.round(x[1] * 4) / 4                       # heavy ties
    x[2] = 0.0                                          # all equal
    x[3, ::3] = -0.0
    x[4] = np.abs(x[4]) * -1e-30                        # tiny negatives, subnormals
    x[5, : n // 2] = np.inf if n > 1 else x[5, : n // 2]
    got = h.hisa_topk_f32(torch.from_numpy(x).cuda(), k).cpu().numpy()
    ref = oracle.topk_f32(x, k)
    assert np.array_equal(got, ref)


# ----------------------------------------------------------------- flat scan


@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
@pytest.mark.parametrize("d,H,B", [(128, 64, 128), (64, 4, 64), (128, 16, 32), (64, 128, 16)])
def test_flat_matches_oracle(dtype, d, H, B):
    case = make_case(batch=2, L=[3000, 1777], H=H, d=d, B=B, m=8, k=300, dtype=dtype, seed=d + H,
                     positions=[np.array([0, 5, 127, 128, 2999, 1500]), np.array([1776, 1000])])
    kv = device_case(case)
    gpu = run_flat(case, kv)
    _, swaps = check_flat(case, gpu)
    assert sum(swaps) <= 2


# ---------------------------------------------------------------------- HISA


@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
@pytest.mark.parametrize("d,H,B,m,k", [(128, 64, 128, 8, 512), (64, 4, 64, 8, 128),
                                       (128, 32, 32, 20, 300), (128, 48, 256, 3, 400),
                                       (64, 16, 16, 40, 200), (128, 64, 8, 64, 256),
                                       (128, 64, 128, 1, 64)])
def test_hisa_matches_oracle(dtype, d, H, B, m, k):
    case = make_case(batch=3, L=[4000, 2500, 700], H=H, d=d, B=B, m=m, k=k, dtype=dtype,
                     seed=11 + B + m,
                     positions=[np.array([0, 1, B - 1, B, 3999, 2048]), np.array([2499, 1234]),
                                np.array([699, 300])])
    kv = device_case(case)
    gpu = run_hisa(case, kv)
    _, swaps = check_hisa(case, gpu)
    assert sum(s for s, _ in swaps) <= 2
    assert kv.status_bits() == 0


def test_hisa_rows_longer_than_the_fused_block_selection():
    """More than 2048 blocks per row (more than the selection kernel stages in
    one CTA's shared memory, and more than the block scoring kernel keeps
    itself)."""
    case = make_case(batch=1, L=20000, H=16, d=64, B=8, m=40, k=200, dtype="bf16", seed=77,
                     positions=np.array([0, 7, 8, 12345, 19999]))
    kv = device_case(case)
    assert kv.nblk > 2048
    gpu = run_hisa(case, kv)
    _, swaps = check_hisa(case, gpu)
    assert sum(s for s, _ in swaps) <= 2
    assert kv.status_bits() == 0


def test_e4m3_caches_whose_scale_rows_are_not_16_byte_aligned():
    """cap % 4 != 0: the per-token scales of a tile do not start on a 16-byte
    boundary, so they are copied one by one instead of in bulk."""
    case = make_case(batch=3, L=[1001, 999, 517], H=64, d=128, B=64, m=6, k=200, dtype="e4m3",
                     seed=91, positions=[np.array([1000, 640, 0]), np.array([998, 63]),
                                         np.array([516, 64])])
    assert case.cap % 4 != 0
    kv = device_case(case)
    _, swaps = check_hisa(case, run_hisa(case, kv))
    assert sum(s for s, _ in swaps) <= 2
    _, fswaps = check_flat(case, run_flat(case, kv))
    assert sum(fswaps) <= 2
    assert kv.status_bits() == 0


@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
@pytest.mark.parametrize("d,H,B,m,k", [(128, 64, 128, 8, 512), (64, 16, 16, 40, 200)])
def test_hisa_max_pooling_matches_oracle(dtype, d, H, B, m, k):
    case = make_case(batch=2, L=[4000, 1500], H=H, d=d, B=B, m=m, k=k, dtype=dtype, seed=21 + B,
                     positions=[np.array([0, B, 3999, 2048]), np.array([1499, 700])])
    kv = device_case(case, pool="max")
    gpu = run_hisa(case, kv)
    _, swaps = check_hisa(case, gpu, pool="max")
    assert sum(s for s, _ in swaps) <= 2
    assert kv.status_bits() == 0


def test_hisa_with_every_block_is_the_flat_scan_bit_exact():
    """m >= #blocks: the same candidates in the same tile order through the
    same scoring kernel, so scores and indices agree exactly."""
    for dtype in ("bf16", "e4m3"):
        for B in (64, 128, 16):
            case = make_case(batch=2, L=[2048, 1500], H=64, d=128, B=B, m=4096, k=333,
                             dtype=dtype, seed=B, positions=[np.array([2047, 77, 1024]),
                                                             np.array([1499, 0])])
            kv = device_case(case)
            hs = run_hisa(case, kv)
            fl = run_flat(case, kv)
            assert np.array_equal(hs["idx"], fl["idx"])
            assert np.array_equal(hs["scores"].view(np.uint32), fl["scores"].view(np.uint32))


def test_tokens_scored_count():
    """Work per row: nb block representatives + min(m, nb) * B token slots."""
    case = make_case(batch=2, L=[5000, 900], H=8, d=128, B=64, m=10, k=100, seed=5,
                     positions=[np.array([4999, 63, 640]), np.array([899])])
    kv = device_case(case)
    gpu = run_hisa(case, kv)
    for i, t in enumerate(case.q_pos):
        nb = t // 64 + 1
        assert tuple(gpu["counts"][i]) == (nb, min(10, nb) * 64)


def test_own_block_kept_and_causal():
    case = make_case(batch=1, L=4096, H=16, d=128, B=128, m=4, k=256, seed=8,
                     positions=np.arange(3000, 3100, 7))
    kv = device_case(case)
    gpu = run_hisa(case, kv)
    for i, t in enumerate(case.q_pos):
        own = t // 128
        assert own in gpu["blocks"][i]
        v = gpu["idx"][i][gpu["idx"][i] >= 0]
        assert np.all(v <= t) and len(v) == min(256, gpu["nblocks"][i] * 128 - (128 * (own + 1) - t - 1))


def test_bad_query_rows_are_flagged_not_faulted():
    h = lib()
    case = make_case(batch=2, L=[500, 300], H=8, d=64, B=16, m=4, k=32, seed=9,
                     positions=[np.array([10]), np.array([20])])
    kv = device_case(case)
    Q, w, qs, qp = queries(case)
    qp[1] = 300          # == len: outside the prefix
    qs[0] = 5            # no such sequence
    idx = h.hisa_select(kv, Q, w, qs, qp, 4, 32)
    fidx = h.dsa_flat_select(kv, Q, w, qs, qp, 32)
    torch.cuda.synchronize()
    assert torch.all(idx == -1) and torch.all(fidx == -1)
    assert kv.status_bits() & h.HISA_DEV_BAD_QUERY


def test_last_position_default_and_empty_batch():
    h = lib()
    case = make_case(batch=3, L=[640, 700, 1], H=8, d=128, B=64, m=4, k=50, seed=10)
    kv = device_case(case)
    Q, w, qs, qp = queries(case)
    a = h.hisa_select(kv, Q, w, qs, qp, 4, 50)
    b = h.hisa_select(kv, Q, w, qs, None, 4, 50)       # NULL q_pos = last position
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    assert a[2, 0].item() == 0 and torch.all(a[2, 1:] == -1)   # one visible key
    e = h.hisa_select(kv, Q[:0], w[:0], qs[:0], qp[:0], 4, 50)
    assert e.shape == (0, 50)


def test_streams_and_workspace_reuse():
    """Back-to-back calls on a side stream reusing one workspace."""
    h = lib()
    case = make_case(batch=4, L=3000, H=64, d=128, B=128, m=8, k=512, seed=12)
    kv = device_case(case)
    Q, w, qs, qp = queries(case)
    ws = h.workspace(h.hisa_select_workspace_bytes(kv, case.n_q, 64, 8, 512))
    ref = h.hisa_select(kv, Q, w, qs, qp, 8, 512)
    s = torch.cuda.Stream()
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        outs = [h.hisa_select(kv, Q, w, qs, qp, 8, 512, ws=ws, stream=s) for _ in range(5)]
    s.synchronize()
    for o in outs:
        assert torch.equal(o, ref)
