"""hisa_select_static: the selection with the library's fixed scratch array in
place of a caller workspace, for callers that cannot allocate device memory
while they select (an engine that has handed all free memory to its KV pages
up front, or a C caller with no allocator).  It runs the same kernels as
hisa_select, so calls in a row must reproduce hisa_select's output exactly,
allocate no memory, and reject a request larger than the array before
launching anything.

"Allocates no memory" is checked two ways: torch's allocator counter, and
the device's free memory (cudaMemGetInfo), which also sees any cudaMalloc or
cudaMallocAsync the library itself might make.  The first call on a device
looks up the array's address, which can load the library's device code, so
the free-memory check brackets the calls after that first one.

This file is collected last on purpose: the static array is shared by every
call on the device, so the test also shows that earlier tests leave nothing
behind that it depends on."""
import numpy as np
import pytest
import torch

from hisa_inputs import make_config
from tests.gpu_util import device_case, lib, queries

pytestmark = pytest.mark.gpu


def _outputs(case, n_q=None):
    n_q = case.n_q if n_q is None else n_q
    idx = torch.full((n_q, case.k), -7, dtype=torch.int32, device="cuda")
    sc = torch.full((n_q, case.k), -7.0, dtype=torch.float32, device="cuda")
    return idx, sc


@pytest.mark.parametrize("cfg", [0, 1, 3])
def test_static_scratch_matches_workspace_call(cfg):
    h = lib()
    case = make_config(cfg)
    kv = device_case(case)
    Q, w, qs, qp = queries(case)
    need = h.hisa_select_workspace_bytes(kv, case.n_q, case.H, case.m, case.k)
    assert 0 < need <= h.HISA_STATIC_SCRATCH_BYTES
    ref_idx, ref_sc = h.hisa_select(kv, Q, w, qs, qp, case.m, case.k, want_scores=True)
    torch.cuda.synchronize()
    ref_idx, ref_sc = ref_idx.cpu().numpy(), ref_sc.cpu().numpy()

    outs = [_outputs(case), _outputs(case), _outputs(case)]
    torch.cuda.synchronize()
    before = torch.cuda.memory_allocated()
    h.hisa_select_static(kv, Q, w, qs, qp, case.m, case.k, *outs[0])
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    for idx, sc in outs[1:]:
        h.hisa_select_static(kv, Q, w, qs, qp, case.m, case.k, idx, sc)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free_before
    assert torch.cuda.memory_allocated() == before
    for idx, sc in outs:
        got_idx, got_sc = idx.cpu().numpy(), sc.cpu().numpy()
        # same kernels, same arithmetic: identical selections; scores within
        # the parity tolerance (they are in fact bit-identical)
        np.testing.assert_array_equal(got_idx, ref_idx)
        fin = np.isfinite(ref_sc)
        np.testing.assert_array_equal(np.isfinite(got_sc), fin)
        assert np.all(np.abs(got_sc[fin] - ref_sc[fin]) <= 1e-3 * (1 + np.abs(ref_sc[fin])))
    assert kv.status_bits() == 0


def test_static_scratch_decode_rows_default_position():
    """q_pos NULL (each row's last position), as a decode step calls it."""
    h = lib()
    case = make_config(1)
    kv = device_case(case)
    Q, w, qs, _ = queries(case)
    ref = h.hisa_select(kv, Q, w, qs, None, case.m, case.k).cpu().numpy()
    idx, _ = _outputs(case)
    for _ in range(2):
        h.hisa_select_static(kv, Q, w, qs, None, case.m, case.k, idx)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(idx.cpu().numpy(), ref)


def test_static_scratch_rejects_oversized_requests():
    h = lib()
    case = make_config(1)
    kv = device_case(case)
    Q, w, qs, qp = queries(case)
    reps = 4                      # 256 rows need about 8.6 MB of scratch
    Q, w, qs, qp = (t.repeat(reps, *([1] * (t.dim() - 1))).contiguous() for t in (Q, w, qs, qp))
    n_q = case.n_q * reps
    assert h.hisa_select_workspace_bytes(kv, n_q, case.H, case.m, case.k) > \
        h.HISA_STATIC_SCRATCH_BYTES
    idx, sc = _outputs(case, n_q)
    with pytest.raises(h.HisaError) as e:
        h.hisa_select_static(kv, Q, w, qs, qp, case.m, case.k, idx, sc)
    assert e.value.code == h.HISA_E_SCRATCH_LIMIT
    torch.cuda.synchronize()
    assert bool((idx == -7).all()) and bool((sc == -7.0).all())   # nothing launched
    # the workspace entry point serves the same request
    h.hisa_select(kv, Q, w, qs, qp, case.m, case.k, idx=idx)
    torch.cuda.synchronize()
    assert bool((idx[:case.n_q] == idx[case.n_q:2 * case.n_q]).all())
