"""The binding refuses caller-owned buffers the library cannot size-check.

The C calls take raw pointers, so a short idx / scores, a w or q_seq of the
wrong length, or a tensor on another device would let the kernels write or
read outside the caller's buffers.  The Python binding checks those shapes
and raises ValueError before the library call.  Each GPU case below backs its
bad tensor with a larger allocation filled with -7, so the check is seen to
hold (the fill survives) without any access outside memory this test owns."""
import numpy as np
import pytest
import torch

from hisa_inputs import make_case


def _case():
    return make_case(batch=2, L=[700, 300], H=4, d=64, B=64, m=3, k=32, seed=5)


def _args(h, case, device):
    kv = h.KVCache.from_case(case, device=device)
    Q = torch.from_numpy(case.Q.view(np.int16)).view(torch.bfloat16).to(device)
    w = torch.from_numpy(case.w).to(device)
    qs = torch.from_numpy(case.q_seq).to(device)
    qp = torch.from_numpy(case.q_pos).to(device)
    return kv, Q, w, qs, qp


def _backed(shape_numel, dtype, device, fill=-7):
    """A contiguous tensor of `shape_numel` entries at the start of a buffer
    twice that size, all set to `fill`."""
    big = torch.full((2 * shape_numel + 64,), fill, dtype=dtype, device=device)
    return big, big[:shape_numel]


def _bad_calls(h, case, device):
    """(description, call, backing buffers that must keep their fill)."""
    kv, Q, w, qs, qp = _args(h, case, device)
    n_q, k, m = case.n_q, case.k, case.m
    calls = []
    big, short_idx = _backed(n_q * k - 1, torch.int32, device)
    calls.append(("short idx", lambda: h.hisa_select_static(kv, Q, w, qs, qp, m, k, short_idx), big))
    big2, idx_ok = _backed(n_q * k, torch.int32, device)
    bigs, short_sc = _backed(n_q * k - 5, torch.float32, device)
    calls.append(("short scores",
                  lambda: h.hisa_select_static(kv, Q, w, qs, qp, m, k, idx_ok, short_sc), big2))
    w_short = w.reshape(-1)[:-1].contiguous()
    calls.append(("w of the wrong shape",
                  lambda: h.hisa_select_static(kv, Q, w_short, qs, qp, m, k, idx_ok), big2))
    calls.append(("q_seq of the wrong length",
                  lambda: h.hisa_select_static(kv, Q, w, qs[:-1].contiguous(), qp, m, k, idx_ok), big2))
    calls.append(("q_pos of the wrong length",
                  lambda: h.hisa_select_static(kv, Q, w, qs, qp[:-1].contiguous(), m, k, idx_ok), big2))
    Q2 = Q.reshape(n_q, -1).contiguous()
    calls.append(("Q not 3-D", lambda: h.hisa_select_static(kv, Q2, w, qs, qp, m, k, idx_ok), big2))
    Qd = torch.zeros((n_q, case.H, 2 * case.d), dtype=torch.bfloat16, device=device)
    calls.append(("Q head dim not d", lambda: h.hisa_select_static(kv, Qd, w, qs, qp, m, k, idx_ok), big2))
    calls.append(("idx of the wrong dtype",
                  lambda: h.hisa_select_static(kv, Q, w, qs, qp, m, k, idx_ok.float()), big2))
    calls.append(("hisa_select with a short idx",
                  lambda: h.hisa_select(kv, Q, w, qs, qp, m, k, idx=short_idx), big))
    calls.append(("hisa_select with short scores",
                  lambda: h.hisa_select(kv, Q, w, qs, qp, m, k, idx=idx_ok, scores=short_sc,
                                        want_scores=True), big2))
    calls.append(("dsa_flat_select with a short idx",
                  lambda: h.dsa_flat_select(kv, Q, w, qs, qp, k, idx=short_idx), big))
    calls.append(("hisa_levels_select with a short idx",
                  lambda: h.hisa_levels_select([kv], Q, w, qs, qp, [m], k, idx=short_idx), big))
    calls.append(("hisa_levels_select with one keep count for two levels",
                  lambda: h.hisa_levels_select([kv, h.superblock_index(kv, 4)], Q, w, qs, qp, [m], k,
                                               idx=idx_ok), big2))
    ws_f32 = torch.zeros(1 << 20, dtype=torch.float32, device=device)
    calls.append(("workspace not bytes",
                  lambda: h.hisa_select(kv, Q, w, qs, qp, m, k, ws=ws_f32, idx=idx_ok), big2))
    return calls, (big, big2, bigs)


def _run(h, case, device):
    calls, backs = _bad_calls(h, case, device)
    for what, call, _ in calls:
        with pytest.raises(ValueError):
            call()
    for b in backs:
        assert bool((b == -7).all()), "a refused call wrote to its output"
    return len(calls)


@pytest.mark.skipif(torch.cuda.is_available(), reason="the GPU variant runs instead")
def test_binding_refuses_bad_buffers_cpu_tensors():
    """Host tensors: every bad case must be refused in Python (the library is
    never reached, so no device is needed)."""
    import hierarchical_top_indexer_b200 as h
    assert _run(h, _case(), "cpu") == 14


@pytest.mark.gpu
def test_binding_refuses_bad_buffers():
    import hierarchical_top_indexer_b200 as h
    case = _case()
    assert _run(h, case, "cuda") == 14
    torch.cuda.synchronize()
    # and the well-formed call still works on the same tensors
    kv, Q, w, qs, qp = _args(h, case, "cuda")
    h.hisa_pool_blocks(kv)
    idx = torch.full((case.n_q, case.k), -7, dtype=torch.int32, device="cuda")
    h.hisa_select_static(kv, Q, w, qs, qp, case.m, case.k, idx)
    ref = h.hisa_select(kv, Q, w, qs, qp, case.m, case.k)
    torch.cuda.synchronize()
    assert torch.equal(idx, ref)
