"""Parity at the full workload sizes (32K-128K contexts, top-k 2048), through
the same calls the bench times.  The oracle checks every row where it is
cheap and a seeded sample of rows elsewhere."""
import numpy as np
import pytest
import torch

from hisa_inputs import make_config
from tests.gpu_util import (AppendRecorder, check_flat, check_hisa, device_case, lib, run_flat,
                            run_hisa)
from tests.parity import iou

pytestmark = pytest.mark.gpu


def _sample(n, count, seed):
    if count >= n:
        return np.arange(n)
    return np.sort(np.random.default_rng(seed).choice(n, size=count, replace=False))


@pytest.mark.parametrize("cfg,hisa_rows,flat_rows", [(0, 16, 16), (1, 64, 6), (2, 256, 8),
                                                     (3, 32, 3)])
def test_config_parity(cfg, hisa_rows, flat_rows):
    case = make_config(cfg)
    kv = device_case(case)
    gpu_h = run_hisa(case, kv)
    gpu_f = run_flat(case, kv)
    assert kv.status_bits() == 0
    rows = _sample(case.n_q, hisa_rows, cfg)
    _, swaps = check_hisa(case, gpu_h, rows)
    n_swaps = sum(s for s, _ in swaps) + sum(t for _, t in swaps)
    assert n_swaps <= max(2, len(rows) // 8), f"{n_swaps} near-threshold swaps"
    check_flat(case, gpu_f, _sample(case.n_q, flat_rows, cfg + 100))
    # structure on every row
    for i in range(case.n_q):
        t = case.q_pos[i]
        v = gpu_h["idx"][i][gpu_h["idx"][i] >= 0]
        assert np.all(v <= t) and np.all(np.diff(v) > 0)
        assert tuple(gpu_h["counts"][i]) == (t // case.B + 1, min(case.m, t // case.B + 1) * case.B)
    mean_iou = float(np.mean([iou(a, b) for a, b in zip(gpu_h["idx"], gpu_f["idx"])]))
    print(f"config {cfg}: mean IoU(HISA, flat) = {mean_iou:.4f}")
    assert 0.0 < mean_iou <= 1.0


def test_streaming_append_config():
    """512 appends at 128K: after every append, select for the new last
    position.  Every step is checked: the block the append changed equals a
    from-scratch re-pool of that block bit for bit (and the oracle's mean
    within the pooled tolerance), and all 512 selections satisfy the parity
    rule against the oracle, which pools the grown cache from scratch for
    each row."""
    h = lib()
    case = make_config(4)
    steps = case.append_keys.shape[0]
    kv = device_case(case)
    L0 = int(case.lens[0])
    idx_all, sc_all, blocks_all, nblk_all, counts_all = [], [], [], [], []
    rec = AppendRecorder()
    qs = torch.zeros(1, dtype=torch.int32, device="cuda")
    for s in range(steps):
        tok = torch.from_numpy(case.append_keys[s].view(np.int16)).cuda()
        h.hisa_append(kv, tok)
        rec.record(kv)
        Q = torch.from_numpy(case.append_Q[s].view(np.int16)).view(torch.bfloat16).cuda()
        w = torch.from_numpy(case.append_w[s]).cuda()
        r = h.hisa_select_inspect(kv, Q, w, qs, None, case.m, case.k)
        idx_all.append(r["idx"])
        sc_all.append(r["scores"])
        blocks_all.append(r["blocks"])
        nblk_all.append(r["nblocks"])
        counts_all.append(r["counts"])
    torch.cuda.synchronize()
    assert kv.len.item() == L0 + steps and kv.status_bits() == 0
    assert rec.verify(kv) == steps                  # every append against a re-pool
    inc = kv.pooled.clone()
    h.hisa_pool_blocks(kv)
    torch.cuda.synchronize()
    assert torch.equal(inc, kv.pooled)
    # oracle on the grown cache, one row per step at position L0 + s
    grown = make_config(4)
    grown.keys[0, L0:L0 + steps] = grown.append_keys[:, 0]
    grown.lens = np.array([L0 + steps], np.int32)
    grown.Q = grown.append_Q[:, 0]
    grown.w = grown.append_w[:, 0]
    grown.q_seq = np.zeros(steps, np.int32)
    grown.q_pos = (L0 + np.arange(steps)).astype(np.int32)
    gpu = dict(idx=torch.cat(idx_all).cpu().numpy(), scores=torch.cat(sc_all).cpu().numpy(),
               blocks=torch.cat(blocks_all).cpu().numpy(), nblocks=torch.cat(nblk_all).cpu().numpy())
    rows = np.arange(steps)                          # all 512 steps
    _, swaps = check_hisa(grown, gpu, rows)
    assert len(swaps) == steps
    assert sum(a + b for a, b in swaps) <= max(2, len(rows) // 8)
    counts = torch.cat(counts_all).cpu().numpy()
    for s in range(steps):
        t = L0 + s
        assert tuple(counts[s]) == (t // case.B + 1, min(case.m, t // case.B + 1) * case.B)
    assert kv.status_bits() == 0
    print(f"streaming: {steps}/{steps} steps checked against the oracle, {steps} appends re-pooled")
