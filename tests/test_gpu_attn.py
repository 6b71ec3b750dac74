"""Sparse attention over selected tokens against the oracle (plain definition
in double).  Tolerance from the arithmetic: the logits are exact bf16
products summed in fp32; the softmax weights w_j (normalised by their fp32
sum) are rounded to bf16 (relative error <= 2^-9 each) before the
weights-times-values product, so out = sum_j w_j (1 + d_j) v_j with
sum_j w_j = 1 and |d_j| <= 2^-9, and the hardware 2^x adds about 2^-22:
|out - out_ref| <= 2^-9 * max |v| over the row's entries plus fp32
accumulation; the tests allow 2^-8 * max |v| + 1e-5, and 2^-8 on lse."""
import math

import numpy as np
import pytest
import torch

import oracle
from hisa_inputs import bf16_bits, bf16_to_f32, make_config
from tests.gpu_util import device_case, lib, queries

pytestmark = pytest.mark.gpu
D = 128


def _inputs(batch, cap, lens, n_q, Ha, seed):
    rng = np.random.default_rng(seed)
    K = bf16_bits(rng.standard_normal((batch, cap, D), dtype=np.float32))
    V = bf16_bits(rng.standard_normal((batch, cap, D), dtype=np.float32))
    Qa = bf16_bits(rng.standard_normal((n_q, Ha, D), dtype=np.float32))
    return K, V, Qa, np.asarray(lens, np.int32)


def _dev16(x):
    return torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()


def run_gpu(K, V, Qa, lens, q_seq, idx, scale):
    h = lib()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = h.hisa_sparse_attn(_dev16(Qa), _dev16(K), _dev16(V), torch.from_numpy(lens).cuda(),
                                  torch.from_numpy(np.asarray(q_seq, np.int32)).cuda(),
                                  torch.from_numpy(np.ascontiguousarray(idx, np.int32)).cuda(), scale,
                                  status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return out.cpu().numpy(), lse.cpu().numpy()


def check(K, V, Qa, lens, q_seq, idx, scale, rows=None):
    out, lse = run_gpu(K, V, Qa, lens, q_seq, idx, scale)
    rows = np.arange(len(q_seq)) if rows is None else np.asarray(rows)
    ro, rl = oracle.sparse_attn(Qa[rows], K, V, lens, np.asarray(q_seq)[rows], idx[rows], scale)
    Vf = bf16_to_f32(V)
    for r, i in enumerate(rows):
        b = int(q_seq[i])
        sel = [s for s in idx[i] if 0 <= s < lens[b]]
        if not sel:
            assert np.all(out[i] == 0) and np.all(np.isneginf(lse[i]))
            continue
        vmax = float(np.abs(Vf[b, sel]).max())
        np.testing.assert_allclose(out[i], ro[r], rtol=0, atol=2.0 ** -8 * vmax + 1e-5)
        np.testing.assert_allclose(lse[i], rl[r], rtol=0, atol=2.0 ** -8)
    return out, lse


@pytest.mark.parametrize("Ha,k,n_q,seed", [(128, 2048, 20, 6), (128, 300, 5, 1), (64, 128, 7, 2),
                                           (16, 1, 4, 3), (128, 4096, 2, 4), (128, 129, 3, 5)])
def test_attention_matches_oracle(Ha, k, n_q, seed):
    # 20 rows of 16 tiles over at most 148 CTAs: segments of several tiles,
    # whose running maxima grow from tile to tile (the rescaling path)
    batch, cap = 3, 5000
    lens = [5000, 3000, 700]
    K, V, Qa, lens = _inputs(batch, cap, lens, n_q, Ha, seed)
    rng = np.random.default_rng(seed + 10)
    q_seq = rng.integers(0, batch, n_q).astype(np.int32)
    idx = np.stack([np.sort(rng.choice(int(lens[b]), min(k, int(lens[b])), replace=False))
                    if k <= lens[b] else rng.integers(0, lens[b], k) for b in q_seq]).astype(np.int32)
    idx = idx[:, :k] if idx.shape[1] >= k else np.pad(idx, ((0, 0), (0, k - idx.shape[1])), constant_values=-1)
    # padding, entries past the sequence's length and repeated indices
    if k >= 8:
        idx[:, -3:] = -1
        idx[0, 1] = lens[q_seq[0]] + 5 if lens[q_seq[0]] + 5 < cap else -1
        idx[-1, 2] = idx[-1, 3]
    check(K, V, Qa, lens, q_seq, idx, 1.0 / math.sqrt(D))


def test_rows_without_valid_entries():
    K, V, Qa, lens = _inputs(2, 600, [600, 100], 3, 32, 7)
    idx = np.full((3, 200), -1, np.int32)
    idx[0, :50] = np.arange(50)
    idx[1, :10] = np.arange(100, 110)          # all past the second sequence's length
    check(K, V, Qa, lens, [0, 1, 0], idx, 0.1)


def test_many_rows_per_cta():
    # 1000 rows of one tile: every CTA reloads the query heads row after row
    n_q = 1000
    K, V, Qa, lens = _inputs(2, 2048, [2048, 1500], n_q, 128, 8)
    rng = np.random.default_rng(9)
    q_seq = rng.integers(0, 2, n_q).astype(np.int32)
    idx = np.stack([np.sort(rng.choice(int(lens[b]), 100, replace=False)) for b in q_seq]).astype(np.int32)
    check(K, V, Qa, lens, q_seq, idx, 1.0 / math.sqrt(D), rows=np.arange(0, n_q, 37))


def test_attention_over_hisa_selection():
    """The decode workload: the indexer's top-2048 of 32K keys per row feeds
    attention with 128 heads over separate key and value caches."""
    case = make_config(1)
    kv = device_case(case)
    Q, w, qs, qp = queries(case)
    idx = lib().hisa_select(kv, Q, w, qs, qp, case.m, case.k).cpu().numpy()
    K, V, Qa, lens = _inputs(case.batch, case.cap, case.lens, case.n_q, 128, 11)
    check(K, V, Qa, lens, case.q_seq, idx, 1.0 / math.sqrt(D), rows=np.arange(0, case.n_q, 8))
