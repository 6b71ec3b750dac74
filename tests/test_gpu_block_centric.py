"""Block-centric token scoring (rows that share their keys, as a prefill
chunk): one key tile per kept block, the query heads of several rows as the
MMA's N.  hisa_select takes that path for many rows per sequence; the same
rows selected in calls of fewer than 256 rows take the row-centric path.
The two must agree bit for bit (the same dot products, accumulated the same
way, and the same head sum), keeping every block must give the flat scan
exactly, and the rows must pass the parity rule against the oracle."""
import numpy as np
import pytest
import torch

from hisa_inputs import make_case
from tests.gpu_util import check_hisa, lib

pytestmark = pytest.mark.gpu


def _rows(case):
    return (torch.from_numpy(case.Q.view(np.int16)).view(torch.bfloat16).cuda(),
            torch.from_numpy(case.w).cuda(), torch.from_numpy(case.q_seq).cuda(),
            torch.from_numpy(case.q_pos).cuda())


def _select(h, kv, case, m, k, chunk=None):
    Q, w, qs, qp = _rows(case)
    n = case.n_q
    if chunk is None:
        r = h.hisa_select_inspect(kv, Q, w, qs, qp, m, k)
    else:
        parts = [h.hisa_select_inspect(kv, Q[i:i + chunk].contiguous(), w[i:i + chunk].contiguous(),
                                       qs[i:i + chunk].contiguous(), qp[i:i + chunk].contiguous(), m, k)
                 for i in range(0, n, chunk)]
        r = {key: torch.cat([p_[key] for p_ in parts]) for key in parts[0]}
    torch.cuda.synchronize()
    return {key: v.cpu().numpy() for key, v in r.items()}


def _prefill_case(H, L=9000, rows=512, batch=1, seed=0, k=300, m=12):
    # query rows at spread positions, several per block, partial own blocks included
    pos = np.sort(np.random.default_rng(seed).choice(np.arange(L // 3, L), size=rows // batch,
                                                     replace=False))
    return make_case(batch=batch, L=L, H=H, d=128, B=128, m=m, k=k, seed=900 + seed + H, positions=pos)


@pytest.mark.parametrize("H", [64, 20, 128])
def test_block_centric_equals_row_centric_bit_exact(H):
    h = lib()
    case = _prefill_case(H)
    kv = h.KVCache.from_case(case)
    h.hisa_pool_blocks(kv)
    bc = _select(h, kv, case, case.m, case.k)                 # 512 rows: block-centric
    rc = _select(h, kv, case, case.m, case.k, chunk=128)      # 128 rows a call: row-centric
    assert np.array_equal(bc["blocks"], rc["blocks"])
    assert np.array_equal(bc["idx"], rc["idx"])
    assert np.array_equal(bc["scores"].view(np.uint32), rc["scores"].view(np.uint32))
    assert np.array_equal(bc["counts"], rc["counts"])
    assert kv.status_bits() == 0


def test_block_centric_keeping_every_block_is_the_flat_scan():
    h = lib()
    case = _prefill_case(64, L=5000, rows=300, seed=3, k=700)
    nb = -(-case.cap // case.B)
    kv = h.KVCache.from_case(case)
    h.hisa_pool_blocks(kv)
    r = _select(h, kv, case, nb + 3, case.k)
    Q, w, qs, qp = _rows(case)
    fi, fs = h.dsa_flat_select(kv, Q, w, qs, qp, case.k, want_scores=True)
    torch.cuda.synchronize()
    assert np.array_equal(r["idx"], fi.cpu().numpy())
    assert np.array_equal(r["scores"].view(np.uint32), fs.cpu().numpy().view(np.uint32))


def test_block_centric_two_sequences_against_oracle():
    h = lib()
    case = _prefill_case(64, L=6000, rows=1024, batch=2, seed=5)
    kv = h.KVCache.from_case(case)
    h.hisa_pool_blocks(kv)
    gpu = _select(h, kv, case, case.m, case.k)
    rc = _select(h, kv, case, case.m, case.k, chunk=200)
    assert np.array_equal(gpu["idx"], rc["idx"])
    rows = np.random.default_rng(1).choice(case.n_q, size=48, replace=False)
    _, swaps = check_hisa(case, gpu, np.sort(rows))
    assert sum(a + b for a, b in swaps) <= 6
    assert kv.status_bits() == 0


def test_block_centric_invalid_rows():
    """Rows whose position lies past their sequence's end give -1 rows and
    HISA_DEV_BAD_QUERY; the other rows are unaffected."""
    h = lib()
    case = _prefill_case(64, L=7000, rows=400, seed=7)
    kv = h.KVCache.from_case(case)
    h.hisa_pool_blocks(kv)
    ref = _select(h, kv, case, case.m, case.k)
    bad = np.array([3, 77, 399])
    case.q_pos[bad] = 7000 + 5
    got = _select(h, kv, case, case.m, case.k)
    assert kv.status_bits() & h.HISA_DEV_BAD_QUERY
    assert np.all(got["idx"][bad] == -1)
    good = np.setdiff1d(np.arange(case.n_q), bad)
    assert np.array_equal(got["idx"][good], ref["idx"][good])
