"""Context-parallel selection on one GPU: a sequence split by token range into
R shards, each shard's calls made in turn (no shard waits on another), the
exchanges done by stacking the shards' outputs in rank order (the layout of
an all-gather).  The merged result must equal hisa_select on the whole cache
bit for bit (indices, scores and kept blocks), and pass the oracle's
two-level parity rule."""
import numpy as np
import pytest
import torch

from hisa_inputs import make_case, make_config
from tests.gpu_util import check_hisa, lib, queries, run_hisa

pytestmark = pytest.mark.gpu


def run_cp(case, R, Lr, m, k, q_pos=None, pool="mean"):
    h = lib()
    shards = [h.KVCache.shard_of_case(case, r * Lr, Lr, pool=pool) for r in range(R)]
    for kv in shards:
        h.hisa_pool_blocks(kv)
    Q, w, qs, qp = queries(case)
    if q_pos is not None:
        qp = torch.from_numpy(np.asarray(q_pos, dtype=np.int32)).cuda()
    c1 = [h.hisa_cp_blocks(kv, r * Lr, Q, w, qs, qp, m) for r, kv in enumerate(shards)]
    kept, _ = h.hisa_merge_topk(torch.stack([c[0] for c in c1]), torch.stack([c[1] for c in c1]), m)
    c2 = [h.hisa_cp_tokens(kv, r * Lr, Q, w, qs, qp, m, k, kept) for r, kv in enumerate(shards)]
    idx, sc = h.hisa_merge_topk(torch.stack([c[0] for c in c2]), torch.stack([c[1] for c in c2]), k)
    torch.cuda.synchronize()
    status = 0
    for kv in shards:
        status |= kv.status_bits()
    return dict(idx=idx.cpu().numpy(), scores=sc.cpu().numpy(), kept=kept.cpu().numpy(),
                cand=[c[0].cpu().numpy() for c in c1], status=status)


def whole(case, m, k, q_pos=None, pool="mean"):
    h = lib()
    kv = h.KVCache.from_case(case, pool=pool)
    h.hisa_pool_blocks(kv)
    Q, w, qs, qp = queries(case)
    if q_pos is not None:
        qp = torch.from_numpy(np.asarray(q_pos, dtype=np.int32)).cuda()
    r = h.hisa_select_inspect(kv, Q, w, qs, qp, m, k)
    torch.cuda.synchronize()
    out = {key: v.cpu().numpy() for key, v in r.items()}
    out["status"] = kv.status_bits()
    return out


def assert_same(cp, ref, m):
    np.testing.assert_array_equal(cp["idx"], ref["idx"])
    got, want = cp["scores"].view(np.uint32), ref["scores"].view(np.uint32)
    live = ref["idx"] >= 0
    np.testing.assert_array_equal(got[live], want[live])
    assert np.all(np.isnan(cp["scores"][~live]))
    mm = ref["blocks"].shape[1]
    np.testing.assert_array_equal(cp["kept"][:, :mm], ref["blocks"])
    assert np.all(cp["kept"][:, mm:] == -1)


def gpu_view(cp, m, mm):
    kept = cp["kept"][:, :mm]
    return dict(idx=cp["idx"], scores=cp["scores"], blocks=kept,
                nblocks=(kept >= 0).sum(axis=1).astype(np.int32))


CASES = [
    # (batch, L per sequence, B, shard length, shards, H, d, m, k, dtype)
    (3, [4096, 3000, 1500], 128, 1024, 4, 16, 128, 6, 256, "bf16"),
    (2, [1536, 1400], 64, 512, 3, 8, 128, 10, 300, "e4m3"),
    (2, [2048, 2048], 64, 256, 8, 4, 64, 5, 200, "bf16"),
    (1, [1024], 128, 1024, 1, 16, 128, 4, 128, "bf16"),
]


def positions(L, Lr):
    """Query positions at shard starts and ends, inside shards, and the last."""
    pos = {0, 5, L - 1, L // 2, L // 3}
    for s in range(0, L, Lr):
        pos.update({s, s - 1, s + Lr // 2})
    return np.array(sorted(p for p in pos if 0 <= p < L))


@pytest.mark.parametrize("batch,Ls,B,Lr,R,H,d,m,k,dtype", CASES)
def test_cp_equals_hisa_select(batch, Ls, B, Lr, R, H, d, m, k, dtype):
    case = make_case(batch=batch, L=Ls, H=H, d=d, B=B, m=m, k=k, dtype=dtype,
                     positions=[positions(L, Lr) for L in Ls], seed=101 + R)
    assert R * Lr >= case.cap
    ref = whole(case, m, k)
    cp = run_cp(case, R, Lr, m, k)
    assert cp["status"] == 0 and ref["status"] == 0
    assert_same(cp, ref, m)
    check_hisa(case, gpu_view(cp, m, ref["blocks"].shape[1]), m=m, k=k)


def test_cp_candidates_mark_the_own_block():
    case = make_case(batch=1, L=[2048], H=8, d=128, B=128, m=4, k=64,
                     positions=np.array([100, 700, 1500]), seed=7)
    cp = run_cp(case, 2, 1024, 4, 64)
    cand0, cand1 = cp["cand"]
    # row at 100 and 700: shard 0 holds the own block (last entry, +inf); shard 1 sees nothing
    for r, t in ((0, 100), (1, 700)):
        own = t // 128
        live = cand0[r][cand0[r] >= 0]
        assert live[-1] == own and np.all(np.diff(live) > 0) and np.all(live <= own)
        assert np.all(cand1[r] == -1)
    # row at 1500: every block of shard 0 competes, the own block (11) is on shard 1
    live0 = cand0[2][cand0[2] >= 0]
    assert len(live0) == 3 and np.all(live0 < 8)
    live1 = cand1[2][cand1[2] >= 0]
    assert live1[-1] == 1500 // 128 and np.all(live1 >= 8)


def test_cp_all_blocks_and_short_rows():
    # m larger than the visible blocks keeps them all; k larger than the candidates pads
    case = make_case(batch=2, L=[1024, 700], H=8, d=128, B=128, m=64, k=4000,
                     positions=[np.array([50, 1023]), np.array([699])], seed=9)
    ref = whole(case, 64, 4000)
    cp = run_cp(case, 4, 256, 64, 4000)
    assert_same(cp, ref, 64)


def test_cp_max_pooling():
    case = make_case(batch=2, L=[3072, 2500], H=16, d=128, B=128, m=5, k=200,
                     positions=[positions(3072, 1024), positions(2500, 1024)], seed=11)
    ref = whole(case, 5, 200, pool="max")
    cp = run_cp(case, 3, 1024, 5, 200, pool="max")
    assert_same(cp, ref, 5)


def test_cp_bad_rows_flag_and_pad():
    case = make_case(batch=2, L=[1024, 512], H=8, d=128, B=128, m=3, k=64,
                     positions=[np.array([10, 1000]), np.array([300])], seed=13)
    q_pos = case.q_pos.copy()
    q_pos[2] = 600                       # past the second sequence's end
    cp = run_cp(case, 2, 512, 3, 64, q_pos=q_pos)
    ref = whole(case, 3, 64, q_pos=q_pos)
    h = lib()
    assert cp["status"] & h.HISA_DEV_BAD_QUERY and ref["status"] & h.HISA_DEV_BAD_QUERY
    assert np.all(cp["idx"][2] == -1) and np.all(ref["idx"][2] == -1)
    np.testing.assert_array_equal(cp["idx"][:2], ref["idx"][:2])


def test_cp_decode_32k_four_shards():
    """The 32K decode workload (64 sequences) split into four 8K shards."""
    case = make_config(1)
    ref = run_hisa(case, _pooled(case))
    cp = run_cp(case, 4, 8192, case.m, case.k, q_pos=case.lens - 1)
    assert cp["status"] == 0
    np.testing.assert_array_equal(cp["idx"], ref["idx"])
    live = ref["idx"] >= 0
    np.testing.assert_array_equal(cp["scores"].view(np.uint32)[live], ref["scores"].view(np.uint32)[live])


def _pooled(case):
    h = lib()
    kv = h.KVCache.from_case(case)
    h.hisa_pool_blocks(kv)
    return kv


@pytest.mark.parametrize("lists,n,k", [(3, 50, 40), (2, 128, 300), (4, 7, 5)])
def test_merge_rule_by_definition(lists, n, k):
    """hisa_merge_topk against a sort by (score desc, id asc) of the non-empty
    entries, with exact ties across lists, empty entries and k above the count."""
    rng = np.random.default_rng(lists * 100 + n)
    rows = 6
    ids = np.full((lists, rows, n), -1, np.int32)
    sc = np.zeros((lists, rows, n), np.float32)
    for r in range(rows):
        base = 0
        for l in range(lists):
            cnt = int(rng.integers(0, n + 1))
            ids[l, r, :cnt] = base + np.sort(rng.choice(1000, cnt, replace=False))
            sc[l, r, :cnt] = rng.integers(0, 6, cnt).astype(np.float32) * 0.5   # many exact ties
            base += 1000                                                       # list ranges ascend
    h = lib()
    idx, out = h.hisa_merge_topk(torch.from_numpy(ids).cuda(), torch.from_numpy(sc).cuda(), k)
    torch.cuda.synchronize()
    idx, out = idx.cpu().numpy(), out.cpu().numpy()
    for r in range(rows):
        ent = sorted((-float(sc[l, r, j]), int(ids[l, r, j])) for l in range(lists) for j in range(n)
                     if ids[l, r, j] >= 0)[:k]
        want = sorted(g for _, g in ent)
        got = [g for g in idx[r] if g >= 0]
        assert got == want
        assert np.all(idx[r, len(want):] == -1) and np.all(np.isnan(out[r, len(want):]))
        score_of = {g: -s for s, g in ent}
        assert all(out[r, i] == score_of[g] for i, g in enumerate(got))
