"""hisa_decode_step: the append and the selection for every sequence's new
last position in one call, the append fused into block scoring where rows are
short enough.  Its results must equal hisa_append followed by hisa_select on
an identical cache, bit for bit (indices, scores, the cache and its index,
lengths and status bits), step after step, on the fused path and on the
separate-launch path; and the selections must pass the parity rule against
the oracle on every step."""
import numpy as np
import pytest
import torch

from hisa_inputs import make_case, make_config
from tests.gpu_util import check_hisa, lib

pytestmark = pytest.mark.gpu


def _twin(case, pool="mean"):
    h = lib()
    a = h.KVCache.from_case(case, pool=pool)
    b = h.KVCache.from_case(case, pool=pool)
    h.hisa_pool_blocks(a)
    h.hisa_pool_blocks(b)
    return a, b


def _tok(case, s):
    t = case.append_keys[s]
    if case.dtype == "bf16":
        return torch.from_numpy(t.view(np.int16)).view(torch.bfloat16).cuda(), None
    return torch.from_numpy(t).cuda(), torch.from_numpy(case.append_scale[s]).cuda()


def _same(x, y):
    if x is None:
        return y is None
    return torch.equal(x.contiguous().view(torch.uint8), y.contiguous().view(torch.uint8))


def run_twins(case, steps, m=None, k=None, pool="mean", set_len=None):
    """Steps of hisa_decode_step on one cache and hisa_append + hisa_select on
    its twin; every output and every cache buffer compared after each step."""
    h = lib()
    m, k = m or case.m, k or case.k
    a, b = _twin(case, pool)
    if set_len is not None:
        a.len.copy_(torch.tensor(set_len, dtype=torch.int32))
        b.len.copy_(torch.tensor(set_len, dtype=torch.int32))
    qs = torch.arange(case.batch, dtype=torch.int32, device="cuda")
    outs = []
    for s in range(steps):
        tok, sc = _tok(case, s)
        Q = torch.from_numpy(case.append_Q[s % case.append_Q.shape[0]].view(np.int16)).view(torch.bfloat16).cuda()
        w = torch.from_numpy(case.append_w[s % case.append_w.shape[0]]).cuda()
        ia, sa = h.hisa_decode_step(a, tok, Q, w, m, k, tok_scale=sc, want_scores=True)
        h.hisa_append(b, tok, sc)
        ib, sb = h.hisa_select(b, Q, w, qs, None, m, k, want_scores=True)
        torch.cuda.synchronize()
        assert torch.equal(ia, ib), f"step {s}: indices differ"
        assert _same(sa, sb), f"step {s}: scores differ"
        for name in ("keys", "key_scale", "pooled", "pooled_hl", "len", "status"):
            assert _same(getattr(a, name), getattr(b, name)), f"step {s}: {name} differs"
        outs.append((ia.cpu().numpy(), sa.cpu().numpy()))
    return a, outs


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("bf16", 64), ("e4m3", 128), ("e4m3", 64)])
@pytest.mark.parametrize("B", [64, 128])
def test_decode_step_equals_append_then_select(dtype, d, B):
    # lengths: empty (set on the device), one key, a block boundary just
    # ahead, just behind, ragged
    L = [1, 1, B - 2, B, 3 * B + 5, 1000]
    case = make_case(batch=len(L), L=L, H=8, d=d, B=B, m=4, k=64, dtype=dtype, seed=71 + d + B,
                     append_steps=6, cap=1100)
    L[0] = 0
    a, _ = run_twins(case, 6, set_len=L)
    assert a.len.cpu().tolist() == [n + 6 for n in L]
    assert a.status_bits() == 0


def test_decode_step_max_pooling():
    case = make_case(batch=3, L=[60, 200, 513], H=8, d=128, B=64, m=3, k=40, seed=81,
                     append_steps=5, cap=700)
    run_twins(case, 5, pool="max")


def test_decode_step_full_and_bad_lengths():
    """A full sequence appends nothing (HISA_DEV_CAPACITY) and selects for
    cap - 1; a length outside [0, cap] gives a -1 row with HISA_DEV_BAD_LEN and
    HISA_DEV_BAD_QUERY -- the same as the two separate calls."""
    h = lib()
    case = make_case(batch=3, L=[254, 100, 50], H=4, d=128, B=64, m=2, k=32, seed=83,
                     append_steps=2, cap=256)
    a, outs = run_twins(case, 2, set_len=[256, 100, 300])
    assert a.status_bits() == h.HISA_DEV_CAPACITY | h.HISA_DEV_BAD_LEN | h.HISA_DEV_BAD_QUERY
    assert a.len.cpu().tolist() == [256, 102, 300]
    for idx, _ in outs:
        assert np.all(idx[2] == -1)
        assert np.all((idx[0] >= 0) & (idx[0] <= 255))


@pytest.mark.parametrize("shape", ["long_rows", "many_rows"])
def test_decode_step_separate_launch_path(shape):
    """Rows of more than 512 blocks, or more than two rows per SM, take the
    separate-launch path; results are the same."""
    if shape == "long_rows":
        case = make_case(batch=2, L=[1100 * 64 + 3, 70000], H=8, d=128, B=64, m=8, k=128, seed=85,
                         append_steps=3, cap=72000)
    else:
        sms = torch.cuda.get_device_properties(0).multi_processor_count
        case = make_case(batch=2 * sms + 3, L=200, H=4, d=64, B=64, m=2, k=16, seed=86,
                         append_steps=2, cap=300)
    run_twins(case, case.append_keys.shape[0])


def test_decode_step_32k_workload_matches_oracle_every_step():
    """The 32K decode workload (64 sequences), 4 steps through the fused path:
    equal to the separate calls, and every row of every step within the
    parity rule against the oracle run on the grown cache."""
    case = make_config(1, cap=32768 + 4, append_steps=4, append_query_sets=4)
    a, outs = run_twins(case, 4)
    L0 = case.lens.copy()
    grown = make_config(1, cap=32768 + 4, append_steps=4, append_query_sets=4)
    for s, (idx, sc) in enumerate(outs):
        for b in range(case.batch):
            grown.keys[b, L0[b] + s] = grown.append_keys[s, b]
        grown.lens = (L0 + s + 1).astype(np.int32)
        grown.Q = grown.append_Q[s]
        grown.w = grown.append_w[s]
        grown.q_seq = np.arange(case.batch, dtype=np.int32)
        grown.q_pos = (L0 + s).astype(np.int32)
        gpu = dict(idx=idx, scores=sc)
        # the token half of the rule needs the kept blocks: rerun the
        # inspection call on a cache grown the same way
        h = lib()
        kv = h.KVCache.from_case(grown)
        h.hisa_pool_blocks(kv)
        r = h.hisa_select_inspect(kv, torch.from_numpy(grown.Q.view(np.int16)).view(torch.bfloat16).cuda(),
                                  torch.from_numpy(grown.w).cuda(), torch.from_numpy(grown.q_seq).cuda(),
                                  torch.from_numpy(grown.q_pos).cuda(), case.m, case.k)
        torch.cuda.synchronize()
        assert np.array_equal(r["idx"].cpu().numpy(), idx)
        gpu.update(blocks=r["blocks"].cpu().numpy(), nblocks=r["nblocks"].cpu().numpy())
        _, swaps = check_hisa(grown, gpu)
        assert sum(x + y for x, y in swaps) <= max(2, case.batch // 8)
        del kv
