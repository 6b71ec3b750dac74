"""GPU parity of the block index: mean- and max-pooling and append (sm_100a kernels)."""
import numpy as np
import pytest
import torch

import oracle
from hisa_inputs import bf16_bits, make_case
from tests.gpu_util import AppendRecorder, check_pooled, device_case, lib

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("B", [1, 16, 64, 100, 128, 512])
def test_pool_matches_oracle(dtype, d, B):
    case = make_case(batch=3, L=[1000, 777, 129], H=2, d=d, B=B, m=4, k=8, dtype=dtype,
                     seed=40 + B + d)
    kv = device_case(case)
    torch.cuda.synchronize()
    check_pooled(case, kv)
    assert kv.status_bits() == 0


@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
def test_pool_block_size_one_is_identity(dtype):
    case = make_case(batch=2, L=300, H=2, d=128, B=1, m=4, k=8, dtype=dtype, seed=3)
    kv = device_case(case)
    got = kv.pooled.cpu().numpy()
    ora = oracle.pool(oracle.Cache.of(case), 1)
    assert np.array_equal(got.astype(np.float64), ora)      # bit-exact


def test_pool_constant_blocks_exact():
    d, B = 128, 64
    keys = np.repeat((np.arange(8, dtype=np.float32) * 0.25 - 1.0)[:, None, None], B, 1)
    keys = np.broadcast_to(keys, (8, B, d)).reshape(1, 8 * B, d)
    case = make_case(batch=1, L=8 * B, H=2, d=d, B=B, m=2, k=4, seed=1)
    case.keys[:] = bf16_bits(keys)
    kv = device_case(case)
    got = kv.pooled.cpu().numpy()[0]
    assert np.array_equal(got, np.repeat((np.arange(8) * 0.25 - 1.0)[:, None], d, 1).astype(np.float32))


@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
@pytest.mark.parametrize("B", [64, 128, 100])
def test_append_equals_repool_bit_exact(dtype, B):
    h = lib()
    steps = 300
    case = make_case(batch=2, L=[1000, 640], H=2, d=128, B=B, m=4, k=8, dtype=dtype, seed=7,
                     append_steps=steps, cap=1400)
    kv = device_case(case)
    rec = AppendRecorder()
    for s in range(steps):
        tok = torch.from_numpy(case.append_keys[s].view(np.int16 if dtype == "bf16" else np.uint8)).cuda()
        sc = None if dtype == "bf16" else torch.from_numpy(case.append_scale[s]).cuda()
        h.hisa_append(kv, tok, sc)
        rec.record(kv)
    torch.cuda.synchronize()
    assert kv.len.cpu().tolist() == [1300, 940]
    assert rec.verify(kv) == 2 * steps          # every append, both sequences
    inc_p = kv.pooled.clone()
    inc_hl = kv.pooled_hl.clone()
    h.hisa_pool_blocks(kv)            # from scratch over the grown cache
    torch.cuda.synchronize()
    for b, n in enumerate([1300, 940]):
        nb = -(-n // B)
        assert torch.equal(inc_p[b, :nb], kv.pooled[b, :nb])
        assert torch.equal(inc_hl[b, :nb], kv.pooled_hl[b, :nb])
    # and the appended rows are where the oracle expects them
    grown = make_case(batch=2, L=[1000, 640], H=2, d=128, B=B, m=4, k=8, dtype=dtype, seed=7,
                      append_steps=steps, cap=1400)
    for b, L0 in enumerate([1000, 640]):
        grown.keys[b, L0:L0 + steps] = grown.append_keys[:, b]
        if dtype == "e4m3":
            grown.key_scale[b, L0:L0 + steps] = grown.append_scale[:, b]
    grown.lens = np.array([1300, 940], np.int32)
    kk = kv.keys.view(torch.int16 if dtype == "bf16" else torch.uint8).cpu().numpy()
    assert np.array_equal(kk.view(grown.keys.dtype), grown.keys)
    check_pooled(grown, kv)


def test_append_past_capacity_sets_status():
    h = lib()
    case = make_case(batch=1, L=64, H=2, d=64, B=16, m=2, k=4, seed=2, cap=64)
    kv = device_case(case)
    tok = torch.zeros((1, 64), dtype=torch.bfloat16, device="cuda")
    h.hisa_append(kv, tok)
    torch.cuda.synchronize()
    assert kv.len.item() == 64
    assert kv.status_bits() & h.HISA_DEV_CAPACITY


# ------------------------------------------------------------- max pooling


@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("B", [1, 16, 100, 128])
def test_pool_max_matches_oracle_bit_exact(dtype, d, B):
    """The elementwise max of fp32 key values is exact on both sides."""
    h = lib()
    case = make_case(batch=3, L=[1000, 777, 129], H=2, d=d, B=B, m=4, k=8, dtype=dtype,
                     seed=60 + B + d)
    kv = h.KVCache.from_case(case, pool="max")
    h.hisa_pool_blocks(kv)
    torch.cuda.synchronize()
    got = kv.pooled.cpu().numpy().astype(np.float64)
    ora = oracle.pool(oracle.Cache.of(case), B, mode="max")
    for b in range(case.batch):
        nbv = -(-int(case.lens[b]) // B)
        assert np.array_equal(got[b, :nbv], ora[b, :nbv])
    hl = kv.pooled_hl.view(torch.int16).cpu().numpy().view(np.uint16)
    g32 = kv.pooled.cpu().numpy()
    for b in range(case.batch):
        nbv = -(-int(case.lens[b]) // B)
        assert np.array_equal(bf16_bits(g32[b, :nbv]), hl[b, :nbv, :d])
    assert kv.status_bits() == 0


@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
def test_append_equals_repool_max_pooling(dtype):
    h = lib()
    steps, B = 200, 64
    case = make_case(batch=2, L=[1000, 640], H=2, d=128, B=B, m=4, k=8, dtype=dtype, seed=17,
                     append_steps=steps, cap=1300)
    kv = h.KVCache.from_case(case, pool="max")
    h.hisa_pool_blocks(kv)
    rec = AppendRecorder()
    for s in range(steps):
        tok = torch.from_numpy(case.append_keys[s].view(np.int16 if dtype == "bf16" else np.uint8)).cuda()
        sc = None if dtype == "bf16" else torch.from_numpy(case.append_scale[s]).cuda()
        h.hisa_append(kv, tok, sc)
        rec.record(kv)
    torch.cuda.synchronize()
    assert rec.verify(kv, pool="max") == 2 * steps
    inc = kv.pooled.clone()
    inc_hl = kv.pooled_hl.clone()
    h.hisa_pool_blocks(kv)
    torch.cuda.synchronize()
    for b, n in enumerate([1200, 840]):
        nb = -(-n // B)
        assert torch.equal(inc[b, :nb], kv.pooled[b, :nb])
        assert torch.equal(inc_hl[b, :nb], kv.pooled_hl[b, :nb])
