"""The seeded input generator: storage formats and the workload recipe."""
import numpy as np
import pytest
import torch

from hisa_inputs import (CONFIGS, bf16_bits, bf16_to_f32, e4m3_codes, e4m3_to_f32, make_case,
                         make_config, quantize_e4m3_rows)


def test_bf16_rounding_matches_torch():
    x = np.random.default_rng(0).standard_normal(200_000).astype(np.float32) * 3
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(bf16_bits(x), ref)
    assert np.array_equal(bf16_to_f32(ref), torch.from_numpy(ref.view(np.int16)).view(
        torch.bfloat16).float().numpy())


def test_e4m3_codes_match_torch_in_range():
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.standard_normal(200_000) * 60, rng.standard_normal(1000) * 1e-3,
                        [0.0, 448.0, -448.0, 2.0 ** -9, 2.0 ** -10, 3 * 2.0 ** -11]])
    x = np.clip(x, -448, 448).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(e4m3_codes(x), ref)


def test_e4m3_saturates_and_decodes():
    assert e4m3_codes(np.array([1e4, -1e4], np.float32)).tolist() == [0x7E, 0xFE]
    allc = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(allc).view(torch.float8_e4m3fn).float().numpy()
    got = e4m3_to_f32(allc)
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert np.array_equal(got[~np.isnan(got)], ref[~np.isnan(ref)])


def test_e4m3_rows_use_max_over_448_scale():
    k = np.random.default_rng(2).standard_normal((5, 16)).astype(np.float32)
    k[3] = 0
    codes, scale = quantize_e4m3_rows(k)
    assert scale[3] == 1.0
    np.testing.assert_array_equal(scale[[0, 1, 2, 4]],
                                  (np.abs(k[[0, 1, 2, 4]]).max(1) / np.float32(448)))
    assert np.all(np.abs(e4m3_to_f32(codes)).max(1)[[0, 1, 2, 4]] == 448.0)


def test_seeded_reproducible():
    a = make_config(0)
    b = make_config(0)
    assert np.array_equal(a.keys, b.keys) and np.array_equal(a.Q, b.Q)
    assert np.array_equal(a.w, b.w)
    c = make_config(0, seed=5)
    assert not np.array_equal(a.keys, c.keys)


def test_config_shapes():
    c0 = make_config(0)
    assert c0.keys.shape == (1, 2048, 64) and c0.Q.shape == (16, 4, 64)
    assert list(c0.q_pos) == list(range(2032, 2048))
    assert (c0.B, c0.m, c0.k) == (64, 8, 128)
    for i, spec in CONFIGS.items():
        assert spec["k"] in (128, 2048)
    s4 = make_config(4, L=1000, append_steps=7)
    assert s4.cap == 1007 and s4.append_keys.shape == (7, 1, 128)
    assert s4.append_Q.shape == (7, 1, 64, 128)
    s3 = make_config(3, batch=2, L=512)
    assert s3.keys.dtype == np.uint8 and s3.key_scale.shape == (2, 512)


def test_recipe_statistics():
    # keys = (mu_block + N(0, 0.25)) / sqrt(d): within-block spread 0.5/sqrt(d),
    # between-block spread 1/sqrt(d); queries N(0, 1)/sqrt(d); w ~ U(0, 1).
    c = make_case(batch=2, L=4096, H=8, d=64, B=64, m=4, k=16, seed=3,
                  positions=np.arange(4000, 4096))
    k = bf16_to_f32(c.keys).astype(np.float64) * np.sqrt(64)
    blocks = k.reshape(2, 64, 64, 64)
    within = blocks - blocks.mean(axis=2, keepdims=True)
    assert abs(within.std() - 0.5) < 0.01
    assert abs(blocks.mean(axis=2).std() - 1.0) < 0.05
    q = bf16_to_f32(c.Q) * 8
    assert abs(q.std() - 1.0) < 0.02
    assert 0.0 <= c.w.min() and c.w.max() < 1.0 and abs(c.w.mean() - 0.5) < 0.02


def test_append_rows_continue_block_clusters():
    c = make_case(batch=1, L=256, H=2, d=64, B=64, m=2, k=8, seed=8, append_steps=64,
                  positions=None)
    base = bf16_to_f32(c.keys[0, 192:256]).mean(0)
    app = bf16_to_f32(c.append_keys[:, 0]).mean(0)       # block 4 (positions 256..319)
    prev = bf16_to_f32(c.keys[0, 128:192]).mean(0)
    # appended rows form a new cluster: their mean is not block 3's mean
    assert np.linalg.norm(app - base) > 0.5 * np.linalg.norm(base - prev) * 0.5


@pytest.mark.parametrize("bad", [dict(positions=np.array([300]))])
def test_positions_must_be_inside_prefix(bad):
    with pytest.raises(AssertionError):
        make_case(batch=1, L=100, H=1, d=8, B=4, m=2, k=3, **bad)
