"""Pins of the oracle's sparse attention: closed forms and the special case
that reduces to a library routine.  Each check returns None when the oracle
(or the library `lib` given) agrees, else a description of the disagreement,
so that both the pin tests and the planted-mistake tests can run them."""
import math

import numpy as np

import oracle
from hisa_inputs import bf16_bits, bf16_to_f32

D = 128


def _bf(x):
    return bf16_bits(np.asarray(x, dtype=np.float32))


def _run(lib, Qa, K, V, lens, q_seq, idx, scale):
    return oracle.sparse_attn(_bf(Qa), _bf(K), _bf(V), lens, q_seq, idx, scale, threads=1, lib=lib)


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape).astype(np.float32)


def single_entry_is_its_value(lib=None):
    """One valid entry: out is that token's value row exactly; lse its logit."""
    K, V, Qa = _rand((1, 80, D), 1), _rand((1, 80, D), 2), _rand((1, 2, D), 3)
    idx = np.array([[-1, 17, -1, 70, 64]], np.int32)           # 70 and 64: past len = 64, inside cap
    out, lse = _run(lib, Qa, K, V, [64], [0], idx, 0.125)
    v = bf16_to_f32(_bf(V))[0, 17].astype(np.float64)
    if not np.array_equal(out[0, 0], v) or not np.array_equal(out[0, 1], v):
        return "single entry: out differs from the value row"
    q, k = bf16_to_f32(_bf(Qa))[0].astype(np.float64), bf16_to_f32(_bf(K))[0, 17].astype(np.float64)
    if not np.allclose(lse[0], 0.125 * (q @ k), rtol=0, atol=1e-12):
        return "single entry: lse differs from scale * q.k"
    return None


def equal_logits_average_the_values(lib=None):
    """A zero query: every entry has logit 0, out is the mean of the values
    and lse = log(number of entries)."""
    V = _rand((1, 40, D), 4)
    idx = np.array([[3, 9, 27, 31, -1, 5]], np.int32)
    out, lse = _run(lib, np.zeros((1, 1, D)), _rand((1, 40, D), 5), V, [40], [0], idx, 0.3)
    want = bf16_to_f32(_bf(V))[0, [3, 9, 27, 31, 5]].astype(np.float64).mean(axis=0)
    if not np.allclose(out[0, 0], want, rtol=0, atol=1e-12):
        return "equal logits: out is not the mean of the values"
    if abs(lse[0, 0] - math.log(5)) > 1e-12:
        return "equal logits: lse is not log(5)"
    return None


def logit_gap_of_log3_weights_three_to_one(lib=None):
    """Two entries whose logits differ by ln 3 get weights 3/4 and 1/4, and
    lse = log(e^(2 ln 3) + e^(ln 3)) = log 12."""
    Qa = np.zeros((1, 1, D), np.float32)
    Qa[0, 0, 0] = 1.0
    K = np.zeros((1, 8, D), np.float32)
    K[0, 2, 0], K[0, 6, 0] = 2.0, 1.0
    V = _rand((1, 8, D), 6)
    out, lse = _run(lib, Qa, K, V, [8], [0], np.array([[6, 2]], np.int32), math.log(3.0))
    v = bf16_to_f32(_bf(V))[0].astype(np.float64)
    if not np.allclose(out[0, 0], 0.75 * v[2] + 0.25 * v[6], rtol=0, atol=1e-12):
        return "ln 3 gap: weights are not 3/4 and 1/4"
    if abs(lse[0, 0] - math.log(12.0)) > 1e-12:
        return "ln 3 gap: lse is not log 12"
    return None


def repeated_entry_counts_twice(lib=None):
    """An index listed twice carries twice the weight: with equal logits,
    entries [s, s, t] average to (2 v_s + v_t) / 3."""
    V = _rand((1, 16, D), 7)
    out, _ = _run(lib, np.zeros((1, 1, D)), _rand((1, 16, D), 8), V, [16], [0],
                  np.array([[4, 4, 11]], np.int32), 1.0)
    v = bf16_to_f32(_bf(V))[0].astype(np.float64)
    if not np.allclose(out[0, 0], (2 * v[4] + v[11]) / 3, rtol=0, atol=1e-12):
        return "repeated entry: not counted twice"
    return None


def no_valid_entry_gives_zero(lib=None):
    out, lse = _run(lib, _rand((1, 2, D), 9), _rand((1, 8, D), 10), _rand((1, 8, D), 11), [4], [0],
                    np.array([[-1, 4, 7, -1]], np.int32), 0.5)
    if np.any(out != 0) or not np.all(np.isneginf(lse)):
        return "no valid entry: out is not 0 or lse is not -inf"
    return None


def matches_library_attention(lib=None):
    """With every entry valid and distinct, the operator is dense attention
    over the gathered rows: torch's scaled_dot_product_attention in float64."""
    import torch
    rng = np.random.default_rng(12)
    batch, cap, Ha, n_q, k = 2, 300, 6, 3, 50
    K, V, Qa = _rand((batch, cap, D), 13), _rand((batch, cap, D), 14), _rand((n_q, Ha, D), 15)
    lens = np.array([300, 120], np.int32)
    q_seq = np.array([0, 1, 0], np.int32)
    idx = np.stack([rng.choice(int(lens[b]), k, replace=False) for b in q_seq]).astype(np.int32)
    scale = 1.0 / math.sqrt(D)
    out, lse = _run(lib, Qa, K, V, lens, q_seq, idx, scale)
    Kf, Vf, Qf = (bf16_to_f32(_bf(x)).astype(np.float64) for x in (K, V, Qa))
    for i in range(n_q):
        b = int(q_seq[i])
        q = torch.from_numpy(Qf[i])[None, :, None, :]                 # [1, Ha, 1, D]
        kk = torch.from_numpy(Kf[b, idx[i]])[None, None].expand(1, Ha, k, D)
        vv = torch.from_numpy(Vf[b, idx[i]])[None, None].expand(1, Ha, k, D)
        ref = torch.nn.functional.scaled_dot_product_attention(q, kk, vv, scale=scale)[0, :, 0].numpy()
        if not np.allclose(out[i], ref, rtol=0, atol=1e-12):
            return "differs from scaled_dot_product_attention"
        logits = (Qf[i] @ Kf[b, idx[i]].T) * scale
        if not np.allclose(lse[i], torch.logsumexp(torch.from_numpy(logits), dim=1).numpy(), rtol=0,
                           atol=1e-12):
            return "lse differs from logsumexp"
    return None


ALL = [single_entry_is_its_value, equal_logits_average_the_values,
       logit_gap_of_log3_weights_three_to_one, repeated_entry_counts_twice,
       no_valid_entry_gives_zero, matches_library_attention]


def any_fails(lib=None):
    for pin in ALL:
        msg = pin(lib)
        if msg:
            return msg
    return None
