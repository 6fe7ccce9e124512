"""Pins of the oracle's dropout (CPU only).

The generator (Philox4x32-10) is pinned to the published known-answer
vectors, and its round structure to numpy's Philox4x64-10 bit generator; the
keep rule to its rate and independence; the dropout forward to a separate
brute force, to closed forms and to unbiasedness; its backward to finite
differences through the forward.  Planted mistakes must fail at least one pin.
"""

import json
import os

import numpy as np
import pytest

from oracle import attention_backward_ref, attention_bruteforce, attention_ref
from oracle.philox import dropout_keep, dropout_threshold, philox4x32, philox4x64_py

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "philox4x32_10_kat.json")


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def test_philox4x32_known_answer_vectors():
    for vec in json.load(open(GOLDEN))["vectors"]:
        c = np.array([int(x, 16) for x in vec["counter"]], dtype=np.uint64)
        k = np.array([int(x, 16) for x in vec["key"]], dtype=np.uint64)
        want = [int(x, 16) for x in vec["output"]]
        assert [int(x) for x in philox4x32(c, k)] == want


def test_philox_rounds_match_numpy_philox4x64():
    """numpy's Philox bit generator is Philox4x64-10; its first four outputs
    are the rounds applied to the counter plus one."""
    rng = np.random.default_rng(5)
    for _ in range(8):
        key = [int(x) for x in rng.integers(0, 2 ** 63, 2)]
        ctr = [int(x) for x in rng.integers(0, 2 ** 63, 4)]
        bg = np.random.Philox(key=np.array(key, dtype=np.uint64), counter=np.array(ctr, dtype=np.uint64))
        raw = [int(x) for x in bg.random_raw(4)]
        assert raw == list(philox4x64_py([ctr[0] + 1] + ctr[1:], key))


def test_philox4x32_vectorised_equals_one_at_a_time():
    rng = np.random.default_rng(6)
    ctr = rng.integers(0, 2 ** 32, (50, 4), dtype=np.uint64)
    key = rng.integers(0, 2 ** 32, 2, dtype=np.uint64)
    batch = philox4x32(ctr, key)
    for i in range(50):
        assert np.array_equal(batch[i], philox4x32(ctr[i], key))


def test_keep_bits_follow_the_stated_layout():
    """Key j of row i takes the (j mod 2) half of word (j mod 8) // 2 of the
    call with counter (j // 8, i, b H + h, offset)."""
    seed, offset, b, h, H, p = 0x1234_5678_9ABC_DEF0, 77, 1, 2, 3, 0.3
    keep = dropout_keep(seed, offset, b, h, H, [5, 9], 20, p)
    t = dropout_threshold(p)
    for r, i in enumerate([5, 9]):
        for j in range(20):
            words = philox4x32(np.array([j // 8, i, b * H + h, offset], dtype=np.uint64),
                               np.array([seed & 0xFFFFFFFF, seed >> 32], dtype=np.uint64))
            w = int(words[(j % 8) // 2])
            u = (w >> 16) if j % 2 else (w & 0xFFFF)
            assert keep[r, j] == (u >= t)


@pytest.mark.parametrize("p", [0.1, 0.5, 0.9])
def test_keep_rate(p):
    keep = dropout_keep(11, 0, 0, 0, 1, np.arange(512), 2048, p)
    n = keep.size
    rate = 1.0 - dropout_threshold(p) / 65536.0
    sigma = np.sqrt(rate * (1 - rate) / n)
    assert abs(keep.mean() - rate) < 5 * sigma
    # rows and columns are not striped: every row and column keeps about the same share
    assert abs(keep.mean(axis=1) - rate).max() < 6 * np.sqrt(rate * (1 - rate) / 2048)
    assert abs(keep.mean(axis=0) - rate).max() < 6 * np.sqrt(rate * (1 - rate) / 512)


def test_streams_are_independent():
    """Different heads, batches, offsets and seeds give unrelated masks:
    agreement near (1-p)^2 + p^2."""
    p = 0.5
    base = dropout_keep(3, 0, 0, 0, 4, np.arange(128), 1024, p)
    for other in (dropout_keep(3, 0, 0, 1, 4, np.arange(128), 1024, p),
                  dropout_keep(3, 0, 1, 0, 4, np.arange(128), 1024, p),
                  dropout_keep(3, 1, 0, 0, 4, np.arange(128), 1024, p),
                  dropout_keep(4, 0, 0, 0, 4, np.arange(128), 1024, p),
                  dropout_keep(3 + (1 << 32), 0, 0, 0, 4, np.arange(128), 1024, p)):
        agree = (base == other).mean()
        assert abs(agree - 0.5) < 5 * np.sqrt(0.25 / base.size)


def test_threshold_rounding_and_range():
    assert dropout_threshold(0.0) == 0
    assert dropout_threshold(0.1) == 6554
    assert dropout_threshold(0.5) == 32768
    for bad in (-0.1, 1.0, 1.5):
        with pytest.raises(ValueError):
            dropout_threshold(bad)


# ----------------------------------------------------------------- forward

def test_dropout_agrees_with_bruteforce():
    for (n_q, n_k, H, h_kv, D, causal, wl) in [(5, 7, 2, 1, 3, False, -1), (9, 9, 2, 2, 4, True, -1),
                                              (6, 10, 1, 1, 2, True, 2)]:
        q, k, v = _rand((2, n_q, H, D), 1), _rand((2, n_k, h_kv, D), 2), _rand((2, n_k, h_kv, D), 3)
        o, l = attention_ref(q, k, v, 0.7, causal, wl, dropout_p=0.3, seed=99, offset=5)
        ob, lb = attention_bruteforce(q.tolist(), k.tolist(), v.tolist(), 0.7, causal, wl, dropout_p=0.3, seed=99,
                                      offset=5)
        assert np.allclose(o, np.array(ob), atol=1e-12)
        assert np.allclose(l, np.array(lb), atol=1e-12)


def test_dropout_leaves_lse_and_constant_v_closed_form():
    """LSE is the softmax normaliser, unchanged by dropout; with every V row
    equal to c, O_i = c * sum_j Z_ij P_ij / (1 - p)."""
    q, k = _rand((1, 40, 2, 4), 4), _rand((1, 40, 2, 4), 5)
    c = np.array([0.5, -2.0, 3.0, 1.0])
    v = np.broadcast_to(c, (1, 40, 2, 4)).copy()
    p = 0.25
    o, l, probs = attention_ref(q, k, v, 0.5, True, -1, return_probs=True, dropout_p=p, seed=7, offset=1)
    _, l0 = attention_ref(q, k, v, 0.5, True)
    assert np.array_equal(l, l0)
    for h in range(2):
        z = dropout_keep(7, 1, 0, h, 2, np.arange(40), 40, p)
        kept = (z * probs[0, h]).sum(axis=1) / (1 - p)
        assert np.allclose(o[0, :, h, :], kept[:, None] * c[None, :], atol=1e-13)


def test_dropout_is_unbiased():
    """Averaged over offsets, the dropout output approaches the plain one."""
    q, k, v = _rand((1, 16, 1, 4), 8), _rand((1, 32, 1, 4), 9), _rand((1, 32, 1, 4), 10)
    o0, _ = attention_ref(q, k, v, 0.6)
    p = 0.4
    outs = np.stack([attention_ref(q, k, v, 0.6, dropout_p=p, seed=123, offset=t)[0] for t in range(600)])
    mean, sd = outs.mean(axis=0), outs.std(axis=0) / np.sqrt(outs.shape[0])
    assert np.all(np.abs(mean - o0) <= 5 * sd + 1e-12)


def test_tiny_dropout_probability_keeps_everything():
    """p below half a 16-bit step rounds to a zero threshold: every key kept,
    O scaled by 1 / (1 - p)."""
    q, k, v = _rand((1, 8, 1, 4), 11), _rand((1, 8, 1, 4), 12), _rand((1, 8, 1, 4), 13)
    p = 1e-6
    o, _ = attention_ref(q, k, v, 1.0, dropout_p=p, seed=1)
    o0, _ = attention_ref(q, k, v, 1.0)
    assert np.allclose(o, o0 / (1 - p), atol=1e-15)


def _mut_normalise_after_drop(q, k, v, scale, causal, wl, p, seed, offset):
    """Mistake: the softmax normaliser taken over the kept keys only."""
    B, n_q, H, D = q.shape
    out = np.zeros_like(q)
    for b in range(B):
        for h in range(H):
            s = scale * q[b, :, h] @ k[b, :, h].T
            vis = np.ones_like(s, dtype=bool) if not causal else np.tril(np.ones_like(s, dtype=bool))
            z = dropout_keep(seed, offset, b, h, H, np.arange(n_q), k.shape[1], p) & vis
            e = np.where(z, np.exp(s - s.max(axis=1, keepdims=True)), 0.0)
            out[b, :, h] = e / np.maximum(e.sum(axis=1, keepdims=True), 1e-300) @ v[b, :, h]
    return out


def _mut_no_rescale(q, k, v, scale, causal, wl, p, seed, offset):
    """Mistake: kept probabilities not divided by 1 - p."""
    o, _ = attention_ref(q, k, v, scale, causal, wl, dropout_p=p, seed=seed, offset=offset)
    return o * (1 - p)


def _mut_swapped_halves(q, k, v, scale, causal, wl, p, seed, offset):
    """Mistake: the high 16-bit half used for even keys."""
    B, n_q, H, D = q.shape
    _, _, probs = attention_ref(q, k, v, scale, causal, wl, return_probs=True)
    out = np.zeros_like(q)
    for b in range(B):
        for h in range(H):
            z = dropout_keep(seed, offset, b, h, H, np.arange(n_q), k.shape[1] + 1, p)
            n = k.shape[1]
            zs = np.empty((n_q, n), dtype=bool)
            idx = np.arange(n) ^ 1
            ok = idx < z.shape[1]
            zs[:, ok] = z[:, idx[ok]]
            out[b, :, h] = (zs * probs[b, h] / (1 - p)) @ v[b, :, h]
    return out


def _dropout_pins(fn):
    # the brute force and the constant-V closed form, through a forward-only function
    q, k, v = _rand((1, 9, 2, 3), 20), _rand((1, 9, 2, 3), 21), _rand((1, 9, 2, 3), 22)
    o = fn(q, k, v, 0.8, True, -1, 0.3, 5, 2)
    ob, _ = attention_bruteforce(q.tolist(), k.tolist(), v.tolist(), 0.8, True, -1, dropout_p=0.3, seed=5, offset=2)
    assert np.allclose(o, np.array(ob), atol=1e-12)
    c = np.array([1.0, -1.0, 2.0])
    vc = np.broadcast_to(c, v.shape).copy()
    _, _, probs = attention_ref(q, k, vc, 0.8, True, -1, return_probs=True)
    oc = fn(q, k, vc, 0.8, True, -1, 0.3, 5, 2)
    z = dropout_keep(5, 2, 0, 0, 2, np.arange(9), 9, 0.3)
    assert np.allclose(oc[0, :, 0], ((z * probs[0, 0]).sum(axis=1) / 0.7)[:, None] * c, atol=1e-12)


@pytest.mark.parametrize("mut", [_mut_normalise_after_drop, _mut_no_rescale, _mut_swapped_halves])
def test_planted_dropout_mistake_is_caught(mut):
    with pytest.raises(AssertionError):
        _dropout_pins(mut)


def test_dropout_pin_harness_accepts_the_oracle():
    _dropout_pins(lambda q, k, v, s, c, w, p, seed, off: attention_ref(q, k, v, s, c, w, dropout_p=p, seed=seed,
                                                                         offset=off)[0])


# ----------------------------------------------------------------- backward

def _fd_grads(q, k, v, do, scale, causal, wl, p, seed, offset, eps=1e-6):
    """Central differences of L = sum(dO * O(q, k, v)) through the dropout forward
    (the keep bits do not depend on q, k, v, so L is smooth in them)."""
    def loss(q_, k_, v_):
        o, _ = attention_ref(q_, k_, v_, scale, causal, wl, dropout_p=p, seed=seed, offset=offset)
        return float(np.sum(do * o))
    grads = []
    for which in range(3):
        args = [q.copy(), k.copy(), v.copy()]
        g = np.zeros_like(args[which])
        it = np.nditer(g, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            plus = [a.copy() for a in args]
            minus = [a.copy() for a in args]
            plus[which][idx] += eps
            minus[which][idx] -= eps
            g[idx] = (loss(*plus) - loss(*minus)) / (2 * eps)
        grads.append(g)
    return grads


def _bwd_fd_pin(fn):
    for (n_q, n_k, H, h_kv, D, causal, wl) in [(5, 6, 2, 1, 3, False, -1), (7, 7, 2, 2, 2, True, -1),
                                              (6, 6, 1, 1, 3, True, 2)]:
        q, k, v = _rand((1, n_q, H, D), 30 + n_q), _rand((1, n_k, h_kv, D), 31), _rand((1, n_k, h_kv, D), 32)
        do = _rand((1, n_q, H, D), 33)
        got = fn(q, k, v, do, 0.7, causal, wl, 0.35, 17, 3)
        want = _fd_grads(q, k, v, do, 0.7, causal, wl, 0.35, 17, 3)
        for g, w in zip(got, want):
            assert np.allclose(g, w, rtol=1e-6, atol=1e-7), float(np.max(np.abs(g - w)))


def test_dropout_backward_matches_finite_differences():
    _bwd_fd_pin(lambda q, k, v, do, s, c, w, p, seed, off: attention_backward_ref(
        q, k, v, do, s, c, w, dropout_p=p, seed=seed, offset=off))


def test_planted_dropout_backward_mistake_is_caught():
    """Mistake: the keep bits applied to dV but not to dP."""
    def mutant(q, k, v, do, s, c, w, p, seed, off):
        dq, dk, dv = attention_backward_ref(q, k, v, do, s, c, w)
        _, _, dv_drop = attention_backward_ref(q, k, v, do, s, c, w, dropout_p=p, seed=seed, offset=off)
        return dq, dk, dv_drop
    with pytest.raises(AssertionError):
        _bwd_fd_pin(mutant)
