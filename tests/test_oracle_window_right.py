"""Pins for the oracle's right window (keys at most w positions after the query).

The pages' sliding-window example passes ``window_size=(256, 256)``, up to
256 keys on each side of the query (Flash Attention | Hermes Skill,
Workflow 2, Step 3).  Each check fixes ``attention_ref`` /
``attention_backward_ref`` with a right window against something other than
their own code: the separately written brute force, the literal rule
"i - l <= j <= i + r", the special cases r = 0 (causal) and r >= N (no
bound), the mirror symmetry that reverses both sequences and swaps the two
windows, a Q = 0 closed form, and finite differences through the forward.
A planted mistake (the right bound off by one, or ignored) must be caught.
"""

import numpy as np
import pytest

import oracle.attention as oa
from oracle import attention_backward_ref, attention_bruteforce, attention_ref, visibility

WINDOWS = [(-1, 0), (-1, 1), (-1, 3), (2, 2), (0, 5), (4, 0), (1, 100), (-1, -1)]


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def pin_bruteforce(fn):
    for (n_q, n_k, D) in [(1, 1, 2), (3, 3, 4), (7, 7, 4), (17, 17, 8), (5, 9, 4), (9, 5, 4)]:
        for wl, wr in WINDOWS:
            q, k, v = _rand((1, n_q, 2, D), 500 + n_q), _rand((1, n_k, 2, D), 510 + n_k), _rand((1, n_k, 2, D), 520)
            o, l = fn(q, k, v, 0.41, False, wl, window_right=wr)
            ob, lb = attention_bruteforce(q.tolist(), k.tolist(), v.tolist(), 0.41, False, wl, window_right=wr)
            np.testing.assert_allclose(o, np.array(ob), rtol=0, atol=1e-12)
            lb = np.array(lb)
            assert np.array_equal(np.isinf(l), np.isinf(lb))
            fin = np.isfinite(lb)
            np.testing.assert_allclose(l[fin], lb[fin], rtol=0, atol=1e-12)


def pin_right_zero_is_causal(fn):
    q, k, v = _rand((2, 13, 2, 4), 530), _rand((2, 13, 2, 4), 531), _rand((2, 13, 2, 4), 532)
    for wl in (-1, 0, 3):
        o1, l1 = fn(q, k, v, 0.7, False, wl, window_right=0)
        o2, l2 = fn(q, k, v, 0.7, True, wl)
        np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-13)
        np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-13)


def pin_wide_right_is_unbounded(fn):
    q, k, v = _rand((1, 11, 2, 4), 540), _rand((1, 11, 2, 4), 541), _rand((1, 11, 2, 4), 542)
    for wl in (-1, 2):
        o1, l1 = fn(q, k, v, 0.7, False, wl, window_right=11)
        o2, l2 = fn(q, k, v, 0.7, False, wl)
        np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-13)
        np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-13)


def pin_mirror_swaps_windows(fn):
    # reversing queries and keys maps "j >= i - l" to "j' <= i' + l": the
    # left and right windows trade places
    n = 15
    q, k, v = _rand((1, n, 2, 4), 550), _rand((1, n, 2, 4), 551), _rand((1, n, 2, 4), 552)
    rq, rk, rv = q[:, ::-1].copy(), k[:, ::-1].copy(), v[:, ::-1].copy()
    for wl, wr in [(2, 5), (0, 3), (6, 1), (-1, 4)]:
        o1, l1 = fn(q, k, v, 0.8, False, wl, window_right=wr)
        # a left bound of -1 is "no bound", which mirrors to no right bound
        o2, l2 = fn(rq, rk, rv, 0.8, False, wr, window_right=wl)
        np.testing.assert_allclose(o1, o2[:, ::-1], rtol=0, atol=1e-12)
        np.testing.assert_allclose(l1, l2[:, :, ::-1], rtol=0, atol=1e-12)


def pin_zero_query_mean(fn):
    # Q = 0: O_i is the mean of V over the keys max(0, i - l) .. min(N-1, i + r)
    n, D = 12, 3
    q = np.zeros((1, n, 1, D))
    k, v = _rand((1, n, 1, D), 560), _rand((1, n, 1, D), 561)
    for wl, wr in [(-1, 2), (1, 1), (3, 0), (0, 4)]:
        o, l = fn(q, k, v, 1.1, False, wl, window_right=wr)
        for i in range(n):
            lo = 0 if wl < 0 else max(0, i - wl)
            hi = n - 1 if wr < 0 else min(n - 1, i + wr)
            np.testing.assert_allclose(o[0, i, 0], v[0, lo:hi + 1, 0].mean(axis=0), rtol=0, atol=1e-13)
            assert abs(l[0, 0, i] - np.log(hi - lo + 1)) < 1e-13


PINS = [pin_bruteforce, pin_right_zero_is_causal, pin_wide_right_is_unbounded, pin_mirror_swaps_windows,
        pin_zero_query_mean]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_oracle_right_window_pin(pin):
    pin(attention_ref)


def test_visibility_literal_two_sided_rule():
    rng = np.random.default_rng(57)
    for _ in range(150):
        n_q, n_k = int(rng.integers(1, 40)), int(rng.integers(1, 40))
        wl, wr = int(rng.integers(-1, 45)), int(rng.integers(-1, 45))
        vis = visibility(np.arange(n_q), n_k, False, wl, wr)
        for i in range(n_q):
            for j in range(n_k):
                assert vis[i, j] == ((wl < 0 or j >= i - wl) and (wr < 0 or j <= i + wr))


@pytest.mark.parametrize("bad", ["off_by_one", "ignored"])
def test_planted_right_window_mistake_is_caught(monkeypatch, bad):
    real = oa.visibility

    def mutated(rows, n_k, causal, window_left, window_right=-1):
        if window_right >= 0:
            window_right = window_right + 1 if bad == "off_by_one" else -1
        return real(rows, n_k, causal, window_left, window_right)

    monkeypatch.setattr(oa, "visibility", mutated)
    caught = False
    for pin in PINS:
        try:
            pin(oa.attention_ref)
        except AssertionError:
            caught = True
    assert caught


def _fd_grads(q, k, v, do, scale, wl, wr, eps=1e-6):
    def loss(q_, k_, v_):
        o, _ = attention_ref(q_, k_, v_, scale, False, wl, window_right=wr)
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


def test_backward_right_window_matches_finite_differences():
    for (n_q, n_k, H, h_kv, D), (wl, wr) in zip([(6, 6, 2, 2, 3), (7, 5, 2, 1, 2), (4, 8, 2, 2, 2)],
                                                [(-1, 1), (2, 2), (0, 3)]):
        q, k = _rand((1, n_q, H, D), 570 + n_q), _rand((1, n_k, h_kv, D), 580 + n_k)
        v, do = _rand((1, n_k, h_kv, D), 590), _rand((1, n_q, H, D), 600)
        got = attention_backward_ref(q, k, v, do, 0.6, False, wl, window_right=wr)
        want = _fd_grads(q, k, v, do, 0.6, wl, wr)
        for g, w in zip(got, want):
            assert np.allclose(g, w, rtol=1e-6, atol=1e-7), float(np.max(np.abs(g - w)))


def test_right_window_with_dropout_reduces_to_causal_and_to_unbounded():
    """With dropout the right window still means j <= i + r: r = 0 gives the causal dropout forward and
    backward, r >= N_k the unbounded ones (the keep bits do not depend on the window)."""
    q, k, v = _rand((2, 9, 2, 4), 800), _rand((2, 9, 2, 4), 801), _rand((2, 9, 2, 4), 802)
    do = _rand((2, 9, 2, 4), 803)
    kw = dict(dropout_p=0.3, seed=12345, offset=7)
    for wl in (-1, 2):
        o1, l1 = attention_ref(q, k, v, 0.6, False, wl, window_right=0, **kw)
        o2, l2 = attention_ref(q, k, v, 0.6, True, wl, **kw)
        np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-13)
        np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-13)
        g1 = attention_backward_ref(q, k, v, do, 0.6, False, wl, window_right=0, **kw)
        g2 = attention_backward_ref(q, k, v, do, 0.6, True, wl, **kw)
        for a, b in zip(g1, g2):
            np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)
        o3, _ = attention_ref(q, k, v, 0.6, False, wl, window_right=9, **kw)
        o4, _ = attention_ref(q, k, v, 0.6, False, wl, **kw)
        np.testing.assert_allclose(o3, o4, rtol=0, atol=1e-13)
