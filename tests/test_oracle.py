"""Pins for the fp64 oracle, independent of the oracle's own code.

Each check fixes the oracle against something other than itself: a
pure-Python brute force written separately, closed forms (constant V, Q = 0,
causal row 0, a two-key window, one-hot scores), invariants (row sums, shift
and key-permutation invariance), scipy's softmax / logsumexp, and the literal
window rule "i - w <= j <= i".  The last tests plant plausible mistakes in the
oracle (on the CPU) and require that at least one pin catches each of them.
"""

import json
import math
import os

import numpy as np
import pytest
import scipy.special

import oracle.attention as oa
from oracle import attention_bruteforce, attention_ref, visibility

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pages_values.json")
MODES = [(False, -1), (True, -1), (True, 0), (True, 1), (True, 3), (False, 2), (True, 100)]


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


# --------------------------------------------------------------------------
# pin functions: each takes an attention function with attention_ref's
# signature and raises AssertionError when it disagrees with the pin
# --------------------------------------------------------------------------

def pin_bruteforce(fn):
    for (n_q, n_k, D) in [(1, 1, 1), (2, 2, 4), (3, 3, 8), (7, 7, 4), (17, 17, 8), (5, 9, 4), (9, 5, 4)]:
        for causal, wl in MODES:
            q = _rand((2, n_q, 2, D), 10 + n_q)
            k = _rand((2, n_k, 2, D), 20 + n_k)
            v = _rand((2, n_k, 2, D), 30 + D)
            scale = 0.37
            o, l = fn(q, k, v, scale, causal, wl)
            ob, lb = attention_bruteforce(q.tolist(), k.tolist(), v.tolist(), scale, causal, wl)
            np.testing.assert_allclose(o, np.array(ob), rtol=0, atol=1e-12)
            lb = np.array(lb)
            assert np.array_equal(np.isinf(l), np.isinf(lb))
            fin = np.isfinite(lb)
            np.testing.assert_allclose(l[fin], lb[fin], rtol=0, atol=1e-12)


def pin_constant_v(fn):
    q, k = _rand((1, 33, 3, 8), 1), _rand((1, 33, 3, 8), 2)
    row = _rand((8,), 3)
    v = np.broadcast_to(row, (1, 33, 3, 8)).copy()
    for causal, wl in MODES:
        o, _ = fn(q, k, v, 0.9, causal, wl)
        np.testing.assert_allclose(o, np.broadcast_to(row, o.shape), rtol=0, atol=1e-12)


def pin_zero_query_mean(fn):
    n = 40
    k, v = _rand((2, n, 2, 4), 4), _rand((2, n, 2, 4), 5)
    q = np.zeros((2, n, 2, 4))
    for causal, wl in MODES:
        o, l = fn(q, k, v, 1.3, causal, wl)
        for i in range(n):
            lo = 0 if wl < 0 else max(0, i - wl)
            hi = i if causal else n - 1
            mean = v[:, lo:hi + 1].mean(axis=1)
            np.testing.assert_allclose(o[:, i], mean, rtol=0, atol=1e-12)
            np.testing.assert_allclose(l[:, :, i], math.log(hi - lo + 1), rtol=0, atol=1e-12)


def pin_scale_zero_mean(fn):
    n = 24
    q, k, v = _rand((1, n, 2, 4), 6), _rand((1, n, 2, 4), 7), _rand((1, n, 2, 4), 8)
    o, l = fn(q, k, v, 0.0, True, -1)
    for i in range(n):
        np.testing.assert_allclose(o[:, i], v[:, :i + 1].mean(axis=1), rtol=0, atol=1e-12)
        np.testing.assert_allclose(l[:, :, i], math.log(i + 1), rtol=0, atol=1e-12)


def pin_causal_row0(fn):
    q, k, v = _rand((2, 16, 3, 8), 9), _rand((2, 16, 3, 8), 10), _rand((2, 16, 3, 8), 11)
    scale = 0.25
    o, l = fn(q, k, v, scale, True, -1)
    np.testing.assert_allclose(o[:, 0], v[:, 0], rtol=0, atol=1e-12)
    dot0 = np.einsum("bhd,bhd->bh", q[:, 0], k[:, 0])
    np.testing.assert_allclose(l[:, :, 0], scale * dot0, rtol=0, atol=1e-12)


def pin_window_zero(fn):
    """causal with a left window of 0: each query sees only its own key."""
    q, k, v = _rand((1, 20, 2, 8), 12), _rand((1, 20, 2, 8), 13), _rand((1, 20, 2, 8), 14)
    scale = 0.5
    o, l = fn(q, k, v, scale, True, 0)
    np.testing.assert_allclose(o, v, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l, scale * np.einsum("bnhd,bnhd->bhn", q, k), rtol=0, atol=1e-12)


def pin_two_key_window(fn):
    """causal, window 1: query i >= 1 sees keys i-1 and i; closed-form sigmoid weights."""
    q, k, v = _rand((1, 12, 1, 4), 15), _rand((1, 12, 1, 4), 16), _rand((1, 12, 1, 4), 17)
    scale = 0.7
    o, l = fn(q, k, v, scale, True, 1)
    for i in range(1, 12):
        a = scale * float(q[0, i, 0] @ k[0, i, 0])
        b = scale * float(q[0, i, 0] @ k[0, i - 1, 0])
        w_self = 1.0 / (1.0 + math.exp(b - a))
        expect = w_self * v[0, i, 0] + (1.0 - w_self) * v[0, i - 1, 0]
        np.testing.assert_allclose(o[0, i, 0], expect, rtol=0, atol=1e-12)
        np.testing.assert_allclose(l[0, 0, i], math.log(math.exp(a) + math.exp(b)), rtol=0, atol=1e-12)


def pin_scipy(fn):
    """softmax weights and LSE against scipy.special on the full score matrix."""
    q, k, v = _rand((1, 30, 2, 6), 18), _rand((1, 30, 2, 6), 19), _rand((1, 30, 2, 6), 20)
    scale = 0.8
    for causal, wl in MODES:
        o, l = fn(q, k, v, scale, causal, wl)
        for h in range(2):
            s = scale * np.einsum("id,jd->ij", q[0, :, h], k[0, :, h])
            i = np.arange(30)[:, None]
            j = np.arange(30)[None, :]
            keep = np.ones((30, 30), bool)
            if causal:
                keep &= ~(j > i)
            if wl >= 0:
                keep &= ~(i - j > wl)
            s = np.where(keep, s, -np.inf)
            p = scipy.special.softmax(s, axis=1)
            np.testing.assert_allclose(o[0, :, h], p @ v[0, :, h], rtol=0, atol=1e-12)
            np.testing.assert_allclose(l[0, h], scipy.special.logsumexp(s, axis=1), rtol=0, atol=1e-12)


def pin_shift_invariance(fn):
    """A constant added to every score of a row leaves O and moves LSE by it."""
    q, k, v = _rand((1, 25, 2, 5), 21), _rand((1, 25, 2, 5), 22), _rand((1, 25, 2, 5), 23)
    c, scale = 3.25, 0.6
    q2 = np.concatenate([q, np.ones((1, 25, 2, 1))], axis=-1)
    k2 = np.concatenate([k, np.full((1, 25, 2, 1), c)], axis=-1)
    for causal, wl in MODES:
        o1, l1 = fn(q, k, v, scale, causal, wl)
        v2 = np.concatenate([v, np.zeros((1, 25, 2, 1))], axis=-1)  # values padded with 0
        o2, l2 = fn(q2, k2, v2, scale, causal, wl)
        np.testing.assert_allclose(o2[..., :5], o1, rtol=0, atol=1e-12)
        assert np.all(o2[..., 5] == 0.0)
        np.testing.assert_allclose(l2, l1 + scale * c, rtol=0, atol=1e-12)


def pin_key_permutation(fn):
    q, k, v = _rand((1, 19, 2, 4), 24), _rand((1, 31, 2, 4), 25), _rand((1, 31, 2, 4), 26)
    perm = np.random.default_rng(27).permutation(31)
    o1, l1 = fn(q, k, v, 0.45, False, -1)
    o2, l2 = fn(q, k[:, perm], v[:, perm], 0.45, False, -1)
    np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l2, l1, rtol=0, atol=1e-12)


def pin_wide_window_is_causal(fn):
    q, k, v = _rand((1, 37, 2, 4), 28), _rand((1, 37, 2, 4), 29), _rand((1, 37, 2, 4), 30)
    o1, l1 = fn(q, k, v, 0.5, True, -1)
    for wl in (36, 37, 1000):
        o2, l2 = fn(q, k, v, 0.5, True, wl)
        np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-12)
        np.testing.assert_allclose(l2, l1, rtol=0, atol=1e-12)


def pin_one_hot_large_scores(fn):
    """Q = K = 30 * identity rows: score 900 on the diagonal, 0 elsewhere; no overflow."""
    n = 16
    eye = np.zeros((1, n, 1, n))
    for i in range(n):
        eye[0, i, 0, i] = 30.0
    v = _rand((1, n, 1, n), 31)
    o, l = fn(eye, eye, v, 1.0, False, -1)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(l))
    np.testing.assert_allclose(o, v, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l, 900.0, rtol=0, atol=1e-12)


def pin_empty_rows(fn):
    """With N_q > N_k + w, late queries see no key: O = 0, LSE = -inf."""
    q, k, v = _rand((1, 12, 1, 4), 32), _rand((1, 4, 1, 4), 33), _rand((1, 4, 1, 4), 34)
    o, l = fn(q, k, v, 1.0, True, 2)
    # query i sees keys max(0, i-2) .. min(i, 3); empty once i - 2 > 3
    for i in range(12):
        if i - 2 > 3:
            assert np.all(o[0, i] == 0.0) and l[0, 0, i] == -np.inf
        else:
            assert np.isfinite(l[0, 0, i])


PINS = [pin_bruteforce, pin_constant_v, pin_zero_query_mean, pin_scale_zero_mean, pin_causal_row0,
        pin_window_zero, pin_two_key_window, pin_scipy, pin_shift_invariance, pin_key_permutation,
        pin_wide_window_is_causal, pin_one_hot_large_scores, pin_empty_rows]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_oracle_pin(pin):
    pin(attention_ref)


def test_rows_sum_to_one_and_nonnegative():
    q, k, v = _rand((2, 29, 2, 4), 40), _rand((2, 29, 2, 4), 41), _rand((2, 29, 2, 4), 42)
    for causal, wl in MODES:
        _, _, p = attention_ref(q, k, v, 1.1, causal, wl, return_probs=True)
        assert np.all(p >= 0)
        np.testing.assert_allclose(p.sum(axis=-1), 1.0, rtol=0, atol=1e-12)
        vis = visibility(np.arange(29), 29, causal, wl)
        assert np.all(p[..., ~vis] == 0)


def test_sampled_rows_match_full():
    q, k, v = _rand((1, 50, 2, 4), 43), _rand((1, 50, 2, 4), 44), _rand((1, 50, 2, 4), 45)
    rows = np.array([0, 3, 17, 49])
    o, l = attention_ref(q, k, v, 0.3, True, 5)
    os_, ls = attention_ref(q, k, v, 0.3, True, 5, rows=rows)
    np.testing.assert_array_equal(os_, o[:, rows])
    np.testing.assert_array_equal(ls, l[:, :, rows])


def test_visibility_literal_window_rule():
    """The sliding-window workload's rule, written literally: visible iff i - w <= j <= i."""
    rng = np.random.default_rng(46)
    for _ in range(200):
        n = int(rng.integers(1, 60))
        w = int(rng.integers(0, 70))
        vis = visibility(np.arange(n), n, True, w)
        for i in range(n):
            for j in range(n):
                assert vis[i, j] == (i - w <= j <= i)


def test_pages_auto_scale_reading():
    """The pages divide D=64 scores by 8.0 and call the default 'auto-scale'; 1/sqrt(64) == 1/8."""
    g = json.load(open(GOLDEN))
    acc = g["accuracy_check"]
    assert 1.0 / math.sqrt(acc["headdim"]) == 1.0 / acc["score_divisor"]
    assert g["no_window"]["window_size"] == [-1, -1]


# --------------------------------------------------------------------------
# planted mistakes: each plausible slip in the oracle must fail >= 1 pin
# --------------------------------------------------------------------------

def _caught(fn):
    for pin in PINS:
        try:
            pin(fn)
        except AssertionError:
            return True
    return False


def _mut_dropped_scale(q, k, v, scale, causal=False, wl=-1, **kw):
    return attention_ref(q, k, v, 1.0, causal, wl, **kw)


def _mut_swapped_kv(q, k, v, scale, causal=False, wl=-1, **kw):
    return attention_ref(q, v, k, scale, causal, wl, **kw)


def _mut_log2_lse(q, k, v, scale, causal=False, wl=-1, **kw):
    o, l = attention_ref(q, k, v, scale, causal, wl, **kw)
    return o, l / math.log(2.0)


def _mut_unnormalised(q, k, v, scale, causal=False, wl=-1, **kw):
    o, l = attention_ref(q, k, v, scale, causal, wl, **kw)
    return o * 1.0001, l


def _mut_transposed_heads(q, k, v, scale, causal=False, wl=-1, **kw):
    # k read with batch and head roles crossed
    return attention_ref(q, np.ascontiguousarray(k[:, :, ::-1]), v, scale, causal, wl, **kw)


def _mut_negated_scores(q, k, v, scale, causal=False, wl=-1, **kw):
    return attention_ref(q, k, v, -scale, causal, wl, **kw)


@pytest.mark.parametrize("mut", [_mut_dropped_scale, _mut_swapped_kv, _mut_log2_lse,
                                 _mut_unnormalised, _mut_transposed_heads, _mut_negated_scores])
def test_planted_mistake_is_caught(mut):
    assert _caught(mut)


@pytest.mark.parametrize("bad", ["strict_causal", "window_off_by_one", "window_ignored", "causal_ignored"])
def test_planted_mask_mistake_is_caught(monkeypatch, bad):
    def mutated(rows, n_k, causal, window_left, window_right=-1):
        i = np.asarray(rows, dtype=np.int64)[:, None]
        j = np.arange(n_k)[None, :]
        vis = np.ones((i.shape[0], n_k), bool)
        if causal and bad != "causal_ignored":
            vis &= (j < i) if bad == "strict_causal" else (j <= i)
        if window_left >= 0 and bad != "window_ignored":
            vis &= (j > i - window_left) if bad == "window_off_by_one" else (j >= i - window_left)
        if window_right >= 0:
            vis &= j <= i + window_right
        return vis

    monkeypatch.setattr(oa, "visibility", mutated)
    assert _caught(oa.attention_ref)


# --------------------------------------------------------------------------
# grouped / multi-query K/V heads (H_kv < H): query head h reads K/V head
# h // (H / H_kv), the reading of "shared K/V across heads" stated in the
# oracle's docstring
# --------------------------------------------------------------------------

def gqa_pin_bruteforce(fn):
    """Against the brute force, whose head map is written as h * H_kv // H."""
    for (H, h_kv) in [(4, 1), (4, 2), (6, 3), (6, 2)]:
        for causal, wl in MODES[:5]:
            q = _rand((1, 7, H, 4), 60 + H)
            k = _rand((1, 9, h_kv, 4), 61 + h_kv)
            v = _rand((1, 9, h_kv, 4), 62 + h_kv)
            o, l = fn(q, k, v, 0.7, causal, wl)
            ob, lb = attention_bruteforce(q.tolist(), k.tolist(), v.tolist(), 0.7, causal, wl)
            np.testing.assert_allclose(o, np.array(ob), rtol=0, atol=1e-12)
            np.testing.assert_allclose(l, np.array(lb), rtol=0, atol=1e-12)


def gqa_pin_constant_v_per_group(fn):
    """V constant over keys and dims within each K/V head, different across heads:
    every visible row of query head h returns K/V head h // (H / H_kv)'s constant."""
    H, h_kv = 8, 4
    q, k = _rand((2, 11, H, 8), 63), _rand((2, 11, h_kv, 8), 64)
    consts = np.array([1.5, -2.0, 0.25, 7.0])
    v = np.broadcast_to(consts[None, None, :, None], (2, 11, h_kv, 8)).copy()
    for causal, wl in [(False, -1), (True, -1), (True, 2)]:
        o, _ = fn(q, k, v, 0.9, causal, wl)
        for h in range(H):
            np.testing.assert_allclose(o[:, :, h, :], consts[h // 2], rtol=0, atol=1e-12)


def gqa_pin_repeated_heads(fn):
    """Sharing a K/V head equals giving each query head its own copy of it (numpy repeat)."""
    H, h_kv = 6, 2
    q, k, v = _rand((2, 13, H, 4), 65), _rand((2, 13, h_kv, 4), 66), _rand((2, 13, h_kv, 4), 67)
    for causal, wl in MODES[:4]:
        o, l = fn(q, k, v, 0.8, causal, wl)
        o2, l2 = fn(q, np.repeat(k, H // h_kv, axis=2), np.repeat(v, H // h_kv, axis=2), 0.8, causal, wl)
        np.testing.assert_allclose(o, o2, rtol=0, atol=1e-13)
        np.testing.assert_allclose(l, l2, rtol=0, atol=1e-13)


def gqa_pin_mqa_zero_query(fn):
    """Multi-query (H_kv = 1) with Q = 0: every head returns the mean of the single V head's
    visible rows and LSE = ln(#visible keys)."""
    q = np.zeros((1, 9, 4, 4))
    k, v = _rand((1, 9, 1, 4), 68), _rand((1, 9, 1, 4), 69)
    o, l = fn(q, k, v, 1.3, True, 3)
    for i in range(9):
        lo = max(0, i - 3)
        for h in range(4):
            np.testing.assert_allclose(o[0, i, h], v[0, lo:i + 1, 0].mean(axis=0), rtol=0, atol=1e-12)
            np.testing.assert_allclose(l[0, h, i], math.log(i - lo + 1), rtol=0, atol=1e-12)


GQA_PINS = [gqa_pin_bruteforce, gqa_pin_constant_v_per_group, gqa_pin_repeated_heads, gqa_pin_mqa_zero_query]


@pytest.mark.parametrize("pin", GQA_PINS, ids=[p.__name__ for p in GQA_PINS])
def test_oracle_gqa_pin(pin):
    pin(attention_ref)


def test_oracle_rejects_uneven_head_groups():
    q, k = _rand((1, 4, 6, 4), 70), _rand((1, 4, 4, 4), 71)
    with pytest.raises(ValueError):
        attention_ref(q, k, k, 1.0)


def test_planted_head_map_mistake_is_caught():
    """An oracle that maps query head h to K/V head h mod H_kv (interleaved groups) fails a pin."""
    def mutated(q, k, v, scale, causal=False, wl=-1, **kw):
        H, h_kv = q.shape[2], k.shape[2]
        idx = np.arange(H) % h_kv
        return attention_ref(q, k[:, :, idx], v[:, :, idx], scale, causal, wl, **kw)

    caught = False
    for pin in GQA_PINS:
        try:
            pin(mutated)
        except AssertionError:
            caught = True
    assert caught


# --------------------------------------------------------------------------
# attention mask (boolean: attend where True; real: added to scale * q.k),
# broadcast over batch / heads
# --------------------------------------------------------------------------

def _bool_mask(shape, seed):
    m = np.random.default_rng(seed).random(shape) > 0.35
    return m


def mask_pin_bruteforce(fn):
    """Against the brute force for boolean and additive masks, broadcast and not."""
    q, k, v = _rand((2, 7, 2, 4), 90), _rand((2, 9, 2, 4), 91), _rand((2, 9, 2, 4), 92)
    masks = [_bool_mask((2, 2, 7, 9), 93), _bool_mask((1, 2, 7, 9), 94), _rand((2, 1, 7, 9), 95),
             np.where(_bool_mask((1, 1, 7, 9), 96), _rand((1, 1, 7, 9), 97), -np.inf)]
    for m in masks:
        for causal, wl in [(False, -1), (True, -1), (True, 2)]:
            o, l = fn(q, k, v, 0.6, causal, wl, mask=m)
            ob, lb = attention_bruteforce(q.tolist(), k.tolist(), v.tolist(), 0.6, causal, wl, mask=m.tolist())
            np.testing.assert_allclose(o, np.array(ob), rtol=0, atol=1e-12)
            np.testing.assert_allclose(l, np.array(lb), rtol=0, atol=1e-12)


def mask_pin_zero_query(fn):
    """Q = 0: the scores are the additive mask alone, so O = softmax(mask) V and
    LSE = logsumexp(mask) (scipy) -- also fixes that the mask is added after scaling."""
    q = np.zeros((1, 6, 1, 4))
    k, v = _rand((1, 11, 1, 4), 98), _rand((1, 11, 1, 4), 99)
    m = 3.0 * _rand((1, 1, 6, 11), 100)
    o, l = fn(q, k, v, 0.37, False, -1, mask=m)
    p = scipy.special.softmax(m[0, 0], axis=-1)
    np.testing.assert_allclose(o[0, :, 0], p @ v[0, :, 0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(l[0, 0], scipy.special.logsumexp(m[0, 0], axis=-1), rtol=0, atol=1e-12)


def mask_pin_causal_pattern(fn):
    """A boolean mask holding the causal pattern (and an additive one holding -inf above the
    diagonal) is causal attention."""
    q, k, v = _rand((1, 13, 2, 4), 101), _rand((1, 13, 2, 4), 102), _rand((1, 13, 2, 4), 103)
    tri = np.tril(np.ones((13, 13), dtype=bool))[None, None]
    o_c, l_c = fn(q, k, v, 0.5, True, -1)
    o_b, l_b = fn(q, k, v, 0.5, False, -1, mask=tri)
    o_a, l_a = fn(q, k, v, 0.5, False, -1, mask=np.where(tri, 0.0, -np.inf))
    for o, l in [(o_b, l_b), (o_a, l_a)]:
        np.testing.assert_allclose(o, o_c, rtol=0, atol=1e-13)
        np.testing.assert_allclose(l, l_c, rtol=0, atol=1e-13)


def mask_pin_row_constant(fn):
    """Adding a per-row constant c_i to every score of row i leaves O and moves LSE by c_i."""
    q, k, v = _rand((1, 8, 1, 4), 104), _rand((1, 8, 1, 4), 105), _rand((1, 8, 1, 4), 106)
    c = np.linspace(-2.0, 5.0, 8)
    m = np.broadcast_to(c[None, None, :, None], (1, 1, 8, 8))
    o0, l0 = fn(q, k, v, 0.8, True, -1)
    o1, l1 = fn(q, k, v, 0.8, True, -1, mask=m)
    np.testing.assert_allclose(o1, o0, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l1[0, 0], l0[0, 0] + c, rtol=0, atol=1e-12)


MASK_PINS = [mask_pin_bruteforce, mask_pin_zero_query, mask_pin_causal_pattern, mask_pin_row_constant]


@pytest.mark.parametrize("pin", MASK_PINS, ids=[p.__name__ for p in MASK_PINS])
def test_oracle_mask_pin(pin):
    pin(attention_ref)


def test_fully_masked_rows_are_empty():
    q, k, v = _rand((1, 4, 1, 4), 107), _rand((1, 5, 1, 4), 108), _rand((1, 5, 1, 4), 109)
    m = np.ones((1, 1, 4, 5), dtype=bool)
    m[0, 0, 2] = False
    o, l = attention_ref(q, k, v, 1.0, mask=m)
    assert np.all(o[0, 2] == 0.0) and l[0, 0, 2] == -np.inf and np.all(np.isfinite(l[0, 0, [0, 1, 3]]))


@pytest.mark.parametrize("bad", ["before_scale", "inverted", "transposed"])
def test_planted_mask_application_mistake_is_caught(bad):
    def mutated(q, k, v, scale, causal=False, wl=-1, mask=None, **kw):
        if mask is None:
            return attention_ref(q, k, v, scale, causal, wl, mask=mask, **kw)
        m = np.asarray(mask)
        if bad == "before_scale" and m.dtype != np.bool_:
            m = m / scale            # the mask scaled along with the scores
        elif bad == "inverted" and m.dtype == np.bool_:
            m = ~m
        elif bad == "transposed" and m.shape[2] == m.shape[3]:
            m = np.swapaxes(m, 2, 3)
        return attention_ref(q, k, v, scale, causal, wl, mask=m, **kw)

    caught = False
    for pin in MASK_PINS:
        try:
            pin(mutated)
        except AssertionError:
            caught = True
    assert caught


# --------------------------------------------------------------------------
# backward: pins for attention_backward_ref.  Each pin takes a function with
# its signature; the finite-difference pin uses only the forward oracle.
# --------------------------------------------------------------------------

BWD_MODES = [(False, -1), (True, -1), (True, 1), (False, 2)]


def _fd_grads(q, k, v, do, scale, causal, wl, eps=1e-6):
    """Central differences of L = sum(dO * O(q, k, v)) through attention_ref."""
    def loss(q_, k_, v_):
        o, _ = attention_ref(q_, k_, v_, scale, causal, wl)
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


def pin_backward_finite_differences(fn):
    for (n_q, n_k, H, h_kv, D) in [(5, 5, 2, 2, 3), (7, 4, 2, 1, 4), (3, 8, 4, 2, 2)]:
        for causal, wl in BWD_MODES:
            q = _rand((1, n_q, H, D), 300 + n_q)
            k = _rand((1, n_k, h_kv, D), 310 + n_k)
            v = _rand((1, n_k, h_kv, D), 320 + D)
            do = _rand((1, n_q, H, D), 330 + H)
            got = fn(q, k, v, do, 0.6, causal, wl)
            want = _fd_grads(q, k, v, do, 0.6, causal, wl)
            for g, w in zip(got, want):
                assert np.allclose(g, w, rtol=1e-6, atol=1e-7), float(np.max(np.abs(g - w)))


def pin_backward_key_shift_invariance(fn):
    # adding one vector to every key moves each query's scores by a constant:
    # O does not change, so the key gradients of each head sum to zero
    for causal, wl in BWD_MODES:
        q = _rand((2, 9, 2, 4), 340)
        k = _rand((2, 9, 2, 4), 341)
        v = _rand((2, 9, 2, 4), 342)
        do = _rand((2, 9, 2, 4), 343)
        _, dk, _ = fn(q, k, v, do, 0.8, causal, wl)
        assert np.allclose(dk.sum(axis=1), 0.0, atol=1e-12)


def pin_backward_uniform_attention(fn):
    # Q = 0: every visible key of row i has weight 1 / n_i, so
    # dV_j = sum over the rows that see key j of dO_i / n_i
    for causal, wl in BWD_MODES:
        n, D = 8, 3
        q = np.zeros((1, n, 1, D))
        k = _rand((1, n, 1, D), 350)
        v = _rand((1, n, 1, D), 351)
        do = _rand((1, n, 1, D), 352)
        _, _, dv = fn(q, k, v, do, 1.3, causal, wl)
        want = np.zeros((n, D))
        for i in range(n):
            seen = [j for j in range(n) if (not causal or j <= i) and (wl < 0 or j >= i - wl)]
            for j in seen:
                want[j] += do[0, i, 0] / len(seen)
        assert np.allclose(dv[0, :, 0], want, atol=1e-13)


def pin_backward_value_linearity(fn):
    # O is linear in V with weights P: for dO = 1 in one column, dV's column
    # is the column sums of P
    for causal, wl in BWD_MODES:
        q = _rand((1, 6, 1, 2), 360)
        k = _rand((1, 6, 1, 2), 361)
        v = _rand((1, 6, 1, 2), 362)
        do = np.zeros((1, 6, 1, 2))
        do[..., 1] = 1.0
        _, _, p = attention_ref(q, k, v, 0.9, causal, wl, return_probs=True)
        _, _, dv = fn(q, k, v, do, 0.9, causal, wl)
        assert np.allclose(dv[0, :, 0, 1], p[0, 0].sum(axis=0), atol=1e-13)
        assert np.allclose(dv[0, :, 0, 0], 0.0, atol=1e-15)


BWD_PINS = [pin_backward_finite_differences, pin_backward_key_shift_invariance, pin_backward_uniform_attention,
            pin_backward_value_linearity]


@pytest.mark.parametrize("pin", BWD_PINS)
def test_oracle_backward_pin(pin):
    pin(oa.attention_backward_ref)


def _bwd_mutant(kind):
    """attention_backward_ref with one plausible mistake planted."""
    def fn(q, k, v, do, scale, causal, wl):
        B, n_q, H, D = q.shape
        h_kv = k.shape[2]
        _, _, probs = attention_ref(q, k, v, scale, causal, wl, return_probs=True)
        dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
        for b in range(B):
            for h in range(H):
                hk = h // (H // h_kv)
                p, g = probs[b, h], do[b, :, h, :]
                dv[b, :, hk, :] += (p if kind == "dv_untransposed" and n_q == p.shape[1] else p.T) @ g
                dp = g @ v[b, :, hk, :].T
                row = (p * dp).sum(axis=1, keepdims=True)
                ds = p * dp if kind == "no_row_term" else p * (dp - row)
                if kind == "sign":
                    ds = -ds
                s = 1.0 if kind == "no_scale" else scale
                dq[b, :, h, :] = s * (ds @ k[b, :, hk, :])
                dk_h = s * (ds.T @ q[b, :, h, :])
                if kind == "last_group_head_only":
                    dk[b, :, hk, :] = dk_h
                else:
                    dk[b, :, hk, :] += dk_h
        return dq, dk, dv
    return fn


@pytest.mark.parametrize("kind", ["no_row_term", "sign", "no_scale", "last_group_head_only", "dv_untransposed"])
def test_planted_backward_mistake_is_caught(kind):
    caught = False
    for pin in BWD_PINS:
        try:
            pin(_bwd_mutant(kind))
        except AssertionError:
            caught = True
    assert caught, kind


def test_backward_mutant_harness_without_mistake_passes():
    for pin in BWD_PINS:
        pin(_bwd_mutant("none"))
