"""Pin checks for an attention oracle, parameterised by implementation.

Each check takes an object with ``fwd(q, k, v, scale, causal) -> (O, LSE)``
and ``bwd(q, k, v, do, scale, causal) -> (dQ, dK, dV, c)`` on one head of
fp64 ``[N, d]`` arrays, and raises AssertionError when the implementation
disagrees with something the pages or the mathematics fix independently of
the implementation's own formula.  ``test_oracle_pins.py`` runs every check on
the C oracle and on the numpy twin, and runs them on deliberately broken
copies of the numpy twin to show that each plausible mistake is caught.
"""
from __future__ import annotations

import math

import numpy as np
from scipy.special import logsumexp, softmax


def _rng(seed):
    return np.random.default_rng(seed)


def _bf16_grid(a):
    """Round fp64 values to the bf16 grid (the inputs the GPU sees are bf16)."""
    import torch
    return torch.from_numpy(np.asarray(a, np.float64)).to(torch.bfloat16).to(torch.float64).numpy()


def check_library_softmax(impl, seed=0):
    """Brute force on tiny inputs against scipy's softmax and logsumexp."""
    rng = _rng(seed)
    for trial in range(12):
        n = int(rng.integers(1, 17))
        d = int(rng.integers(1, 9))
        causal = bool(trial % 2)
        scale = float(rng.uniform(0.1, 1.5))
        q, k, v = (_bf16_grid(rng.standard_normal((n, d))) for _ in range(3))
        o, lse = impl.fwd(q, k, v, scale, causal)
        for i in range(n):
            nv = i + 1 if causal else n
            s = np.array([scale * sum(q[i, x] * k[j, x] for x in range(d)) for j in range(nv)])
            p = softmax(s)
            o_ref = sum(p[j] * v[j] for j in range(nv))
            np.testing.assert_allclose(o[i], o_ref, rtol=0, atol=1e-12)
            np.testing.assert_allclose(lse[i], logsumexp(s), rtol=1e-13, atol=1e-13)


def check_n1_closed_form(impl):
    """N=1: the single key gets all the weight; O = v_0, LSE = S_00, dQ = dK = 0, dV = dO."""
    q = np.array([[1.0, 2.0]])
    k = np.array([[0.5, -1.0]])
    v = np.array([[3.0, -4.0]])
    do = np.array([[0.25, 1.5]])
    for causal in (False, True):
        o, lse = impl.fwd(q, k, v, 0.5, causal)
        assert np.array_equal(o, v), o
        assert lse[0] == 0.5 * (0.5 - 2.0), lse
        dq, dk, dv, _ = impl.bwd(q, k, v, do, 0.5, causal)
        assert np.allclose(dq, 0, atol=1e-15) and np.allclose(dk, 0, atol=1e-15), (dq, dk)
        np.testing.assert_allclose(dv, do, rtol=0, atol=1e-15)


def check_n2_logistic(impl):
    """N=2: P_i0 = sigma(S_i0 - S_i1) (logistic), LSE_i = S_i1 + ln(1 + e^(S_i0 - S_i1))."""
    q = np.array([[1.0], [2.0]])
    k = np.array([[1.0], [0.0]])
    v = np.array([[2.0], [6.0]])
    scale = 1.0
    o, lse = impl.fwd(q, k, v, scale, False)
    for i in range(2):
        a, b = scale * q[i, 0] * k[0, 0], scale * q[i, 0] * k[1, 0]
        sig = 1.0 / (1.0 + math.exp(-(a - b)))
        assert abs(o[i, 0] - (sig * 2.0 + (1 - sig) * 6.0)) < 1e-14
        assert abs(lse[i] - (b + math.log1p(math.exp(a - b)))) < 1e-14
    # causal: row 0 sees only key 0
    o, lse = impl.fwd(q, k, v, scale, True)
    assert o[0, 0] == 2.0 and lse[0] == 1.0
    a, b = 2.0, 0.0
    sig = 1.0 / (1.0 + math.exp(-(a - b)))
    assert abs(o[1, 0] - (sig * 2.0 + (1 - sig) * 6.0)) < 1e-14


def check_rows_sum_to_one(impl, seed=1):
    """A constant value column comes out unchanged, i.e. every row of P sums to 1."""
    rng = _rng(seed)
    n, d = 40, 6
    q, k, v = (_bf16_grid(rng.standard_normal((n, d))) for _ in range(3))
    v[:, 0] = 1.0
    for causal in (False, True):
        o, _ = impl.fwd(q, k, v, 0.7, causal)
        np.testing.assert_allclose(o[:, 0], 1.0, rtol=0, atol=1e-14)


def check_identical_scores(impl, seed=2):
    """All K rows equal: every visible key gets the same weight, O_i = mean of visible v_j,
    LSE_i = S + ln(#visible); and dQ = 0 (every row of dS sums to zero)."""
    rng = _rng(seed)
    n, d = 24, 5
    q = _bf16_grid(rng.standard_normal((n, d)))
    k = np.repeat(_bf16_grid(rng.standard_normal((1, d))), n, axis=0)
    v = _bf16_grid(rng.standard_normal((n, d)))
    do = _bf16_grid(rng.standard_normal((n, d)))
    scale = 0.8
    for causal in (False, True):
        o, lse = impl.fwd(q, k, v, scale, causal)
        for i in range(n):
            nv = i + 1 if causal else n
            np.testing.assert_allclose(o[i], v[:nv].mean(axis=0), rtol=0, atol=1e-13)
            s = scale * float(q[i] @ k[0])
            assert abs(lse[i] - (s + math.log(nv))) < 1e-12
        dq, _, _, _ = impl.bwd(q, k, v, do, scale, causal)
        np.testing.assert_allclose(dq, 0.0, rtol=0, atol=1e-12)


def check_dominant_score(impl):
    """One key aligned with the query at a large scale takes (numerically) all the weight."""
    n, d = 8, 4
    q = np.zeros((n, d))
    q[:, 0] = 1.0
    k = np.zeros((n, d))
    k[:, 1] = 1.0            # orthogonal to every query: score 0
    k[3, 0] = 64.0           # key 3: score 64 * scale
    v = np.arange(n * d, dtype=np.float64).reshape(n, d)
    o, lse = impl.fwd(q, k, v, 1.0, False)
    for i in range(n):
        np.testing.assert_allclose(o[i], v[3], rtol=0, atol=1e-20 + 1e-24 * 64)
        assert abs(lse[i] - 64.0) < 1e-12
    o, _ = impl.fwd(q, k, v, 1.0, True)
    for i in range(3):  # rows 0..2 cannot see key 3: uniform over visible keys
        np.testing.assert_allclose(o[i], v[: i + 1].mean(axis=0), rtol=0, atol=1e-13)
    for i in range(3, n):
        np.testing.assert_allclose(o[i], v[3], rtol=0, atol=1e-20)


def check_causal_future_blind(impl, seed=3):
    """Causal: changing keys/values after position i leaves O_i and LSE_i bit-identical."""
    rng = _rng(seed)
    n, d = 32, 6
    q, k, v = (_bf16_grid(rng.standard_normal((n, d))) for _ in range(3))
    o, lse = impl.fwd(q, k, v, 0.6, True)
    cut = 13
    k2, v2 = k.copy(), v.copy()
    k2[cut + 1:] = _bf16_grid(rng.standard_normal((n - cut - 1, d)) * 5)
    v2[cut + 1:] = _bf16_grid(rng.standard_normal((n - cut - 1, d)) * 5)
    o2, lse2 = impl.fwd(q, k2, v2, 0.6, True)
    assert np.array_equal(o[: cut + 1], o2[: cut + 1])
    assert np.array_equal(lse[: cut + 1], lse2[: cut + 1])
    assert not np.array_equal(o[cut + 1:], o2[cut + 1:])


def check_finite_differences(impl, seed=4, h=1e-6):
    """Central finite differences of L = sum(O * dO) pin dQ, dK and dV."""
    rng = _rng(seed)
    for causal in (False, True):
        n, d = 6, 4
        q, k, v, do = (rng.standard_normal((n, d)) for _ in range(4))
        scale = 0.9
        dq, dk, dv, _ = impl.bwd(q, k, v, do, scale, causal)

        def loss(args):
            o, _ = impl.fwd(args["q"], args["k"], args["v"], scale, causal)
            return float((o * do).sum())

        for name, arr, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
            num = np.zeros_like(arr)
            for idx in np.ndindex(arr.shape):
                plus, minus = arr.copy(), arr.copy()
                plus[idx] += h
                minus[idx] -= h
                args_p = {"q": q, "k": k, "v": v, name: plus}
                args_m = {"q": q, "k": k, "v": v, name: minus}
                num[idx] = (loss(args_p) - loss(args_m)) / (2 * h)
            np.testing.assert_allclose(grad, num, rtol=0, atol=2e-7,
                                       err_msg=f"d{name} (causal={causal})")


def check_gradient_invariants(impl, seed=5):
    """sum_j dK_j = 0 (rows of dS sum to zero) and c_i = rowsum(dO * O)."""
    rng = _rng(seed)
    n, d = 20, 7
    q, k, v, do = (_bf16_grid(rng.standard_normal((n, d))) for _ in range(4))
    for causal in (False, True):
        dq, dk, dv, c = impl.bwd(q, k, v, do, 0.75, causal)
        np.testing.assert_allclose(dk.sum(axis=0), 0.0, rtol=0, atol=1e-12)
        o, _ = impl.fwd(q, k, v, 0.75, causal)
        np.testing.assert_allclose(c, (do * o).sum(axis=1), rtol=0, atol=1e-12)
        # dV columns: sum_j dV_j = sum_i (sum_j P_ij) dO_i = sum_i dO_i
        np.testing.assert_allclose(dv.sum(axis=0), do.sum(axis=0), rtol=0, atol=1e-12)


ALL_FWD_CHECKS = [check_library_softmax, check_n1_closed_form, check_n2_logistic,
                  check_rows_sum_to_one, check_identical_scores, check_dominant_score,
                  check_causal_future_blind]
ALL_BWD_CHECKS = [check_finite_differences, check_gradient_invariants]


# ---------------------------------------------------------------- sliding window (causal)
# An implementation for these checks takes `window` as a keyword: query i sees keys
# i - window .. i.

def check_window_library_softmax(impl, seed=21):
    """Brute force with a window mask against scipy's softmax and logsumexp."""
    rng = _rng(seed)
    for trial in range(10):
        n = int(rng.integers(1, 17))
        d = int(rng.integers(1, 7))
        window = int(rng.integers(0, 6))
        scale = float(rng.uniform(0.2, 1.2))
        q, k, v = (_bf16_grid(rng.standard_normal((n, d))) for _ in range(3))
        o, lse = impl.fwd(q, k, v, scale, True, window=window)
        for i in range(n):
            js = list(range(max(0, i - window), i + 1))
            s = np.array([scale * sum(q[i, x] * k[j, x] for x in range(d)) for j in js])
            p = softmax(s)
            o_ref = sum(pp * v[j] for pp, j in zip(p, js))
            np.testing.assert_allclose(o[i], o_ref, rtol=0, atol=1e-12)
            np.testing.assert_allclose(lse[i], logsumexp(s), rtol=1e-13, atol=1e-13)


def check_window_zero_closed_form(impl, seed=22):
    """window = 0: every query sees only itself, so O_i = v_i and LSE_i = S_ii."""
    rng = _rng(seed)
    n, d = 12, 5
    q, k, v = (_bf16_grid(rng.standard_normal((n, d))) for _ in range(3))
    o, lse = impl.fwd(q, k, v, 0.7, True, window=0)
    assert np.array_equal(o, v)
    np.testing.assert_allclose(lse, 0.7 * (q * k).sum(axis=1), rtol=0, atol=1e-14)
    dq, dk, dv, _ = impl.bwd(q, k, v, q, 0.7, True, window=0)
    np.testing.assert_allclose(dq, 0.0, atol=1e-15)
    np.testing.assert_allclose(dk, 0.0, atol=1e-15)
    np.testing.assert_allclose(dv, q, rtol=0, atol=1e-15)  # dO = q here: dV_j = dO_j


def check_window_past_blind(impl, seed=23):
    """Keys older than the window do not matter: changing them leaves O_i bit-identical,
    and a window reaching the first key equals plain causal attention."""
    rng = _rng(seed)
    n, d, w = 30, 6, 4
    q, k, v = (_bf16_grid(rng.standard_normal((n, d))) for _ in range(3))
    o, lse = impl.fwd(q, k, v, 0.5, True, window=w)
    i0 = 20
    k2, v2 = k.copy(), v.copy()
    k2[: i0 - w] = _bf16_grid(rng.standard_normal((i0 - w, d)) * 4)
    v2[: i0 - w] = 9.0
    o2, lse2 = impl.fwd(q, k2, v2, 0.5, True, window=w)
    assert np.array_equal(o[i0:], o2[i0:]) and np.array_equal(lse[i0:], lse2[i0:])
    assert not np.array_equal(o[: i0 - 1], o2[: i0 - 1])
    oc, lc = impl.fwd(q, k, v, 0.5, True)
    ow, lw = impl.fwd(q, k, v, 0.5, True, window=n - 1)
    np.testing.assert_allclose(ow, oc, rtol=0, atol=1e-14)
    np.testing.assert_allclose(lw, lc, rtol=0, atol=1e-14)


def check_window_finite_differences(impl, seed=24, h=1e-6):
    """Central finite differences of L = sum(O * dO) with a window."""
    rng = _rng(seed)
    n, d, w = 7, 3, 2
    q, k, v, do = (rng.standard_normal((n, d)) for _ in range(4))
    dq, dk, dv, _ = impl.bwd(q, k, v, do, 0.8, True, window=w)

    def loss(args):
        o, _ = impl.fwd(args["q"], args["k"], args["v"], 0.8, True, window=w)
        return float((o * do).sum())

    for name, arr, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            plus, minus = arr.copy(), arr.copy()
            plus[idx] += h
            minus[idx] -= h
            num[idx] = (loss({"q": q, "k": k, "v": v, name: plus})
                        - loss({"q": q, "k": k, "v": v, name: minus})) / (2 * h)
        np.testing.assert_allclose(grad, num, rtol=0, atol=2e-7, err_msg=f"d{name} (window)")


ALL_WINDOW_CHECKS = [check_window_library_softmax, check_window_zero_closed_form,
                     check_window_past_blind, check_window_finite_differences]


# ---------------------------------------------------------------- decoding against a cache
# Each check takes ``decode(q, k, v, seqlens, scale, causal, window=-1) -> (O, LSE)`` with
# q [B, N_q, H, d], k/v [B, N_kv, H_kv, d], O [B, N_q, H, d] and LSE [B, H, N_q].

def _decode_case(rng, B, n_q, H, h_kv, n_kv, d):
    return (_bf16_grid(rng.standard_normal((B, n_q, H, d))),
            _bf16_grid(rng.standard_normal((B, n_kv, h_kv, d))),
            _bf16_grid(rng.standard_normal((B, n_kv, h_kv, d))))


def check_decode_library_softmax(decode, seed=41):
    """Brute force against scipy: the queries are the last N_q positions of each cached
    sequence, query head h reads key/value head h // (H / H_kv), and only the first
    seqlens[b] cache positions exist."""
    rng = _rng(seed)
    B, n_q, H, h_kv, n_kv, d = 3, 3, 4, 2, 13, 5
    lens = [13, 6, 3]
    q, k, v = _decode_case(rng, B, n_q, H, h_kv, n_kv, d)
    for causal, window in ((True, -1), (False, -1), (True, 0), (True, 2), (True, 4)):
        o, lse = decode(q, k, v, lens, 0.6, causal, window)
        for b in range(B):
            n = lens[b]
            for h in range(H):
                kv = h // (H // h_kv)
                for i in range(n_q):
                    pos = n - n_q + i
                    keys = [j for j in range(n)
                            if not causal or (j <= pos and (window < 0 or j >= pos - window))]
                    s = np.array([0.6 * sum(q[b, i, h, x] * k[b, j, kv, x] for x in range(d)) for j in keys])
                    p = softmax(s)
                    o_ref = sum(p[t] * v[b, j, kv] for t, j in enumerate(keys))
                    np.testing.assert_allclose(o[b, i, h], o_ref, rtol=0, atol=1e-12)
                    np.testing.assert_allclose(lse[b, h, i], logsumexp(s), rtol=1e-13, atol=1e-13)


def check_decode_cache_tail_ignored(decode, seed=42):
    """Cache positions past a sequence's length do not exist: NaN there changes nothing."""
    rng = _rng(seed)
    q, k, v = _decode_case(rng, 2, 2, 2, 1, 9, 4)
    lens = [5, 9]
    o1, l1 = decode(q, k, v, lens, 0.5, True)
    k2, v2 = k.copy(), v.copy()
    k2[0, 5:] = np.nan
    v2[0, 5:] = np.nan
    o2, l2 = decode(q, k2, v2, lens, 0.5, True)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def check_decode_grouped_equals_expanded(decode, seed=43):
    """Grouped key/value heads give what the same cache repeated per query head gives."""
    rng = _rng(seed)
    q, k, v = _decode_case(rng, 2, 2, 6, 2, 7, 4)
    og, lg = decode(q, k, v, [7, 4], 0.4, True)
    oe, le = decode(q, np.repeat(k, 3, axis=2), np.repeat(v, 3, axis=2), [7, 4], 0.4, True)
    np.testing.assert_allclose(og, oe, rtol=0, atol=1e-14)
    np.testing.assert_allclose(lg, le, rtol=0, atol=1e-14)


def check_decode_empty_rows(decode, seed=44):
    """An empty cache, or a query placed before the start of its sequence, sees no key:
    O = 0 and LSE = -inf; the other rows are unaffected."""
    rng = _rng(seed)
    q, k, v = _decode_case(rng, 2, 3, 1, 1, 6, 3)
    o, lse = decode(q, k, v, [0, 2], 0.5, True)
    assert np.all(o[0] == 0) and np.all(lse[0] == -np.inf)
    assert np.all(o[1, 0] == 0) and lse[1, 0, 0] == -np.inf
    # the second query of sequence 1 stands at position 0 and sees only key 0
    np.testing.assert_allclose(o[1, 1, 0], v[1, 0, 0], rtol=0, atol=1e-15)
    assert np.isfinite(lse[1, 0, 1]) and np.isfinite(lse[1, 0, 2])


ALL_DECODE_CHECKS = [check_decode_library_softmax, check_decode_cache_tail_ignored,
                     check_decode_grouped_equals_expanded, check_decode_empty_rows]
