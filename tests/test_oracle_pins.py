"""The oracle pinned to things other than itself (CPU only)."""
import json
import os

import numpy as np
import pytest

import oracle
from tests import oracle_pins as pins

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


class COracle:
    """The C oracle (full rows) seen through the pin interface."""

    @staticmethod
    def fwd(q, k, v, scale, causal, window=-1):
        return oracle.fwd_rows(q, k, v, scale, causal, window=window)

    @staticmethod
    def bwd(q, k, v, do, scale, causal, window=-1):
        dq, c, dk, dv = oracle.bwd_rows(q, k, v, do, scale, causal, window=window)
        return dq, dk, dv, c


class DenseOracle:
    @staticmethod
    def fwd(q, k, v, scale, causal, window=-1):
        o, lse, _ = oracle.dense_fwd(q, k, v, scale, causal, window)
        return o, lse

    @staticmethod
    def bwd(q, k, v, do, scale, causal, window=-1):
        return oracle.dense_bwd(q, k, v, do, scale, causal, window)


class OnlineOracle:
    """The streaming form, keys in uneven tiles; backward borrowed from the dense twin."""

    @staticmethod
    def fwd(q, k, v, scale, causal, window=-1):
        n = np.asarray(q).shape[0]
        widths, left, w = [], n, 1
        while left:
            widths.append(min(w, left))
            left -= widths[-1]
            w = w % 5 + 2
        return oracle.online_fwd(q, k, v, scale, causal, widths, window)

    bwd = DenseOracle.bwd


IMPLS = {"c": COracle, "dense": DenseOracle, "online": OnlineOracle}


@pytest.mark.parametrize("impl", sorted(IMPLS))
@pytest.mark.parametrize("check", pins.ALL_FWD_CHECKS, ids=lambda f: f.__name__)
def test_forward_pins(impl, check):
    check(IMPLS[impl])


@pytest.mark.parametrize("impl", ["c", "dense"])
@pytest.mark.parametrize("check", pins.ALL_BWD_CHECKS, ids=lambda f: f.__name__)
def test_backward_pins(impl, check):
    check(IMPLS[impl])


@pytest.mark.parametrize("impl", sorted(IMPLS))
@pytest.mark.parametrize("check", pins.ALL_WINDOW_CHECKS, ids=lambda f: f.__name__)
def test_window_pins(impl, check):
    if impl == "online" and check is pins.check_window_finite_differences:
        pytest.skip("the streaming form has no backward of its own")
    check(IMPLS[impl])


def test_c_oracle_window_sampled_rows_and_bad_args():
    rng = np.random.default_rng(31)
    n, d = 200, 8
    q, k, v, do = (rng.standard_normal((n, d)) for _ in range(4))
    rows = np.array([0, 3, 64, 199])
    o_all, l_all = oracle.fwd_rows(q, k, v, 0.3, True, window=17)
    o, l = oracle.fwd_rows(q, k, v, 0.3, True, rows, window=17)
    assert np.array_equal(o, o_all[rows]) and np.array_equal(l, l_all[rows])
    dq_all, c_all, dk_all, dv_all = oracle.bwd_rows(q, k, v, do, 0.3, True, window=17)
    dq, c, dk, dv = oracle.bwd_rows(q, k, v, do, 0.3, True, rows, rows, window=17)
    assert np.array_equal(dk, dk_all[rows]) and np.array_equal(dq, dq_all[rows])
    p = oracle.prob_row(q, k, 0.3, True, 100, window=17)
    assert abs(p.sum() - 1) < 1e-14 and np.all(p[:83] == 0) and np.all(p[101:] == 0)
    with pytest.raises(RuntimeError):
        oracle.fwd_rows(q, k, v, 0.3, False, window=5)   # a window needs causal attention


def test_prob_row_matches_library_softmax():
    from scipy.special import softmax
    rng = np.random.default_rng(7)
    n, d = 37, 9
    q, k = rng.standard_normal((n, d)), rng.standard_normal((n, d))
    for causal in (False, True):
        for i in (0, 1, 17, n - 1):
            p = oracle.prob_row(q, k, 0.4, causal, i)
            nv = i + 1 if causal else n
            assert abs(p.sum() - 1.0) < 1e-14
            assert np.all(p[nv:] == 0.0)
            np.testing.assert_allclose(p[:nv], softmax(0.4 * (k[:nv] @ q[i])), rtol=1e-13, atol=1e-16)


def test_online_equals_two_pass_random_tiles():
    """The pages' central claim: the streaming softmax reaches the two-pass result."""
    rng = np.random.default_rng(11)
    for trial in range(6):
        n, d = int(rng.integers(50, 300)), int(rng.integers(4, 40))
        q, k, v = (rng.standard_normal((n, d)) * 2 for _ in range(3))
        causal = bool(trial % 2)
        widths, left = [], n
        while left:
            widths.append(int(min(left, rng.integers(1, 64))))
            left -= widths[-1]
        o1, l1 = oracle.online_fwd(q, k, v, 0.3, causal, widths)
        o2, l2 = oracle.fwd_rows(q, k, v, 0.3, causal)
        np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-12)
        np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-12)


def test_c_oracle_sampled_rows_equal_full_rows():
    rng = np.random.default_rng(12)
    n, d = 300, 16
    q, k, v, do = (rng.standard_normal((n, d)) for _ in range(4))
    rows = np.array([0, 1, 5, 150, 299])
    for causal in (False, True):
        o_all, l_all = oracle.fwd_rows(q, k, v, 0.25, causal)
        o, l = oracle.fwd_rows(q, k, v, 0.25, causal, rows)
        assert np.array_equal(o, o_all[rows]) and np.array_equal(l, l_all[rows])
        dq_all, c_all, dk_all, dv_all = oracle.bwd_rows(q, k, v, do, 0.25, causal)
        dq, c, dk, dv = oracle.bwd_rows(q, k, v, do, 0.25, causal, rows, rows)
        assert np.array_equal(dq, dq_all[rows]) and np.array_equal(dk, dk_all[rows])
        assert np.array_equal(dv, dv_all[rows]) and np.array_equal(c, c_all[rows])


def test_c_oracle_rejects_bad_rows():
    q = np.zeros((4, 2))
    with pytest.raises(RuntimeError):
        oracle.fwd_rows(q, q, q, 1.0, False, [4])
    with pytest.raises(RuntimeError):
        oracle.bwd_rows(q, q, q, q, 1.0, False, [-1], [0])


def test_golden_regression_cases():
    """Expected values written by tests/golden/make_golden.py (oracle only)."""
    with open(os.path.join(GOLDEN, "oracle_small_cases.json")) as f:
        cases = json.load(f)["cases"]
    from exact_io_aware_93_b200.inputs import make_inputs
    for case in cases:
        t = make_inputs(1, 1, case["N"], case["d"], case["seed"], with_do=True)
        q, k, v, do = (t[n][0, :, 0].double().numpy() for n in ("q", "k", "v", "do"))
        o, lse = oracle.fwd_rows(q, k, v, case["scale"], case["causal"])
        dq, _, dk, dv = oracle.bwd_rows(q, k, v, do, case["scale"], case["causal"])
        for name, got in (("o", o), ("lse", lse), ("dq", dq), ("dk", dk), ("dv", dv)):
            np.testing.assert_allclose(got, np.array(case[name]), rtol=1e-12, atol=1e-13,
                                       err_msg=f"{case['name']}:{name}")


def test_page_score_matrix_table():
    """The score-matrix sizes the pages print (N^2 x 2 bytes per head, FP16)."""
    from exact_io_aware_93_b200.accounting import score_matrix_bytes
    with open(os.path.join(GOLDEN, "score_matrix_table.json")) as f:
        table = json.load(f)
    for row in table["rows"]:
        n = row["context_length"]
        assert score_matrix_bytes(n, 1, 2) == n * n * 2
        got = score_matrix_bytes(n, 1, 2)
        assert abs(got - row["per_head_bytes"]) / row["per_head_bytes"] < row["rel_tol"], row
        assert abs(got * 32 - row["per_layer_32_heads_bytes"]) / row["per_layer_32_heads_bytes"] \
            < row["rel_tol"], row
        assert abs(n * n - row["scores_per_head"]) / row["scores_per_head"] < row["rel_tol"], row
