"""Plant plausible mistakes in a copy of the oracle and check that the pins catch each one.

The mistakes live only in this file, in CPU numpy code: a dropped scale, an
off-by-one causal mask, a swapped operand, a wrong sign, a missing term.
"""
import numpy as np
import pytest

from tests import oracle_pins as pins


def _fwd(q, k, v, scale, causal, *, use_scale=True, mask_shift=0, lse_no_max=False,
         reverse_v=False, no_norm=False, window=-1, window_shift=0):
    q, k, v = (np.asarray(a, np.float64) for a in (q, k, v))
    n = q.shape[0]
    s = (scale if use_scale else 1.0) * (q @ k.T)
    vis = np.tril(np.ones((n, n), bool), k=mask_shift) if causal else np.ones((n, n), bool)
    if window >= 0:
        vis = vis & ~np.tril(np.ones((n, n), bool), k=-(window + 1 + window_shift))
    s = np.where(vis, s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    l = e.sum(axis=1, keepdims=True)
    p = e if no_norm else e / l
    vv = v[::-1] if reverse_v else v
    lse = np.log(l)[:, 0] if lse_no_max else (m + np.log(l))[:, 0]
    return p @ vv, lse, p


def _bwd(q, k, v, do, scale, causal, *, sign=1.0, c_from_dp=False, dk_scale=True,
         dv_untransposed=False, fwd_kw=None, window=-1):
    q, k, v, do = (np.asarray(a, np.float64) for a in (q, k, v, do))
    _, _, p = _fwd(q, k, v, scale, causal, window=window, **(fwd_kw or {}))
    dp = do @ v.T
    c = dp.sum(axis=1) if c_from_dp else (p * dp).sum(axis=1)
    ds = sign * p * (dp - c[:, None])
    dk = (scale if dk_scale else 1.0) * (ds.T @ q)
    dv = (p @ do) if dv_untransposed else (p.T @ do)
    return scale * (ds @ k), dk, dv, c


def _impl(fwd_kw=None, bwd_kw=None):
    fwd_kw, bwd_kw = fwd_kw or {}, bwd_kw or {}

    class Mutant:
        @staticmethod
        def fwd(q, k, v, scale, causal, window=-1):
            o, lse, _ = _fwd(q, k, v, scale, causal, window=window, **fwd_kw)
            return o, lse

        @staticmethod
        def bwd(q, k, v, do, scale, causal, window=-1):
            return _bwd(q, k, v, do, scale, causal, fwd_kw=fwd_kw, window=window, **bwd_kw)
    return Mutant


MUTANTS = {
    "dropped_scale": _impl(fwd_kw={"use_scale": False}),
    "mask_sees_next_key": _impl(fwd_kw={"mask_shift": 1}),
    "mask_misses_diagonal": _impl(fwd_kw={"mask_shift": -1}),
    "lse_without_max": _impl(fwd_kw={"lse_no_max": True}),
    "values_reversed": _impl(fwd_kw={"reverse_v": True}),
    "unnormalised_p": _impl(fwd_kw={"no_norm": True}),
    "ds_sign_flipped": _impl(bwd_kw={"sign": -1.0}),
    "row_constant_from_dp_only": _impl(bwd_kw={"c_from_dp": True}),
    "dk_missing_scale": _impl(bwd_kw={"dk_scale": False}),
    "dv_untransposed": _impl(bwd_kw={"dv_untransposed": True}),
    "window_one_key_too_many": _impl(fwd_kw={"window_shift": 1}),
    "window_one_key_too_few": _impl(fwd_kw={"window_shift": -1}),
}


def _fails_some_pin(impl):
    for check in pins.ALL_FWD_CHECKS + pins.ALL_BWD_CHECKS + pins.ALL_WINDOW_CHECKS:
        try:
            with np.errstate(all="ignore"):
                check(impl)
        except (AssertionError, ValueError, FloatingPointError, IndexError):
            return True
    return False


def test_unmutated_copy_passes():
    assert not _fails_some_pin(_impl())


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    assert _fails_some_pin(MUTANTS[name]), f"no pin catches mutant {name}"
