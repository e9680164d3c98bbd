"""The decoding oracle pinned to brute force and invariants (CPU only), and planted
mistakes in a numpy copy of it that the pins must catch."""
import numpy as np
import pytest

import oracle
from tests import oracle_pins as pins


@pytest.mark.parametrize("check", pins.ALL_DECODE_CHECKS, ids=lambda f: f.__name__)
def test_decode_pins(check):
    check(oracle.decode_rows)


def test_decode_equals_whole_sequence_rows():
    """The decode of the last N_q positions equals the same rows of the whole sequence's
    forward pass (the numpy whole-matrix twin), with and without a window."""
    rng = np.random.default_rng(45)
    n, n_q, d = 40, 5, 8
    qs, ks, vs = (rng.standard_normal((n, d)) for _ in range(3))
    for window in (-1, 0, 3, 39):
        o_ref, l_ref, _ = oracle.dense_fwd(qs, ks, vs, 0.35, True, window)
        o, lse = oracle.decode_rows(qs[None, n - n_q:, None], ks[None, :, None], vs[None, :, None],
                                    None, 0.35, True, window)
        np.testing.assert_allclose(o[0, :, 0], o_ref[n - n_q:], rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse[0, 0], l_ref[n - n_q:], rtol=0, atol=1e-13)


def test_decode_rejects_window_without_causal():
    q = np.zeros((1, 1, 1, 2))
    with pytest.raises(ValueError):
        oracle.decode_rows(q, q, q, None, 1.0, False, 3)


def _decode_mutant(q, k, v, seqlens, scale, causal, window=-1, *, pos_shift=0, head_mod=False,
                   ignore_lens=False, noncausal_masks=False):
    B, n_q, H, d = q.shape
    n_kv, h_kv = k.shape[1], k.shape[2]
    lens = [n_kv] * B if (seqlens is None or ignore_lens) else list(seqlens)
    o = np.zeros((B, n_q, H, d))
    lse = np.full((B, H, n_q), -np.inf)
    for b in range(B):
        n = lens[b]
        for h in range(H):
            kv = h % h_kv if head_mod else h // (H // h_kv)
            for i in range(n_q):
                pos = n - n_q + i + pos_shift
                j = np.arange(n)
                vis = (j <= pos) if (causal or noncausal_masks) else np.ones(n, bool)
                if window >= 0:
                    vis &= j >= pos - window
                if not vis.any():
                    continue
                s = np.where(vis, scale * (k[b, :n, kv] @ q[b, i, h]), -np.inf)
                m = s.max()
                e = np.exp(s - m)
                o[b, i, h] = e @ v[b, :n, kv] / e.sum()
                lse[b, h, i] = m + np.log(e.sum())
    return o, lse


def _mutant(**kw):
    return lambda q, k, v, lens, scale, causal, window=-1: _decode_mutant(q, k, v, lens, scale, causal,
                                                                          window, **kw)


DECODE_MUTANTS = {
    "query_one_position_late": _mutant(pos_shift=1),
    "query_one_position_early": _mutant(pos_shift=-1),
    "kv_head_by_modulo": _mutant(head_mod=True),
    "cache_length_ignored": _mutant(ignore_lens=True),
    "noncausal_masked": _mutant(noncausal_masks=True),
}


def _fails_some_decode_pin(decode):
    for check in pins.ALL_DECODE_CHECKS:
        try:
            with np.errstate(all="ignore"):
                check(decode)
        except (AssertionError, ValueError, FloatingPointError, IndexError):
            return True
    return False


def test_unmutated_decode_copy_passes():
    assert not _fails_some_decode_pin(_mutant())


@pytest.mark.parametrize("name", sorted(DECODE_MUTANTS))
def test_decode_mutant_is_caught(name):
    assert _fails_some_decode_pin(DECODE_MUTANTS[name]), f"no pin catches mutant {name}"
