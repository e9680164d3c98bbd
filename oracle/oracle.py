"""fp64 CPU oracle for exact attention -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
leg of ``bench.py`` may import this module.  It never touches the CUDA path.

Three independent routes to the same numbers, all fp64, all on one head
(row-major ``[N, d]`` arrays):

* ``fwd_rows`` / ``prob_row`` / ``bwd_rows``: the plain C definition in
  ``attention_oracle.c`` (OpenMP over rows), used at full sizes on sampled
  rows.  Forward = standard attention softmax(scale * Q K^T) V with the score
  row materialised and a two-pass softmax ("Flash Attention Explained",
  institutepm.com, section "The Problem Standard Attention Has"; holysheep.ai
  review, section "What Is Flash Attention and Why Does It Matter?").
* ``dense_fwd`` / ``dense_bwd``: the same definition as whole-matrix numpy
  algebra, for tiny cases and cross-checks.
* ``online_fwd``: the streaming form the pages describe -- keys processed
  tile by tile while a running row maximum and a running row sum are kept and
  earlier partial results are rescaled whenever the maximum grows
  ("Flash Attention Explained", "Compute softmax incrementally"; holysheep.ai
  review, "the online softmax algorithm combined with tiling").  It exists to
  pin the claim that the streaming result equals the two-pass result.
* ``decode_rows``: decoding -- N_q new queries per sequence, placed after a
  cached prefix of per-sequence length, against a key/value cache; each
  (sequence, head) is ``fwd_rows`` evaluated at the queries' positions.

Causal: key j visible to query i iff j <= i.  LSE is the natural-log
log-sum-exp of the scaled, visible scores.

Parity status: pinned (see ``tests/test_oracle_pins.py``): library softmax /
logsumexp (scipy) on brute-force tiny inputs, logistic closed form at N=2,
N=1 closed form, identical-score and dominant-score cases, rows of P summing
to one, central finite differences of L = sum(O * dO) for the gradients,
sum_j dK_j = 0, and online == two-pass.  ``decode_rows`` is pinned by scipy
brute force over positions, head groups and cache lengths, by the NaN-filled
cache tail changing nothing, by grouped == expanded heads, by the empty-row
cases, and by equality with the whole-sequence rows of ``dense_fwd``
(``tests/test_oracle_decode_pins.py``, which also plants five mistakes in a
numpy copy and checks that each is caught).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attention_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "liboracle.so")
_lib = None
_lock = threading.Lock()

_dp = ctypes.POINTER(ctypes.c_double)
_ip = ctypes.POINTER(ctypes.c_int64)


def build_oracle(force: bool = False) -> str:
    """Compile the C oracle with gcc (plain -O2, no fast-math) and return its path."""
    with _lock:
        fresh = (os.path.exists(_LIB_PATH)
                 and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC))
        if fresh and not force:
            return _LIB_PATH
        os.makedirs(_BUILD_DIR, exist_ok=True)
        tmp = f"{_LIB_PATH}.{os.getpid()}.tmp"
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True, capture_output=True, text=True)
        os.replace(tmp, _LIB_PATH)
        return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    path = build_oracle()
    lib = ctypes.CDLL(path)
    lib.oracle_fwd_rows.argtypes = [_dp, _dp, _dp, ctypes.c_int64, ctypes.c_int, ctypes.c_double,
                                    ctypes.c_int, ctypes.c_int64, _ip, ctypes.c_int64, _dp, _dp]
    lib.oracle_fwd_rows.restype = ctypes.c_int
    lib.oracle_prob_row.argtypes = [_dp, _dp, ctypes.c_int64, ctypes.c_int, ctypes.c_double,
                                    ctypes.c_int, ctypes.c_int64, ctypes.c_int64, _dp]
    lib.oracle_prob_row.restype = ctypes.c_int
    lib.oracle_bwd_rows.argtypes = [_dp, _dp, _dp, _dp, ctypes.c_int64, ctypes.c_int,
                                    ctypes.c_double, ctypes.c_int, ctypes.c_int64,
                                    _ip, ctypes.c_int64, _dp, _dp,
                                    _ip, ctypes.c_int64, _dp, _dp]
    lib.oracle_bwd_rows.restype = ctypes.c_int
    lib.oracle_num_threads.restype = ctypes.c_int
    lib.oracle_set_num_threads.argtypes = [ctypes.c_int]
    _lib = lib
    return lib


def oracle_threads(n: int | None = None) -> int:
    """Set (if n is given) and return the OpenMP thread count the C oracle uses."""
    lib = _load()
    if n is not None:
        lib.oracle_set_num_threads(int(n))
    return int(lib.oracle_num_threads())


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


def _rows(r) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(r, dtype=np.int64).reshape(-1))


def _ptr(a: np.ndarray, t):
    return a.ctypes.data_as(t)


def _check_head(q, k, v):
    if q.ndim != 2 or k.shape != q.shape or v.shape != q.shape:
        raise ValueError(f"one head of shape [N, d] expected, got {q.shape}, {k.shape}, {v.shape}")


def fwd_rows(q, k, v, scale: float, causal: bool, rows=None, window: int = -1):
    """O (fp64 [len(rows), d]) and LSE (fp64 [len(rows)]) of one head at the given query rows.

    window >= 0 (causal only): query i sees keys i - window .. i."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    _check_head(q, k, v)
    n, d = q.shape
    rows = _rows(np.arange(n) if rows is None else rows)
    o = np.empty((rows.size, d), np.float64)
    lse = np.empty(rows.size, np.float64)
    rc = _load().oracle_fwd_rows(_ptr(q, _dp), _ptr(k, _dp), _ptr(v, _dp), n, d, float(scale),
                                 int(bool(causal)), int(window), _ptr(rows, _ip), rows.size,
                                 _ptr(o, _dp), _ptr(lse, _dp))
    if rc != 0:
        raise RuntimeError(f"oracle_fwd_rows failed ({rc})")
    return o, lse


def prob_row(q, k, scale: float, causal: bool, i: int, window: int = -1) -> np.ndarray:
    """The normalised attention probabilities P_i. of one query row (zeros where masked)."""
    q, k = _f64(q), _f64(k)
    n, d = q.shape
    p = np.empty(n, np.float64)
    rc = _load().oracle_prob_row(_ptr(q, _dp), _ptr(k, _dp), n, d, float(scale),
                                 int(bool(causal)), int(window), int(i), _ptr(p, _dp))
    if rc != 0:
        raise RuntimeError(f"oracle_prob_row failed ({rc})")
    return p


def bwd_rows(q, k, v, do, scale: float, causal: bool, qrows=None, krows=None, window: int = -1):
    """Gradients of L = sum(O * dO) for one head.

    Returns (dq [len(qrows), d], c [len(qrows)], dk [len(krows), d], dv [len(krows), d]),
    where c_i = sum_t P_it dP_it is the Jacobian row constant.
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    _check_head(q, k, v)
    n, d = q.shape
    qrows = _rows(np.arange(n) if qrows is None else qrows)
    krows = _rows(np.arange(n) if krows is None else krows)
    dq = np.empty((qrows.size, d), np.float64)
    c = np.empty(qrows.size, np.float64)
    dk = np.empty((krows.size, d), np.float64)
    dv = np.empty((krows.size, d), np.float64)
    rc = _load().oracle_bwd_rows(_ptr(q, _dp), _ptr(k, _dp), _ptr(v, _dp), _ptr(do, _dp), n, d,
                                 float(scale), int(bool(causal)), int(window),
                                 _ptr(qrows, _ip), qrows.size, _ptr(dq, _dp), _ptr(c, _dp),
                                 _ptr(krows, _ip), krows.size, _ptr(dk, _dp), _ptr(dv, _dp))
    if rc != 0:
        raise RuntimeError(f"oracle_bwd_rows failed ({rc})")
    return dq, c, dk, dv


def _visible(n: int, causal: bool, window: int = -1) -> np.ndarray:
    i = np.arange(n)[:, None]
    j = np.arange(n)[None, :]
    vis = (j <= i) if causal else np.ones((n, n), dtype=bool)
    if window >= 0:
        vis = vis & (j >= i - window)
    return vis


def dense_fwd(q, k, v, scale: float, causal: bool, window: int = -1):
    """Whole-matrix fp64 standard attention of one head: (O [N, d], LSE [N], P [N, N])."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    n = q.shape[0]
    s = scale * (q @ k.T)
    s = np.where(_visible(n, causal, window), s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    l = e.sum(axis=1, keepdims=True)
    p = e / l
    return p @ v, (m + np.log(l))[:, 0], p


def dense_bwd(q, k, v, do, scale: float, causal: bool, window: int = -1):
    """Whole-matrix fp64 gradients of L = sum(O * dO): (dQ, dK, dV, c)."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    _, _, p = dense_fwd(q, k, v, scale, causal, window)
    dp = do @ v.T
    c = (p * dp).sum(axis=1)
    ds = p * (dp - c[:, None])
    return scale * (ds @ k), scale * (ds.T @ q), p.T @ do, c


def online_fwd(q, k, v, scale: float, causal: bool, tile_widths, window: int = -1):
    """Streaming (online-softmax) forward of one head, keys consumed in tiles of the given widths.

    State per query row: running maximum m, running sum l of exp(s - m), and an
    unnormalised output accumulator; when a tile raises m, the earlier sum and
    accumulator are multiplied by exp(m_old - m_new).  After the last tile
    O = acc / l and LSE = m + ln l.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    n, d = q.shape
    widths = [int(w) for w in tile_widths]
    if sum(widths) != n or min(widths) < 1:
        raise ValueError("tile widths must be positive and cover all keys")
    vis = _visible(n, causal, window)
    m = np.full(n, -np.inf)
    l = np.zeros(n)
    acc = np.zeros((n, d))
    start = 0
    for w in widths:
        cols = slice(start, start + w)
        s = scale * (q @ k[cols].T)
        s = np.where(vis[:, cols], s, -np.inf)
        m_new = np.maximum(m, s.max(axis=1))
        # rows that have seen no visible key yet keep m = -inf; guard exp(-inf - -inf)
        alpha = np.where(np.isfinite(m_new), np.exp(np.where(np.isfinite(m), m - m_new, -np.inf)), 1.0)
        e = np.where(np.isfinite(m_new)[:, None], np.exp(s - m_new[:, None]), 0.0)
        l = alpha * l + e.sum(axis=1)
        acc = alpha[:, None] * acc + e @ v[cols]
        m = m_new
        start += w
    return acc / l[:, None], m + np.log(l)


def decode_rows(q, k, v, seqlens, scale: float, causal: bool, window: int = -1, heads=None):
    """Decoding: the outputs of N_q new queries per sequence against a key/value cache.

    ``q``: [B, N_q, H, d]; ``k``, ``v``: [B, N_kv, H_kv, d], the cache, of which only the
    first ``seqlens[b]`` positions of sequence b are real (``None``: all N_kv).  Query head
    h reads key/value head h // (H // H_kv) ("Flash Attention Explained", institutepm.com,
    "Grouped Query Attention").  With causal masking query i of sequence b stands at
    position len_b - N_q + i, right after the cached prefix it extends, and sees the keys
    at or before it (and, with a window, no more than ``window`` positions back); without
    it every cached key is visible.  This is the generation phase the pages set against
    prompt processing ("What Is Flash Attention?", bestllmfor.com, table "What you
    actually gain on a local machine").

    Each (b, h) is the plain definition of ``fwd_rows`` on one head: the queries are placed
    at their positions in an otherwise empty query block of the sequence's length and only
    those rows are evaluated.  A query that sees no key (empty cache, or a position before
    the start) gets O = 0 and LSE = -inf.  ``heads`` restricts the work to a list of (b, h)
    pairs; other outputs stay NaN.

    Returns O (fp64 [B, N_q, H, d]) and LSE (fp64 [B, H, N_q]).
    """
    q = np.asarray(q)
    k = np.asarray(k)
    v = np.asarray(v)
    B, n_q, H, d = q.shape
    n_kv, h_kv = k.shape[1], k.shape[2]
    if k.shape != (B, n_kv, h_kv, d) or v.shape != k.shape or H % h_kv:
        raise ValueError(f"bad decode shapes {q.shape}, {k.shape}, {v.shape}")
    if window >= 0 and not causal:
        raise ValueError("a window needs causal attention")
    lens = np.full(B, n_kv, np.int64) if seqlens is None else np.clip(np.asarray(seqlens, np.int64), 0, n_kv)
    group = H // h_kv
    o = np.full((B, n_q, H, d), np.nan)
    lse = np.full((B, H, n_q), np.nan)
    todo = [(b, h) for b in range(B) for h in range(H)] if heads is None else [tuple(x) for x in heads]
    for b, h in todo:
        n = int(lens[b])
        kh, vh = k[b, :n, h // group], v[b, :n, h // group]
        o[b, :, h] = 0.0
        lse[b, h] = -np.inf
        if n == 0:
            continue
        for i in range(n_q):
            pos = n - n_q + i if causal else 0
            if pos < 0:
                continue
            qh = np.zeros((n, d))
            qh[pos] = q[b, i, h]
            oi, li = fwd_rows(qh, kh, vh, scale, causal, [pos], window)
            o[b, i, h], lse[b, h, i] = oi[0], li[0]
    return o, lse
