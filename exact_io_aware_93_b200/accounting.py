"""Work and traffic accounting used by the benchmark (no attention arithmetic).

FLOP convention: the forward pass does two B*H*N*N*d contractions (Q K^T and
P V) at 2 flop per multiply-add, i.e. 4*B*H*N^2*d, halved when causal; the
backward pass counts 2.5x the forward.

Algorithmic bytes are the bytes a kernel must move at minimum: each operand
read once, each result written once (bf16 tensors 2 bytes per element, fp32
statistics 4 bytes).
"""
from __future__ import annotations


def fwd_flops(B: int, H: int, N: int, d: int, causal: bool) -> float:
    f = 4.0 * B * H * N * N * d
    return f / 2 if causal else f


def bwd_flops(B: int, H: int, N: int, d: int, causal: bool) -> float:
    return 2.5 * fwd_flops(B, H, N, d, causal)


def fwd_bytes(B: int, H: int, N: int, d: int) -> int:
    """Q, K, V read and O written (bf16), LSE written (fp32)."""
    return 2 * 4 * B * H * N * d + 4 * B * H * N


def bwd_bytes(B: int, H: int, N: int, d: int) -> int:
    """Q, K, V, O, dO read and dQ, dK, dV written (bf16); LSE and D (fp32) read/written once;
    the fp32 dQ accumulator written once and read once."""
    return 2 * 8 * B * H * N * d + 3 * 4 * B * H * N + 2 * 4 * B * H * N * d


def score_matrix_bytes(N: int, heads: int, bytes_per_score: int = 2) -> int:
    """Size of the N x N score matrix standard attention would materialise."""
    return N * N * heads * bytes_per_score


def visible_pairs(N: int, causal: bool, window: int = -1) -> float:
    """(query, key) pairs per head that the FLOP convention counts: N^2 (non-causal), N^2 / 2
    (causal), and with a causal window of W keys before the query the exact count
    sum_i min(i, W) + 1."""
    if window < 0:
        return N * N / 2 if causal else float(N * N)
    w = min(window, N - 1)
    return w * (w + 1) / 2 + (N - w) * (w + 1)


def fwd_flops_window(B: int, H: int, N: int, d: int, causal: bool, window: int = -1) -> float:
    return 4.0 * B * H * d * visible_pairs(N, causal, window)


def bwd_flops_window(B: int, H: int, N: int, d: int, causal: bool, window: int = -1) -> float:
    return 2.5 * fwd_flops_window(B, H, N, d, causal, window)


def decode_cache_keys(length: int, N_q: int, causal: bool, window: int = -1) -> int:
    """Cache positions of one sequence that some new query can see: all `length` of them,
    or with a causal window the last N_q + window (fewer when the cache is shorter)."""
    n = max(0, int(length))
    if causal and window >= 0:
        return min(n, N_q + window)
    return n


def decode_bytes(seqlens, B: int, H: int, H_kv: int, N_q: int, d: int, causal: bool, window: int = -1) -> int:
    """Algorithmic bytes of one decode call: the visible K and V cache rows of every
    key/value head read once (bf16), Q read and O written (bf16), LSE written (fp32) and
    the lengths read (int32)."""
    keys = sum(decode_cache_keys(n, N_q, causal, window) for n in seqlens)
    return 2 * 2 * keys * H_kv * d + 2 * 2 * B * N_q * H * d + 4 * B * H * N_q + 4 * B


def decode_flops(seqlens, H: int, N_q: int, d: int, causal: bool, window: int = -1) -> float:
    """4*d flops per visible (query, key) pair and query head."""
    pairs = 0
    for n in seqlens:
        n = max(0, int(n))
        for i in range(N_q):
            pos = n - N_q + i if causal else n - 1
            if pos < 0:
                continue
            pairs += (min(pos, window) + 1) if (causal and window >= 0) else (pos + 1 if causal else n)
    return 4.0 * d * H * pairs
