"""Compare CUDA-path outputs with the fp64 oracle on the same seeded bf16 inputs.

Tolerances (written here, used by every parity test):
  O    : max |O_gpu - O_ref| <= 1e-2            (O is bf16)
  LSE  : max |LSE_gpu - LSE_ref| / max(1, |LSE_ref|) <= 1e-3
  dQ, dK, dV : max |g - g_ref| / max |g_ref| <= 2e-2, per tensor over the checked rows
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from exact_io_aware_93_b200.inputs import head_row_seed, sample_rows

O_TOL = 1e-2
LSE_TOL = 1e-3
GRAD_TOL = 2e-2
# Rows beyond the five configurations (grouped heads, sliding windows): O is judged by the
# error in excess of half a bf16 ulp at the reference value (the rounding every bf16 output
# carries; at |O| >= 4 it alone exceeds 1e-2), and gradient errors are divided by
# max(max|g_ref|, GRAD_ABS_FLOOR) because some of these problems have gradients that are
# exactly zero (a window of 0 keys makes dQ = dK = 0).
GRAD_ABS_FLOOR = 1e-3
# Small random problems (a row seeing one or two keys, a nearly one-hot softmax) have
# gradients dQ, dK that are near zero by cancellation, dS = P o (dP - D) with dP ~ D, so the
# roundings the method performs by design dominate them: D from the stored 16-bit O, the
# 16-bit P that enters dS and dV, the 16-bit dS operand of the dK and dQ products, and the
# 16-bit outputs.  grad_errors_gqa(bounded=True) judges only the error in excess of that
# rounding bound (grad_rounding_bounds, checked against an fp64 simulation of exactly those
# roundings), still relative to max |g_ref|.


def bf16_half_ulp(x: np.ndarray) -> np.ndarray:
    """Half the spacing of the bf16 grid at |x| (8 significant bits)."""
    ax = np.maximum(np.abs(x), np.finfo(np.float32).tiny)
    return np.exp2(np.floor(np.log2(ax)) - 8)


def half_ulp(x: np.ndarray, dtype: torch.dtype) -> np.ndarray:
    """Half the spacing of the output type's grid at |x|: bf16 (8 significant bits) or
    fp16 (11 significant bits; subnormal spacing below 2^-14)."""
    if dtype == torch.float16:
        ax = np.maximum(np.abs(x), 2.0 ** -14)
        return np.exp2(np.floor(np.log2(ax)) - 11)
    return bf16_half_ulp(x)


def _head(t: torch.Tensor, b: int, h: int) -> np.ndarray:
    return t[b, :, h, :].to(torch.float64).numpy()


def fwd_errors(inputs, o_gpu, lse_gpu, scale, causal, rows_per_head=None, seed=0, heads=None):
    """Max errors of (O, LSE) over the checked rows of the given heads (default: all)."""
    B, N, H, _ = inputs["q"].shape
    o_gpu = o_gpu.cpu()
    lse_gpu = lse_gpu.cpu()
    heads = heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]
    worst_o, worst_l, where = 0.0, 0.0, None
    for b, h in heads:
        rows = sample_rows(N, rows_per_head, head_row_seed(seed, b, h)).numpy()
        o_ref, lse_ref = oracle.fwd_rows(_head(inputs["q"], b, h), _head(inputs["k"], b, h),
                                         _head(inputs["v"], b, h), scale, causal, rows)
        o_g = o_gpu[b, rows, h, :].to(torch.float64).numpy()
        l_g = lse_gpu[b, h, rows].to(torch.float64).numpy()
        eo = np.abs(o_g - o_ref)
        el = np.abs(l_g - lse_ref) / np.maximum(1.0, np.abs(lse_ref))
        if not np.all(np.isfinite(o_g)) or not np.all(np.isfinite(l_g)):
            return float("inf"), float("inf"), (b, h, "non-finite")
        if eo.max() > worst_o:
            r, c = (int(x) for x in np.unravel_index(eo.argmax(), eo.shape))
            o_ref_bf16 = float(torch.tensor(o_ref[r, c]).to(torch.bfloat16).double())
            worst_o = float(eo.max())
            where = dict(b=b, h=h, row=int(rows[r]), col=c, o_ref=float(o_ref[r, c]),
                         o_gpu=float(o_g[r, c]), err_vs_bf16_ref=abs(float(o_g[r, c]) - o_ref_bf16))
        worst_l = max(worst_l, float(el.max()))
    return worst_o, worst_l, where


def grad_errors(inputs, grads_gpu, scale, causal, heads_full, heads_sampled):
    """Relative max errors of dQ, dK, dV: full heads, plus (b, h, rows) sampled heads."""
    B, N, H, _ = inputs["q"].shape
    num = {"dq": 0.0, "dk": 0.0, "dv": 0.0}
    den = {"dq": 0.0, "dk": 0.0, "dv": 0.0}
    jobs = [(b, h, None) for b, h in heads_full] + list(heads_sampled)
    for b, h, rows in jobs:
        rows_np = np.arange(N) if rows is None else np.asarray(rows)
        dq, _, dk, dv = oracle.bwd_rows(_head(inputs["q"], b, h), _head(inputs["k"], b, h),
                                        _head(inputs["v"], b, h), _head(inputs["do"], b, h),
                                        scale, causal, rows_np, rows_np)
        for name, ref in (("dq", dq), ("dk", dk), ("dv", dv)):
            got = grads_gpu[name][b, rows_np, h, :].to(torch.float64).cpu().numpy()
            num[name] = max(num[name], float(np.abs(got - ref).max()))
            den[name] = max(den[name], float(np.abs(ref).max()))
    return {n: num[n] / max(den[n], 1e-30) for n in num}


def _kv_head(t, b, hkv):
    return t[b, :, hkv, :].to(torch.float64).numpy()


def fwd_errors_gqa(inputs, o_gpu, lse_gpu, scale, causal, window=-1, rows_per_head=None, seed=0):
    """Forward errors when K/V have fewer heads than Q: query head h reads key/value head
    h // (H / H_kv).  The O error is the excess over half a bf16 ulp (see GRAD_ABS_FLOOR)."""
    B, N, H, _ = inputs["q"].shape
    Hkv = inputs["k"].shape[2]
    group = H // Hkv
    o_gpu, lse_gpu = o_gpu.cpu(), lse_gpu.cpu()
    worst_o, worst_l = 0.0, 0.0
    for b in range(B):
        for h in range(H):
            rows = sample_rows(N, rows_per_head, head_row_seed(seed, b, h)).numpy()
            o_ref, lse_ref = oracle.fwd_rows(_head(inputs["q"], b, h), _kv_head(inputs["k"], b, h // group),
                                             _kv_head(inputs["v"], b, h // group), scale, causal, rows,
                                             window=window)
            o_g = o_gpu[b, rows, h, :].to(torch.float64).numpy()
            l_g = lse_gpu[b, h, rows].to(torch.float64).numpy()
            worst_o = max(worst_o, float((np.abs(o_g - o_ref) - half_ulp(o_ref, o_gpu.dtype)).max()))
            worst_l = max(worst_l, float((np.abs(l_g - lse_ref) / np.maximum(1.0, np.abs(lse_ref))).max()))
    return worst_o, worst_l


def grad_rounding_bounds(q, k, v, do, scale, causal, window, dtype):
    """Per-element bounds (dQ, dK, dV of one query head, fp64) on the effect of the roundings
    the backward performs by design: D = rowsum(dO o O) from O rounded to `dtype`, P rounded
    to `dtype` (in dS and dV), dS rounded to `dtype` (operand of the dK and dQ products), plus
    a 1e-6 relative allowance for fp32 accumulation.  The outputs' own rounding is added by
    the caller."""
    O, _, P = oracle.dense_fwd(q, k, v, scale, causal, window)
    dP = do @ v.T
    D = (do * O).sum(1)
    dD = (np.abs(do) * half_ulp(O, dtype)).sum(1) + 1e-6 * (np.abs(do) * np.abs(O)).sum(1)
    dS = P * (dP - D[:, None])
    seen = P > 0
    edS = np.where(seen, P * dD[:, None] + half_ulp(P, dtype) * (np.abs(dP - D[:, None]) + dD[:, None])
                   + half_ulp(dS, dtype) + 1e-6 * P * (np.abs(do) @ np.abs(v).T), 0.0)
    return (scale * edS @ np.abs(k), scale * edS.T @ np.abs(q),
            np.where(seen, half_ulp(P, dtype), 0.0).T @ np.abs(do))


def grad_errors_gqa(inputs, grads_gpu, scale, causal, window=-1, bounded=False):
    """Relative max errors of dQ, dK, dV (every row) with grouped key/value heads: dK and dV
    of a key/value head are the sums over the query heads that share it.  bounded=True counts
    only the error in excess of grad_rounding_bounds plus half an ulp of each output."""
    B, N, H, d = inputs["q"].shape
    Hkv = inputs["k"].shape[2]
    group = H // Hkv
    dtype = inputs["q"].dtype
    num = {"dq": 0.0, "dk": 0.0, "dv": 0.0}
    den = {"dq": 0.0, "dk": 0.0, "dv": 0.0}

    def excess(got, ref, bound):
        if not bounded:
            return float(np.abs(got - ref).max())
        return float(np.maximum(np.abs(got - ref) - bound - half_ulp(ref, dtype), 0.0).max())

    for b in range(B):
        for hk in range(Hkv):
            dk_ref = np.zeros((N, d))
            dv_ref = np.zeros((N, d))
            dk_bound = np.zeros((N, d))
            dv_bound = np.zeros((N, d))
            for h in range(hk * group, (hk + 1) * group):
                qh, kh, vh, doh = (_head(inputs["q"], b, h), _kv_head(inputs["k"], b, hk),
                                   _kv_head(inputs["v"], b, hk), _head(inputs["do"], b, h))
                dq, _, dk, dv = oracle.bwd_rows(qh, kh, vh, doh, scale, causal, window=window)
                dk_ref += dk
                dv_ref += dv
                bq = 0.0
                if bounded:
                    bq, bk, bv = grad_rounding_bounds(qh, kh, vh, doh, scale, causal, window, dtype)
                    dk_bound += bk
                    dv_bound += bv
                got = grads_gpu["dq"][b, :, h, :].to(torch.float64).cpu().numpy()
                num["dq"] = max(num["dq"], excess(got, dq, bq))
                den["dq"] = max(den["dq"], float(np.abs(dq).max()))
            for name, ref, bound in (("dk", dk_ref, dk_bound), ("dv", dv_ref, dv_bound)):
                got = grads_gpu[name][b, :, hk, :].to(torch.float64).cpu().numpy()
                num[name] = max(num[name], excess(got, ref, bound))
                den[name] = max(den[name], float(np.abs(ref).max()))
    return {n: num[n] / max(den[n], GRAD_ABS_FLOOR) for n in num}


def decode_errors(inputs, o_gpu, lse_gpu, scale, causal, window=-1, heads=None):
    """(O error, LSE error) of a decode call against ``oracle.decode_rows`` over the given
    (b, h) pairs (default: all).  O: excess over half a bf16 ulp, as for the grouped rows;
    LSE: relative as everywhere, and -inf exactly where the oracle has -inf (no key seen)."""
    q = inputs["q"].double().numpy()
    k = inputs["k"].double().numpy()
    v = inputs["v"].double().numpy()
    o_ref, lse_ref = oracle.decode_rows(q, k, v, inputs["seqlens"].numpy(), scale, causal, window, heads=heads)
    B, n_q, H, _ = q.shape
    pairs = heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]
    o_g = o_gpu.cpu().double().numpy()
    l_g = lse_gpu.cpu().double().numpy()
    out_dtype = o_gpu.dtype
    worst_o, worst_l = 0.0, 0.0
    for b, h in pairs:
        og, orf = o_g[b, :, h], o_ref[b, :, h]
        lg, lrf = l_g[b, h], lse_ref[b, h]
        if not np.all(np.isfinite(og)):
            return float("inf"), float("inf")
        empty = np.isneginf(lrf)
        if not np.array_equal(np.isneginf(lg), empty):
            return float("inf"), float("inf")
        worst_o = max(worst_o, float((np.abs(og - orf) - half_ulp(orf, out_dtype)).max()))
        if (~empty).any():
            worst_l = max(worst_l, float((np.abs(lg[~empty] - lrf[~empty]) /
                                          np.maximum(1.0, np.abs(lrf[~empty]))).max()))
    return worst_o, worst_l


def e4m3_values(inputs, name: str) -> np.ndarray:
    """The fp64 values e4m3 codes stand for: code * descale (exact in fp64)."""
    return inputs[name].to(torch.float64).numpy() * float(inputs[name + "_descale"])


def fwd_errors_e4m3(inputs, o_gpu, lse_gpu, scale, causal, window=-1, rows_per_head=None, seed=0, heads=None):
    """Forward check for e4m3 inputs against the oracle on the dequantised values.

    The kernel rounds the softmax weights to e4m3 before the P.V product and normalises by
    their sum.  With w the exact weights of a row, p_j = 2^(x_j - m) for the kernel's
    reference maximum m (at most 8 below the row maximum, never above it) and e4m3 rounding
    error |p~_j - p_j| <= max(2^-4 p_j, 2^-10) (half an ulp in the normal range, half the
    subnormal spacing below 2^-6), the output obeys
        |O~_c - O_c| <= sum_j E_j |v_jc - O_c| / (1 - sum_j E_j),
        E_j = max(2^-4 w_j, 2^-10 w_max)   over the visible keys j,
    the worst case over m (m at the row maximum makes the absolute term largest).  Returns
    (largest excess of |O~ - O| over that bound plus half a bf16 ulp and an fp32 slack of
    1e-5 max|v| -- at most 0 when the bound holds --, largest |O~ - O|, LSE error)."""
    q, k, v = (e4m3_values(inputs, n) for n in ("q", "k", "v"))
    B, N, H, _ = q.shape
    group = H // k.shape[2]
    o_gpu, lse_gpu = o_gpu.cpu(), lse_gpu.cpu()
    heads = heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]
    excess, worst, worst_l = -np.inf, 0.0, 0.0
    for b, h in heads:
        qh, kh, vh = q[b, :, h], k[b, :, h // group], v[b, :, h // group]
        rows = sample_rows(N, rows_per_head, head_row_seed(seed, b, h)).numpy()
        o_ref, lse_ref = oracle.fwd_rows(qh, kh, vh, scale, causal, rows, window=window)
        o_g = o_gpu[b, rows, h, :].to(torch.float64).numpy()
        l_g = lse_gpu[b, h, rows].to(torch.float64).numpy()
        worst_l = max(worst_l, float((np.abs(l_g - lse_ref) / np.maximum(1.0, np.abs(lse_ref))).max()))
        slack = 1e-5 * np.abs(vh).max()
        for r, i in enumerate(rows):
            w = oracle.prob_row(qh, kh, scale, causal, int(i), window=window)
            j = np.arange(N)
            vis = (j <= i) if causal else np.ones(N, bool)
            if window >= 0:
                vis &= j >= i - window
            e = np.where(vis, np.maximum(2.0 ** -4 * w, 2.0 ** -10 * w.max()), 0.0)
            bound = (e @ np.abs(vh - o_ref[r])) / (1.0 - e.sum())
            err = np.abs(o_g[r] - o_ref[r])
            worst = max(worst, float(err.max()))
            excess = max(excess, float((err - bound - bf16_half_ulp(o_ref[r]) - slack).max()))
    return excess, worst, worst_l
