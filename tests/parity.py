"""Comparison helpers for the GPU-vs-oracle parity tests.

Tolerances (written here once, used by every parity test):
  * scores:    |I_gpu - I_ref| <= 1e-3 * max(|I_ref|, 1e-3 * max_s |I_ref[t, :]|)
  * selection: identical sets, except keys whose oracle score lies within 1e-3
               (relative) of the oracle k-th score; the GPU set must still hold
               exactly min(k, p+1) unique causal keys, ascending, -1 padded
  * attention: max-abs <= 2e-2, mean-abs <= 2e-3, relative L2 <= 1e-2 per row,
               and |o_gpu| > 0.5 |o_ref| (an all-zero output would otherwise pass);
               lse within 1e-4 absolute.
"""
from __future__ import annotations

import numpy as np

SCORE_RTOL = 1e-3
BAND_RTOL = 1e-3
ATT_MAX_ABS = 2e-2
ATT_MEAN_ABS = 2e-3
ATT_REL_L2 = 1e-2
LSE_ABS = 1e-4


def check_scores(gpu_row: np.ndarray, ref_row: np.ndarray, where=""):
    ref = np.asarray(ref_row, np.float64)
    got = np.asarray(gpu_row, np.float64)
    floor = 1e-3 * np.abs(ref).max() if ref.size else 0.0
    tol = SCORE_RTOL * np.maximum(np.abs(ref), floor)
    err = np.abs(got - ref)
    bad = np.nonzero(err > tol)[0]
    assert bad.size == 0, (f"{where}: {bad.size} scores out of tolerance, first s={bad[0]} "
                           f"gpu={got[bad[0]]} ref={ref[bad[0]]}")


def check_selection(gpu_idx: np.ndarray, ref_scores, ref_idx: np.ndarray, k: int, p: int, where=""):
    gpu_idx = np.asarray(gpu_idx, np.int64)
    n = p + 1
    v = gpu_idx[gpu_idx >= 0]
    m = min(k, n)
    assert len(v) == m, f"{where}: {len(v)} selected, expected {m}"
    assert (gpu_idx[m:] == -1).all(), f"{where}: padding"
    assert (np.diff(v) > 0).all(), f"{where}: not ascending/unique"
    assert v.min() >= 0 and v.max() <= p, f"{where}: non-causal index"
    r = ref_idx[ref_idx >= 0]
    if n <= k:
        assert np.array_equal(v, np.arange(n)), f"{where}: short row must select every key"
        return 0
    sc = np.asarray(ref_scores, np.float64)
    kth = np.sort(sc)[::-1][k - 1]
    band = np.abs(sc - kth) <= BAND_RTOL * abs(kth)
    diff = np.setxor1d(v, r)
    outside = diff[~band[diff]]
    assert outside.size == 0, (f"{where}: {outside.size} selection differences outside the tie band, "
                               f"e.g. s={outside[:5]} scores={sc[outside[:5]]} kth={kth}")
    return int(diff.size)


def check_attention(gpu_out, ref_out, gpu_lse=None, ref_lse=None, where=""):
    g = np.asarray(gpu_out, np.float64)
    r = np.asarray(ref_out, np.float64)
    err = np.abs(g - r)
    assert err.max() <= ATT_MAX_ABS, f"{where}: max abs err {err.max()}"
    assert err.mean() <= ATT_MEAN_ABS, f"{where}: mean abs err {err.mean()}"
    rn = np.linalg.norm(r, axis=-1)
    en = np.linalg.norm(g - r, axis=-1)
    ok = rn > 0
    if ok.any():
        rel = (en[ok] / rn[ok]).max()
        assert rel <= ATT_REL_L2, f"{where}: rel L2 err {rel}"
        assert (np.linalg.norm(g, axis=-1)[ok] > 0.5 * rn[ok]).all(), f"{where}: output collapsed"
    if gpu_lse is not None and ref_lse is not None:
        gl = np.asarray(gpu_lse, np.float64)
        rl = np.asarray(ref_lse, np.float64)
        fin = np.isfinite(rl)
        assert np.array_equal(np.isfinite(gl), fin), f"{where}: lse finiteness"
        if fin.any():
            lerr = np.abs(gl[fin] - rl[fin]).max()
            assert lerr <= LSE_ABS, f"{where}: lse err {lerr}"
    return float(err.max())


def bf16_to_f64(t) -> np.ndarray:
    import torch
    return t.detach().to("cpu", torch.float32).double().numpy()


# Indexer alignment target (KL). The GPU forms a = exp(z - lse) from fp32-accumulated
# bf16 logits and the forward's lse; the log-domain error of both together stays under
# 2e-4 (the attention tests bound lse to LSE_ABS = 1e-4), so p is within about 2e-4
# relative. Tolerances: p within KL_P_RTOL relative (plus a 1e-9 floor for p ~ 0);
# since dKL = sum_s dp_s (ln p_s - ln r_s + 1), KL within
# KL_P_RTOL * (1 + sum_s p_s (|ln p_s| + |ln r_s|)) of the oracle's value.
KL_P_RTOL = 1e-3


def check_kl(gpu_kl, gpu_p, ref_kl, ref_p, sel, idx, where=""):
    gk = float(gpu_kl)
    gp = np.asarray(gpu_p, np.float64)
    rp = np.asarray(ref_p, np.float64)
    ok = (np.asarray(idx) >= 0)
    assert np.all(gp[~ok] == 0.0), f"{where}: p outside the set"
    perr = np.abs(gp - rp)
    assert (perr <= KL_P_RTOL * rp + 1e-9).all(), f"{where}: p err {perr.max()} (rel {(perr / np.maximum(rp, 1e-30)).max()})"
    s = np.asarray(sel, np.float64)[ok]
    if ok.any():
        log_r = s - (s.max() + np.log(np.exp(s - s.max()).sum()))
        pp = rp[ok]
        nz = pp > 0
        bound = KL_P_RTOL * (1.0 + float(np.sum(pp[nz] * (np.abs(np.log(pp[nz])) + np.abs(log_r[nz])))))
    else:
        bound = 1e-12
    assert abs(gk - ref_kl) <= bound, f"{where}: kl {gk} vs {ref_kl} (bound {bound})"
    return abs(gk - ref_kl)


# ---------------------------------------------------------------------------
# Sparse-stage gradients
# ---------------------------------------------------------------------------
# Attention backward: P and dz enter their GEMMs rounded to bf16 (relative error at
# most 2^-9 each, independent from slot to slot) and D = dout . out uses the
# forward's bf16 output. Each gradient is a sum over up to 2048 slots in which
# these errors do not line up, so its relative error is of order 2^-9 ~ 2e-3.
# Bound: 1e-2 per row (a row under a tenth of the RMS row norm is held to 1e-2 of
# that tenth) and 5e-3 over the whole tensor.
GRAD_ATT_ROW = 1e-2
GRAD_ATT_ALL = 5e-3
# Indexer backward: fp64 contractions on exact code dots; fp32 only in the stored
# results and in the atomic sums of key gradients (2^-24 relative per addition, so
# about 2^-24 sqrt(n / 2) after n additions of random sign: 1e-6 at 2000 tokens).
GRAD_IDX_ROW = 1e-5
GRAD_IDX_ALL = 1e-5
# KL score gradient r - p: fp32 softmax of at most 4096 scores.
KL_GRAD_RTOL = 1e-4
KL_GRAD_ATOL = 1e-6


def check_grad(gpu, ref, row_tol, all_tol, where, floor=0.1):
    """Row-wise relative L2 error of a gradient (rows = the last axis), with rows
    under floor * the RMS row norm held to row_tol of that floor, plus the relative
    Frobenius error of the whole tensor. Returns the worst row ratio."""
    g = np.asarray(gpu, np.float64)
    r = np.asarray(ref, np.float64)
    g = g.reshape(-1, g.shape[-1])
    r = r.reshape(-1, r.shape[-1])
    assert g.shape == r.shape, where
    rn = np.linalg.norm(r, axis=1)
    en = np.linalg.norm(g - r, axis=1)
    rms = float(np.sqrt(np.mean(rn ** 2)))
    assert rms > 0, f"{where}: reference gradient is zero"
    den = np.maximum(rn, floor * rms)
    ratio = en / den
    bad = np.flatnonzero(ratio > row_tol)
    assert bad.size == 0, (f"{where}: {bad.size} of {rn.size} rows off, worst relative error "
                           f"{ratio.max():.3g} at row {int(np.argmax(ratio))}")
    tot = float(np.linalg.norm(g - r) / np.linalg.norm(r))
    assert tot <= all_tol, f"{where}: relative Frobenius error {tot:.3g}"
    return float(ratio.max())
