"""Comparison rules between the CUDA path and the CPU oracle.

Tolerance (per logit): |y_gpu - y_oracle| <= 2e-3 * ||h_t||_2 * max_j |W_hat[v, j]|
(fp32 accumulation).  LSE is 1-Lipschitz in the max-norm of the logits, so
|dLSE_t| <= max_v tol[t, v]; CE = LSE - y[target] gets twice that.  An argmax
may differ from the oracle's only where the oracle's gap between its maximum
and the chosen row is within the tolerance of those two rows.
"""
import numpy as np


def check_argmax_exact(am_gpu, expected, what="argmax"):
    """Exact comparison (no tolerance rule): used where the expected row is
    fixed by construction, e.g. equal maxima that must resolve to the lowest
    index."""
    am_gpu = np.asarray(am_gpu)
    bad = np.nonzero(am_gpu != np.asarray(expected))[0]
    assert bad.size == 0, f"{what}: token {bad[0]} gpu {am_gpu[bad[0]]}, expected {np.asarray(expected)[bad[0]]}"


def check_logits(y_gpu, y_ref, tol, what="logits"):
    err = np.abs(np.asarray(y_gpu, np.float64) - y_ref)
    ratio = err / tol
    worst = np.unravel_index(np.argmax(ratio), ratio.shape)
    assert np.all(np.isfinite(y_gpu)), f"{what}: non-finite values"
    assert ratio.max() <= 1.0, (f"{what}: max |err|/tol = {ratio.max():.3g} at {worst} "
                                f"(gpu {y_gpu[worst]!r}, oracle {y_ref[worst]!r}, tol {tol[worst]:.3g})")
    return float(ratio.max())


def check_argmax(am_gpu, y_ref, tol, what="argmax"):
    import oracle
    _, am_ref, _ = oracle.lse_argmax_ce(y_ref)
    for t, (a, b) in enumerate(zip(np.asarray(am_gpu), am_ref)):
        if a == b:
            continue
        assert 0 <= a < y_ref.shape[1], f"{what}[{t}] = {a} out of range"
        gap = y_ref[t, b] - y_ref[t, a]
        assert gap <= max(tol[t, a], tol[t, b]), f"{what}[{t}]: gpu {a}, oracle {b}, gap {gap:.3g}"


def check_lse_ce(lse_gpu, ce_gpu, y_ref, tol, targets=None):
    """LSE and CE against the oracle's own values (oracle.lse_argmax_ce).

    Bound: the logit tolerance (LSE is 1-Lipschitz in the max-norm of the
    logits) plus the fp32 evaluation of the log-sum-exp itself, a few units in
    the 24th bit of log(sum) (of order 1) and of the returned value: 2^-20 (1 +
    |LSE|).  The second term only matters when the logits are tiny against
    log V (a token with a very small norm)."""
    import oracle
    lse_ref, _, ce_ref = oracle.lse_argmax_ce(y_ref, None if ce_gpu is None else np.asarray(targets))
    bound = tol.max(axis=1) + 2.0 ** -20 * (1.0 + np.abs(lse_ref))
    d = np.abs(np.asarray(lse_gpu, np.float64) - lse_ref)
    assert np.all(d <= bound), f"lse: max |err|/bound = {(d / bound).max():.3g}"
    if ce_gpu is not None:
        d = np.abs(np.asarray(ce_gpu, np.float64) - ce_ref)
        assert np.all(d <= 2 * bound), f"ce: max |err|/bound = {(d / (2 * bound)).max():.3g}"


def check_build_properties(W_rows, comps, rows, T_p, g, g_B, fp16_decode, dequantize, what="build"):
    """Properties any correct build has, checkable on sampled head rows without
    the full truncated SVDs (used where the oracle cannot rebuild the head):
      * B_c has orthonormal rows, so R_hat R_hat^T = I up to INT8 rounding;
      * A_c = W V_c = W B_c^T: each L_hat row is within ~half an INT5 step of
        W[v] R_hat^T;
      * the SC4 codes quantise W - A_c B_c: their deviation from
        W[v] - (W[v] R_hat^T) R_hat is mostly far below half a step (the rest
        is R_hat's rounding);
      * the correction A_w B_w removes most of the activation-metric error
        ||(E - A_w B_w) T_p||^2 of Eq. 8 on those rows.
    The bounds were set with margin from heads the oracle builds."""
    Rh = dequantize(comps["R"], comps["s_R"], None)
    orth = np.abs(Rh @ Rh.T - np.eye(Rh.shape[0])).max()
    assert orth < 0.01, f"{what}: R_hat R_hat^T deviates from I by {orth:.3g}"
    Lh = dequantize(comps["L"][rows], comps["s_L"][rows], None)
    Ac = W_rows @ Rh.T
    sL = fp16_decode(comps["s_L"][rows])[:, None]
    dev_L = np.abs(Lh - Ac) / sL
    assert dev_L.max() < 0.6, f"{what}: L_hat off W R_hat^T by {dev_L.max():.3g} INT5 steps"
    Qh = dequantize(comps["q"][rows], comps["s_res"][rows], g)
    sres = np.repeat(fp16_decode(comps["s_res"][rows]), g, axis=1)
    dev_q = np.abs(Qh - (W_rows - Ac @ Rh)) / sres
    assert np.median(dev_q) < 0.3 and dev_q.max() < 2.0, (
        f"{what}: SC4 codes off the residual (median {np.median(dev_q):.3g}, max {dev_q.max():.3g} steps)")
    E = W_rows - (Lh @ Rh + Qh)
    corr = dequantize(comps["A"][rows], comps["s_A"][rows], None) @ dequantize(comps["B"], comps["s_B"], g_B)
    before = np.sum((E @ T_p) ** 2)
    after = np.sum(((E - corr) @ T_p) ** 2)
    assert after < 0.25 * before, f"{what}: the correction leaves {after / before:.3g} of the metric error"
