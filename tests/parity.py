"""Comparison rules between the CUDA path and the CPU oracle.

Tolerance (per logit): |y_gpu - y_oracle| <= 2e-3 * ||h_t||_2 * max_j |W_hat[v, j]|
(fp32 accumulation).  LSE is 1-Lipschitz in the max-norm of the logits, so
|dLSE_t| <= max_v tol[t, v]; CE = LSE - y[target] gets twice that.  An argmax
may differ from the oracle's only where the oracle's gap between its maximum
and the chosen row is within the tolerance of those two rows.
"""
import numpy as np


def check_logits(y_gpu, y_ref, tol, what="logits"):
    err = np.abs(np.asarray(y_gpu, np.float64) - y_ref)
    ratio = err / tol
    worst = np.unravel_index(np.argmax(ratio), ratio.shape)
    assert np.all(np.isfinite(y_gpu)), f"{what}: non-finite values"
    assert ratio.max() <= 1.0, (f"{what}: max |err|/tol = {ratio.max():.3g} at {worst} "
                                f"(gpu {y_gpu[worst]!r}, oracle {y_ref[worst]!r}, tol {tol[worst]:.3g})")
    return float(ratio.max())


def check_argmax(am_gpu, y_ref, tol, what="argmax"):
    am_ref = np.argmax(y_ref, axis=1)
    for t, (a, b) in enumerate(zip(np.asarray(am_gpu), am_ref)):
        if a == b:
            continue
        assert 0 <= a < y_ref.shape[1], f"{what}[{t}] = {a} out of range"
        gap = y_ref[t, b] - y_ref[t, a]
        assert gap <= max(tol[t, a], tol[t, b]), f"{what}[{t}]: gpu {a}, oracle {b}, gap {gap:.3g}"


def check_lse_ce(lse_gpu, ce_gpu, y_ref, tol, targets=None):
    m = y_ref.max(axis=1)
    lse_ref = m + np.log(np.exp(y_ref - m[:, None]).sum(axis=1))
    bound = tol.max(axis=1)
    d = np.abs(np.asarray(lse_gpu, np.float64) - lse_ref)
    assert np.all(d <= bound), f"lse: max |err|/bound = {(d / bound).max():.3g}"
    if ce_gpu is not None:
        ce_ref = lse_ref - y_ref[np.arange(y_ref.shape[0]), np.asarray(targets)]
        d = np.abs(np.asarray(ce_gpu, np.float64) - ce_ref)
        assert np.all(d <= 2 * bound), f"ce: max |err|/bound = {(d / (2 * bound)).max():.3g}"
