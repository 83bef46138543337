"""CPU oracle for the ARCHead packed LM-head (float64, numpy).

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  It shares no code
with the CUDA library (``quantized_output_head_b200``) and is never on the
product path.

Source: "ARCHead: Activation-Metric Residual Correction for Large Language
Model Output Heads" (arXiv 2608.02703), §3.1-§3.4.  Each function names the
section / equation it follows.  Every dequantised value is exact in float64
(an integer code times a decoded fp16 scale), so the forward pass below is the
plain definition of what the packed head computes:

    W_hat = Q5(A_c) Q8(B_c) + Q_SC4(residual) + A_w B_w       (Eq. 3 and Eq. 6)
    logits = h W_hat^T                                        (Eq. 7, evaluated densely)

Readings of points the pages leave open (each also listed in the design notes):
  * quantiser: symmetric, no zero point; scale = fp16(amax / qmax) with
    qmax = 7 (INT4), 15 (INT5), 127 (INT8); codes = clamp(rint(x / s)) using the
    fp16-rounded scale; amax = 0 gives scale 0 and codes 0.  Rounding is
    round-half-to-even.
  * the rank-r_c core A_c B_c is the unweighted truncated SVD of W, with the
    singular values on the left factor (A_c = U S, B_c = V^T), mirroring Eq. 5;
  * the SC4 residual is taken against the unquantised core, W - A_c B_c (Eq. 3
    as printed); its group scales are fp16;
  * the "randomised" truncated SVD of Eq. 4 is replaced by the exact SVD that
    it approximates (§3.2, remark after the proof);
  * a singular pair (u_i, v_i) is defined only up to a common sign; each is
    taken with the first largest-magnitude entry of v_i positive, so the
    quantised factors are a function of the head alone;
  * damping lambda = 1e-2 and metric power p = 0.75 unless given.

Parity pins (tests/test_oracle_pins.py) tie every function here to something
other than itself: Eckart-Young optimality in the T_p metric (Eq. 8-9), the
p = 1/2, lambda = 0 reduction to the empirical logit MSE (Eq. 1), the C = I
reduction to the Frobenius objective (§3.1), exact rational brute force of the
single-branch products, Eq. 6 vs Eq. 7 agreement, quantiser round-trip bounds,
the byte count of Eq. 10 against the built arrays, and log-sum-exp / argmax /
cross-entropy against scipy and Python loops.  The quality figures of the
pages (perplexity, top-1 agreement on real text) need weights and data that
are not available: parity unpinned for those, by construction.
"""
from __future__ import annotations

from typing import Dict, Optional, Tuple

import numpy as np

# ------------------------------------------------------------------ decoding
QRANGE = {4: (-8, 7), 5: (-16, 15), 8: (-128, 127)}
FP16_MAX = 65504.0


def fp16_decode(bits) -> np.ndarray:
    """IEEE binary16 bit patterns -> float64 (exact)."""
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def fp16_encode(x) -> np.ndarray:
    """float64 -> IEEE binary16 bit pattern, round to nearest even."""
    x = np.asarray(x, dtype=np.float64)
    if np.any(np.abs(x) > FP16_MAX):
        raise ValueError("value outside the fp16 range")
    return x.astype(np.float16).view(np.uint16)


def bf16_decode(bits) -> np.ndarray:
    """bfloat16 bit patterns -> float64 (exact): the 16 bits are the top half of a float32."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


# ---------------------------------------------------------------- quantisers
def quantize_symmetric(x: np.ndarray, bits: int, group: Optional[int]) -> Tuple[np.ndarray, np.ndarray]:
    """b-bit symmetric group quantiser Q_b of §3.2 (Eq. 3) and §3.3.

    x: [rows, cols] float64.  ``group`` = columns sharing one scale along a row;
    None means one scale per row.  Returns (codes int8 [rows, cols],
    scale bits uint16 [rows, cols // group]).
    """
    qmin, qmax = QRANGE[bits]
    rows, cols = x.shape
    if cols == 0:                # a rank-0 factor: no codes; its per-row scales are fp16(0) = 0
        return np.zeros((rows, 0), dtype=np.int8), np.zeros((rows, 1 if group is None else 0), dtype=np.uint16)
    G = cols if group is None else group
    if cols % G:
        raise ValueError("group size must divide the row length")
    xg = x.reshape(rows, cols // G, G)
    amax = np.abs(xg).max(axis=2)
    s_bits = fp16_encode(amax / qmax)
    s = fp16_decode(s_bits)
    codes = np.zeros_like(xg)
    nz = s > 0
    codes[nz] = np.clip(np.rint(xg[nz] / s[nz][:, None]), qmin, qmax)
    return codes.reshape(rows, cols).astype(np.int8), s_bits


def dequantize(codes: np.ndarray, s_bits: np.ndarray, group: Optional[int]) -> np.ndarray:
    """codes [rows, cols] x per-group fp16 scales -> float64 (exact)."""
    codes = np.asarray(codes)
    rows, cols = codes.shape
    if codes.size == 0:          # a rank-0 factor: the branch is an empty sum
        return np.zeros((rows, cols))
    s = fp16_decode(s_bits).reshape(rows, -1)
    G = cols if group is None else group
    return codes.astype(np.float64) * np.repeat(s, G, axis=1)


# ------------------------------------------------------- activation metric
def damped_metric(H: np.ndarray, lam: float, p: float):
    """§3.1: C = H^T H / N (Eq. 1), C_lam = C + lam * mean(diag C) * I = Q Lambda Q^T,
    T_p = Q Lambda^p Q^T and T_p^{-1} = Q Lambda^{-p} Q^T (Eq. 2)."""
    N = H.shape[0]
    C = H.T @ H / N
    c_bar = float(np.mean(np.diag(C)))
    C_lam = C + lam * c_bar * np.eye(C.shape[0])
    evals, Q = np.linalg.eigh(C_lam)
    if evals.min() <= 0:
        raise ValueError("damped covariance is not positive definite")
    T_p = (Q * evals ** p) @ Q.T
    T_p_inv = (Q * evals ** (-p)) @ Q.T
    return C, C_lam, T_p, T_p_inv


def truncated_svd(M: np.ndarray, r: int):
    """Rank-r truncated SVD (Eckart-Young), singular values descending; each
    pair's sign fixed so that the first largest-magnitude entry of the right
    singular vector is positive (the pages leave the sign open)."""
    U, S, Vt = np.linalg.svd(M, full_matrices=False)
    U, S, Vt = U[:, :r].copy(), S[:r], Vt[:r].copy()
    for i in range(Vt.shape[0]):
        if Vt[i, np.argmax(np.abs(Vt[i]))] < 0:
            U[:, i] = -U[:, i]
            Vt[i] = -Vt[i]
    return U, S, Vt


def correction_factors(E: np.ndarray, T_p: np.ndarray, T_p_inv: np.ndarray, r_r: int):
    """Eq. 4-5: E T_p ~ U S V^T (rank r_r), A_w = U S, B_w = V^T T_p^{-1}."""
    U, S, Vt = truncated_svd(E @ T_p, r_r)
    return U * S[None, :], Vt @ T_p_inv


def metric_objective(E: np.ndarray, A: np.ndarray, B: np.ndarray, T_p: np.ndarray) -> float:
    """Eq. 8: || (E - A B) T_p ||_F^2."""
    return float(np.sum(((E - A @ B) @ T_p) ** 2))


# ------------------------------------------------------------ construction
def build_packed_head(W: np.ndarray, H: np.ndarray, r_c: int, r_r: int, g: int, g_B: int,
                      p: float = 0.75, lam: float = 1e-2) -> Dict[str, np.ndarray]:
    """Packed-head construction of §3.4 (Algorithm 1), in the order of Eq. 2-5.

    Returns the canonical packed components (codes int8, scales fp16 bits) and,
    under keys starting with '_', the float64 intermediates used by the pins.
    """
    V, d = W.shape
    # Eq. 2: damped metric from the calibration activations.
    C, C_lam, T_p, T_p_inv = damped_metric(H, lam, p)
    # Eq. 3: rank-r_c core, quantised factors, SC4 residual.
    U, S, Vt = truncated_svd(W, r_c)
    A_c = U * S[None, :]
    B_c = Vt
    L, s_L = quantize_symmetric(A_c, 5, None)
    R, s_R = quantize_symmetric(B_c, 8, None)
    q, s_res = quantize_symmetric(W - A_c @ B_c, 4, g)
    W_d = dequantize(L, s_L, None) @ dequantize(R, s_R, None) + dequantize(q, s_res, g)
    # Eq. 4-5: activation-metric correction of what the core leaves.
    E = W - W_d
    A_w, B_w = correction_factors(E, T_p, T_p_inv, r_r)
    # INT8 factors: A_w per row, B_w per group of g_B along d (§3.2, last paragraph).
    A, s_A = quantize_symmetric(A_w, 8, None)
    B, s_B = quantize_symmetric(B_w, 8, g_B)
    return dict(L=L, s_L=s_L.reshape(V), R=R, s_R=s_R.reshape(r_c), q=q, s_res=s_res,
                A=A, s_A=s_A.reshape(V), B=B, s_B=s_B,
                _C=C, _C_lam=C_lam, _T_p=T_p, _T_p_inv=T_p_inv, _A_c=A_c, _B_c=B_c,
                _W_d=W_d, _E=E, _A_w=A_w, _B_w=B_w)


# ----------------------------------------------------------------- forward
def dequantized_factors(comp: Dict[str, np.ndarray], g: int, g_B: int):
    """Float64 values of the five stored matrices: L_hat, R_hat, Q_hat, A_hat, B_hat."""
    Lh = dequantize(comp["L"], comp["s_L"], None)
    Rh = dequantize(comp["R"], comp["s_R"], None)
    Qh = dequantize(comp["q"], comp["s_res"], g)
    Ah = dequantize(comp["A"], comp["s_A"], None)
    Bh = dequantize(comp["B"], comp["s_B"], g_B)
    return Lh, Rh, Qh, Ah, Bh


def w_hat_rows(comp: Dict[str, np.ndarray], g: int, g_B: int, rows: np.ndarray) -> np.ndarray:
    """Rows of W_hat = L_hat R_hat + Q_hat + A_hat B_hat (Eq. 3 + Eq. 6), float64."""
    Rh = dequantize(comp["R"], comp["s_R"], None)
    Bh = dequantize(comp["B"], comp["s_B"], g_B)
    Lh = dequantize(comp["L"][rows], comp["s_L"][rows], None)
    Qh = dequantize(comp["q"][rows], comp["s_res"][rows], g)
    Ah = dequantize(comp["A"][rows], comp["s_A"][rows], None)
    return Lh @ Rh + Qh + Ah @ Bh


def logits(comp: Dict[str, np.ndarray], g: int, g_B: int, h_bits: np.ndarray,
           rows: Optional[np.ndarray] = None, chunk: int = 4096):
    """Eq. 7 evaluated as the dense product h W_hat^T, W_hat formed row block by row block.

    Returns (y [T, n_rows] float64, rowmax [n_rows] = max_j |W_hat[v, j]|).
    """
    h = bf16_decode(h_bits)
    V = comp["L"].shape[0]
    rows = np.arange(V) if rows is None else np.asarray(rows)
    y = np.empty((h.shape[0], rows.size))
    rowmax = np.empty(rows.size)
    for i in range(0, rows.size, chunk):
        blk = w_hat_rows(comp, g, g_B, rows[i:i + chunk])
        y[:, i:i + chunk] = h @ blk.T
        rowmax[i:i + chunk] = np.abs(blk).max(axis=1)
    return y, rowmax


def logits_factored(comp: Dict[str, np.ndarray], g: int, g_B: int, h_bits: np.ndarray) -> np.ndarray:
    """Eq. 7 in its factored form: (h R_hat^T) L_hat^T + h Q_hat^T + (h B_hat^T) A_hat^T."""
    h = bf16_decode(h_bits)
    Lh, Rh, Qh, Ah, Bh = dequantized_factors(comp, g, g_B)
    return (h @ Rh.T) @ Lh.T + h @ Qh.T + (h @ Bh.T) @ Ah.T


def lse_argmax_ce(y: np.ndarray, targets: Optional[np.ndarray] = None):
    """Per token over the vocabulary: log-sum-exp, lowest index of the maximum,
    and cross-entropy LSE - y[target] (the head feeds softmax directly, §1)."""
    m = y.max(axis=1)
    lse = m + np.log(np.sum(np.exp(y - m[:, None]), axis=1))
    am = np.argmax(y, axis=1)          # numpy returns the first (lowest) index of the maximum
    ce = None
    if targets is not None:
        ce = lse - y[np.arange(y.shape[0]), np.asarray(targets)]
    return lse, am, ce


def tolerance(h_bits: np.ndarray, rowmax: np.ndarray, rel: float = 2e-3) -> np.ndarray:
    """Per-element logit tolerance rel * ||h_t||_2 * max_j |W_hat[v, j]|, shape [T, n_rows]."""
    hn = np.linalg.norm(bf16_decode(h_bits), axis=1)
    return rel * hn[:, None] * rowmax[None, :]


# ----------------------------------------------------------------- sampling
# Not part of the paper: temperature sampling from the head's logits by the
# Gumbel-max construction (argmax_v of y_v / tau + G_v with G_v independent
# standard Gumbel draws samples v with probability softmax(y / tau)_v), the
# definition behind the library's sampling entry point.  The draws come from
# Philox4x64-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy
# as 1, 2, 3", SC 2011), written here from that definition: ten rounds of two
# 64 x 64 -> 128-bit multiplies with the published multipliers, the key bumped
# by the published Weyl constants between rounds.
_PHILOX_M0, _PHILOX_M1 = np.uint64(0xD2E7470EE14C6C93), np.uint64(0xCA5A826395121157)
_PHILOX_W0, _PHILOX_W1 = np.uint64(0x9E3779B97F4A7C15), np.uint64(0xBB67AE8584CAA73B)
_M32 = np.uint64(0xFFFFFFFF)


def _mulhilo64(a: np.ndarray, b: np.uint64):
    """High and low 64-bit words of a * b (uint64, elementwise), from 32-bit limbs."""
    a = np.asarray(a, dtype=np.uint64)
    a0, a1 = a & _M32, a >> np.uint64(32)
    b0, b1 = np.uint64(int(b) & 0xFFFFFFFF), np.uint64(int(b) >> 32)
    p00, p01, p10, p11 = a0 * b0, a0 * b1, a1 * b0, a1 * b1
    mid = (p00 >> np.uint64(32)) + (p01 & _M32) + (p10 & _M32)
    lo = (p00 & _M32) | ((mid & _M32) << np.uint64(32))
    hi = p11 + (p01 >> np.uint64(32)) + (p10 >> np.uint64(32)) + (mid >> np.uint64(32))
    return hi, lo


def philox4x64(ctr0, ctr1, ctr2, ctr3, key0, key1, rounds: int = 10):
    """Philox4x64-R on uint64 arrays (broadcast): returns the four output words."""
    c = [np.asarray(x, dtype=np.uint64) for x in (ctr0, ctr1, ctr2, ctr3)]
    k0, k1 = np.asarray(key0, dtype=np.uint64), np.asarray(key1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        for _ in range(rounds):
            hi0, lo0 = _mulhilo64(c[0], _PHILOX_M0)
            hi1, lo1 = _mulhilo64(c[2], _PHILOX_M1)
            c = [hi1 ^ c[1] ^ k0, lo1, hi0 ^ c[3] ^ k1, lo0]
            k0, k1 = k0 + _PHILOX_W0, k1 + _PHILOX_W1
    return c


def gumbel_noise(seed: int, token_ids: np.ndarray, rows: np.ndarray) -> np.ndarray:
    """G[t, v] for global token ids and global vocabulary rows: word (v mod 4)
    of Philox4x64-10 at counter (token, v div 4, 0, 0), key (seed, 0); its top 23
    bits k give u = (k + 1/2) / 2^23 in (0, 1), and G = -log(-log(u))."""
    t = np.asarray(token_ids, dtype=np.uint64)[:, None]
    v = np.asarray(rows, dtype=np.uint64)[None, :]
    w = philox4x64(t, v >> np.uint64(2), 0, 0, np.uint64(seed), 0)
    sel = (v & np.uint64(3)).astype(np.int64)
    word = np.choose(np.broadcast_to(sel, np.broadcast_shapes(t.shape, v.shape)),
                     [np.broadcast_to(x, np.broadcast_shapes(t.shape, v.shape)) for x in w])
    u = ((word >> np.uint64(41)).astype(np.float64) + 0.5) / 2.0 ** 23
    return -np.log(-np.log(u))


def sample_gumbel(y: np.ndarray, temperature: float, seed: int, offset: int, row0: int = 0):
    """Sampled row per token (first maximum of y / tau + G) and the perturbed
    values z = y / tau + G.  Token t uses counter offset + t; rows are global
    (row0 + local index)."""
    y = np.asarray(y, dtype=np.float64)
    T, V = y.shape
    g = gumbel_noise(seed, offset + np.arange(T, dtype=np.uint64), row0 + np.arange(V, dtype=np.uint64))
    z = y / temperature + g
    return row0 + np.argmax(z, axis=1), z


# ------------------------------------------------------------- byte count
def component_bytes(V: int, d: int, r_c: int, r_r: int, g: int, g_B: int) -> Dict[str, int]:
    """numel x element size of every registered packed tensor (Eq. 10); INT5 and
    INT4 codes count 5/8 and 1/2 byte per element (the format's bit width)."""
    return dict(
        L=(V * r_c * 5 + 7) // 8, s_L=2 * V,
        R=r_c * d, s_R=2 * r_c,
        q=(V * d + 1) // 2, s_res=2 * V * (d // g),
        A=V * r_r, s_A=2 * V,
        B=r_r * d, s_B=2 * r_r * (d // g_B),
    )


def packed_bytes(V: int, d: int, r_c: int, r_r: int, g: int, g_B: int) -> int:
    """Eq. 10: bytes(ARCHead) = sum_i numel(theta_i) * element_size(theta_i)."""
    return sum(component_bytes(V, d, r_c, r_r, g, g_B).values())
