"""Pins that tie the CPU oracle to the pages' mathematics (no GPU).

Source: "ARCHead: Activation-Metric Residual Correction for Large Language
Model Output Heads", §3.1-§3.3, Eq. 1-10.  Each test checks the oracle against
something other than itself: IEEE bit patterns, exact rational arithmetic,
Eckart-Young (via a symmetric eigensolver, not the SVD the oracle uses),
scipy's logsumexp, Python loops, and the figures printed on the pages.  The
mutation tests at the end plant plausible mistakes in the oracle and check that
some pin catches each one.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import scipy.special

import archead_inputs as gen
import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- encodings
@pytest.mark.parametrize("bits,value", [
    (0x3C00, 1.0), (0xC000, -2.0), (0x7BFF, 65504.0), (0x0001, 2.0 ** -24),
    (0x0400, 2.0 ** -14), (0x3555, 0.333251953125), (0x8000, -0.0),
])
def test_fp16_decode_ieee(bits, value):
    assert oracle.fp16_decode(np.array([bits], np.uint16))[0] == value


@pytest.mark.parametrize("bits,value", [
    (0x3F80, 1.0), (0xC040, -3.0), (0x0001, 2.0 ** -133), (0x7F7F, (2 - 2 ** -7) * 2.0 ** 127),
    (0x3E80, 0.25),
])
def test_bf16_decode_ieee(bits, value):
    assert oracle.bf16_decode(np.array([bits], np.uint16))[0] == value


# ---------------------------------------------------------------- quantiser
def test_quantizer_hand_example_half_even():
    # amax 14 with INT4 (qmax 7) gives scale exactly 2; 5/2 and 1/2 are ties -> even.
    codes, s = oracle.quantize_symmetric(np.array([[14.0, 5.0, -5.0, 1.0]]), 4, None)
    assert oracle.fp16_decode(s)[0, 0] == 2.0
    assert codes.tolist() == [[7, 2, -2, 0]]


def test_quantizer_zero_group():
    codes, s = oracle.quantize_symmetric(np.zeros((2, 8)), 8, 4)
    assert (codes == 0).all() and (s == 0).all()


@pytest.mark.parametrize("bits,group", [(4, 16), (5, None), (8, None), (8, 8)])
def test_quantizer_roundtrip_bound(bits, group):
    rng = np.random.default_rng(3)
    x = rng.standard_normal((37, 64)) * np.exp(rng.standard_normal((37, 1)))
    codes, s_bits = oracle.quantize_symmetric(x, bits, group)
    qmin, qmax = oracle.QRANGE[bits]
    assert codes.min() >= qmin and codes.max() <= qmax
    G = 64 if group is None else group
    s = np.repeat(oracle.fp16_decode(s_bits), G, axis=1)
    amax = np.repeat(np.abs(x.reshape(37, -1, G)).max(axis=2), G, axis=1)
    # the fp16 scale is the nearest half to amax / qmax (relative error <= 2^-11)
    assert np.all(np.abs(s - amax / qmax) <= 2.0 ** -11 * amax / qmax)
    err = np.abs(x - oracle.dequantize(codes, s_bits, group))
    assert np.all(err <= s / 2 + 2.0 ** -10 * np.abs(x))


# --------------------------------------------------------- activation metric
def _aniso(n, d, seed):
    rng = np.random.default_rng(seed)
    Q, _ = np.linalg.qr(rng.standard_normal((d, d)))
    lam = 10.0 * np.arange(1, d + 1) ** -1.5
    return (rng.standard_normal((n, d)) * np.sqrt(lam)) @ Q.T


def test_metric_half_power_undamped_is_logit_mse():
    """Eq. 1 and Eq. 2: with p = 1/2 and lambda = 0, ||Delta T_p||_F^2 = (1/N)||H Delta^T||_F^2."""
    H = _aniso(512, 24, 0)
    Delta = np.random.default_rng(1).standard_normal((40, 24))
    _, _, T_half, _ = oracle.damped_metric(H, 0.0, 0.5)
    lhs = np.sum((Delta @ T_half) ** 2)
    rhs = np.sum((H @ Delta.T) ** 2) / H.shape[0]
    assert abs(lhs - rhs) <= 1e-10 * rhs


def test_metric_powers_compose():
    H = _aniso(300, 16, 2)
    _, C_lam, T_p, T_inv = oracle.damped_metric(H, 0.3, 0.75)
    _, _, T_1, _ = oracle.damped_metric(H, 0.3, 1.0)
    np.testing.assert_allclose(T_p @ T_inv, np.eye(16), atol=1e-10)
    np.testing.assert_allclose(T_1, C_lam, rtol=1e-10, atol=1e-12)
    # damping adds lambda * mean(diag C) on the diagonal
    C = H.T @ H / H.shape[0]
    np.testing.assert_allclose(C_lam - C, 0.3 * np.mean(np.diag(C)) * np.eye(16), atol=1e-12)


def test_identity_metric_is_plain_truncated_svd():
    """§3.1: C = I is the Frobenius objective, so the correction is the plain truncated SVD of E."""
    rng = np.random.default_rng(4)
    N, d, r = 256, 20, 3
    Qn, _ = np.linalg.qr(rng.standard_normal((N, d)))
    H = Qn * math.sqrt(N)                       # H^T H / N = I
    E = rng.standard_normal((30, d))
    _, _, T_p, T_inv = oracle.damped_metric(H, 0.0, 0.75)
    A, B = oracle.correction_factors(E, T_p, T_inv, r)
    # best rank-r approximation in Frobenius norm, from the eigenvectors of E^T E
    w, Vv = np.linalg.eigh(E.T @ E)
    top = Vv[:, np.argsort(w)[::-1][:r]]
    np.testing.assert_allclose(A @ B, E @ top @ top.T, atol=1e-9)


def test_truncated_svd_sign_convention():
    """Singular pairs are fixed up to a joint sign: with known singular vectors
    whose largest entries are negative, the oracle returns them negated on
    both sides (product unchanged, largest entry of each v_i positive)."""
    rng = np.random.default_rng(12)
    m, n, r = 40, 12, 4
    U0, _ = np.linalg.qr(rng.standard_normal((m, n)))
    V0, _ = np.linalg.qr(rng.standard_normal((n, n)))
    for i in range(n):                          # make each column's largest entry negative
        if V0[np.argmax(np.abs(V0[:, i])), i] > 0:
            V0[:, i] = -V0[:, i]
    s = np.array([9.0, 7.0, 5.0, 3.0] + [1.0 / (k + 2) for k in range(n - 4)])
    M = (U0 * s) @ V0.T
    U, S, Vt = oracle.truncated_svd(M, r)
    np.testing.assert_allclose(S, s[:r], rtol=1e-12)
    np.testing.assert_allclose(Vt, -V0[:, :r].T, atol=1e-10)
    np.testing.assert_allclose(U, -U0[:, :r], atol=1e-10)
    for i in range(r):
        assert Vt[i, np.argmax(np.abs(Vt[i]))] > 0
    # the sign choice leaves the best rank-r approximation unchanged
    np.testing.assert_allclose((U * S) @ Vt, (U0[:, :r] * s[:r]) @ V0[:, :r].T, atol=1e-10)


def _ey_case(seed=5, V=48, d=24, r=4):
    rng = np.random.default_rng(seed)
    H = _aniso(400, d, seed + 1)
    E = rng.standard_normal((V, d)) * 0.01
    _, _, T_p, T_inv = oracle.damped_metric(H, 1e-2, 0.75)
    return E, T_p, T_inv, r


def test_eckart_young_closed_form():
    """Eq. 8-9: the minimum over rank-r products equals the tail energy of E T_p."""
    E, T_p, T_inv, r = _ey_case()
    A, B = oracle.correction_factors(E, T_p, T_inv, r)
    Et = E @ T_p
    ev = np.sort(np.linalg.eigvalsh(Et.T @ Et))[::-1]   # sigma_i^2, by a symmetric eigensolver
    tail = float(np.sum(ev[r:]))
    assert abs(oracle.metric_objective(E, A, B, T_p) - tail) <= 1e-9 * np.sum(ev)


def test_eckart_young_brute_force():
    E, T_p, T_inv, r = _ey_case(7)
    A, B = oracle.correction_factors(E, T_p, T_inv, r)
    best = oracle.metric_objective(E, A, B, T_p)
    rng = np.random.default_rng(8)
    for _ in range(1000):
        Ar = rng.standard_normal(A.shape) * A.std()
        Br = rng.standard_normal(B.shape) * B.std()
        assert oracle.metric_objective(E, Ar, Br, T_p) >= best
    for eps in (1e-3, 1e-2):
        for _ in range(200):
            dA = rng.standard_normal(A.shape) * eps * np.abs(A).max()
            dB = rng.standard_normal(B.shape) * eps * np.abs(B).max()
            assert oracle.metric_objective(E, A + dA, B + dB, T_p) >= best * (1 - 1e-12)


# ----------------------------------------------------- exact single branches
def _F(x):
    return Fraction(float(x))


def _tiny_components(V=3, d=32, r_c=4, r_r=2, g=16, g_B=8, seed=11):
    return gen.random_components(gen.HeadShape(V, d, r_c, r_r, g, g_B), seed)


def _exact_logits(comp, h_bits, g, g_B, branches):
    """Rational-arithmetic logits of the selected branches, by Python loops."""
    h = [[_F(v) for v in row] for row in oracle.bf16_decode(h_bits)]
    V, d = comp["q"].shape
    r_c, r_r = comp["L"].shape[1], comp["A"].shape[1]
    s16 = lambda b: _F(oracle.fp16_decode(np.array([b], np.uint16))[0])
    out = []
    for ht in h:
        row = []
        for v in range(V):
            acc = Fraction(0)
            if "core" in branches:
                for k in range(r_c):
                    z = s16(comp["s_R"][k]) * sum(int(comp["R"][k, j]) * ht[j] for j in range(d))
                    acc += s16(comp["s_L"][v]) * int(comp["L"][v, k]) * z
            if "res" in branches:
                for j in range(d):
                    acc += s16(comp["s_res"][v, j // g]) * int(comp["q"][v, j]) * ht[j]
            if "corr" in branches:
                for k in range(r_r):
                    z = sum(s16(comp["s_B"][k, j // g_B]) * int(comp["B"][k, j]) * ht[j] for j in range(d))
                    acc += s16(comp["s_A"][v]) * int(comp["A"][v, k]) * z
            row.append(acc)
        out.append(row)
    return out


def _zero_branches(comp, keep):
    c = {k: v.copy() for k, v in comp.items()}
    if "core" not in keep:
        c["L"][:] = 0
    if "res" not in keep:
        c["q"][:] = 0
    if "corr" not in keep:
        c["A"][:] = 0
    return c


@pytest.mark.parametrize("keep", [("core",), ("res",), ("corr",), ("core", "res", "corr")])
def test_branches_match_exact_rational(keep):
    comp = _zero_branches(_tiny_components(), keep)
    h_bits, _ = gen.random_hidden(32, 2, seed=12)
    y, _ = oracle.logits(comp, 16, 8, h_bits)
    exact = _exact_logits(comp, h_bits, 16, 8, keep)
    for t in range(2):
        for v in range(3):
            e = float(exact[t][v])
            assert abs(y[t, v] - e) <= 1e-12 * max(1e-300, abs(e)) + 1e-18


def test_zero_residual_and_correction_is_core_product():
    """Eq. 3 + Eq. 6 with q = 0 and A = 0: logits = (h R_hat^T) L_hat^T, by integer matmuls."""
    comp = _zero_branches(_tiny_components(V=17, d=64, r_c=8, r_r=4), ("core",))
    h_bits, _ = gen.random_hidden(64, 3, seed=13)
    y, _ = oracle.logits(comp, 16, 8, h_bits)
    h = oracle.bf16_decode(h_bits)
    sR = oracle.fp16_decode(comp["s_R"])
    sL = oracle.fp16_decode(comp["s_L"])
    z = (h @ comp["R"].astype(np.int64).T.astype(np.float64)) * sR[None, :]
    ref = (z @ comp["L"].astype(np.float64).T) * sL[None, :]
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-15)


def test_rank_zero_branches_are_empty_sums():
    """r_c = r_r = 0: only the SC4 residual remains (Eq. 3 and Eq. 6 with empty factors)."""
    comp = gen.random_components(gen.HeadShape(16, 64, 0, 0, 16, 1), 2)
    h_bits, _ = gen.random_hidden(64, 2, seed=3)
    y, _ = oracle.logits(comp, 16, 1, h_bits)
    exact = _exact_logits(comp, h_bits, 16, 1, ("res",))
    for t in range(2):
        for v in range(16):
            e = float(exact[t][v])
            assert abs(y[t, v] - e) <= 1e-12 * abs(e) + 1e-18


def test_factored_equals_dense():
    """Eq. 6 (dense W_hat) and Eq. 7 (factored) give the same logits."""
    comp = gen.random_components(gen.HeadShape(300, 256, 32, 8, 64, 64), 21)
    h_bits, _ = gen.random_hidden(256, 5, seed=22)
    y, _ = oracle.logits(comp, 64, 64, h_bits, chunk=97)
    yf = oracle.logits_factored(comp, 64, 64, h_bits)
    np.testing.assert_allclose(y, yf, rtol=1e-12, atol=1e-12 * np.abs(y).max())


# ------------------------------------------------------------ construction
@pytest.fixture(scope="module")
def built_cfg1():
    W, H, h_bits, targets = gen.dense_head_inputs()
    comp = oracle.build_packed_head(W, H, r_c=32, r_r=8, g=64, g_B=64, p=0.75, lam=1e-2)
    return W, H, h_bits, targets, comp


def test_builder_codes_and_shapes(built_cfg1):
    W, H, h_bits, targets, c = built_cfg1
    expect = dict(L=(1024, 32), s_L=(1024,), R=(32, 256), s_R=(32,), q=(1024, 256), s_res=(1024, 4),
                  A=(1024, 8), s_A=(1024,), B=(8, 256), s_B=(8, 4))
    for k, shp in expect.items():
        assert c[k].shape == shp, k
    for k, bits in (("L", 5), ("R", 8), ("q", 4), ("A", 8), ("B", 8)):
        lo, hi = oracle.QRANGE[bits]
        assert c[k].min() >= lo and c[k].max() <= hi


def test_builder_core_is_best_rank_rc(built_cfg1):
    """Eq. 3 reading: A_c B_c is the unweighted best rank-r_c approximation of W."""
    W, _, _, _, c = built_cfg1
    ev = np.sort(np.linalg.eigvalsh(W.T @ W))[::-1]
    err = np.sum((W - c["_A_c"] @ c["_B_c"]) ** 2)
    assert abs(err - np.sum(ev[32:])) <= 1e-8 * np.sum(ev)


def test_builder_correction_is_metric_optimal(built_cfg1):
    """Eq. 8: the unquantised correction attains the tail energy of E T_p, and the
    INT8 correction still lowers the metric error of the core."""
    _, _, _, _, c = built_cfg1
    E, T_p = c["_E"], c["_T_p"]
    Et = E @ T_p
    ev = np.sort(np.linalg.eigvalsh(Et.T @ Et))[::-1]
    opt = oracle.metric_objective(E, c["_A_w"], c["_B_w"], T_p)
    assert abs(opt - np.sum(ev[8:])) <= 1e-8 * np.sum(ev)
    Aq = oracle.dequantize(c["A"], c["s_A"], None)
    Bq = oracle.dequantize(c["B"], c["s_B"], 64)
    base = oracle.metric_objective(E, np.zeros_like(Aq), np.zeros_like(Bq), T_p)
    quant = oracle.metric_objective(E, Aq, Bq, T_p)
    assert opt < quant < base


def test_builder_wd_matches_components(built_cfg1):
    W, _, _, _, c = built_cfg1
    Lh, Rh, Qh, Ah, Bh = oracle.dequantized_factors(c, 64, 64)
    np.testing.assert_allclose(c["_W_d"], Lh @ Rh + Qh, rtol=0, atol=1e-14)
    np.testing.assert_allclose(c["_E"], W - c["_W_d"], rtol=0, atol=1e-14)


def test_built_head_logits_close_to_dense(built_cfg1):
    """The packed head approximates W's logits on held-out anisotropic states."""
    W, H, h_bits, _, c = built_cfg1
    y, _ = oracle.logits(c, 64, 64, h_bits)
    y_dense = oracle.bf16_decode(h_bits) @ W.T
    y_core, _ = oracle.logits(_zero_branches(c, ("core", "res")), 64, 64, h_bits)
    err_full = np.sum((y - y_dense) ** 2)
    err_core = np.sum((y_core - y_dense) ** 2)
    assert err_full < err_core


# --------------------------------------------------------------- byte count
def test_packed_bytes_equals_built_arrays(built_cfg1):
    """Eq. 10: sum of numel * element size over the registered arrays (INT5 at 5 bits, INT4 at 4)."""
    _, _, _, _, c = built_cfg1
    bits = dict(L=5, R=8, q=4, A=8, B=8, s_L=16, s_R=16, s_res=16, s_A=16, s_B=16)
    total_bits = sum(c[k].size * b for k, b in bits.items())
    assert total_bits % 8 == 0
    assert oracle.packed_bytes(1024, 256, 32, 8, 64, 64) == total_bits // 8 == 182400


def test_pages_dense_head_size():
    """The pages' Qwen3-8B head: 151,936 x 4,096 in BF16 is 1187 MB (MiB).  The
    printed "GB" figures (1.18, 1.28) are MiB / 1000 truncated to two decimals."""
    pn = json.load(open(os.path.join(GOLDEN, "page_numbers.json")))
    V, d = pn["qwen3_8b_head_shape"]["V"], pn["qwen3_8b_head_shape"]["d"]
    mib = V * d * 2 / 2 ** 20
    assert round(mib) == pn["qwen3_8b_dense_bf16_mib"]["value"]
    assert math.floor(mib / 10) / 100 == pn["qwen3_8b_dense_bf16_gb_approx"]["value"]
    gm = pn["gemma_4_e4b_head_shape_assumed"]
    gmib = gm["V"] * gm["d"] * 2 / 2 ** 20
    assert math.floor(gmib / 10) / 100 == pn["gemma_4_e4b_dense_bf16_gb_approx"]["value"]
    # the printed compression ratio is the quotient of the two printed sizes
    assert abs(1187.0 / pn["qwen3_8b_packed_mib"]["value"] - pn["qwen3_8b_packed_mib"]["ratio"]) < 2e-3


def test_packed_bytes_configs_fraction():
    """At the Qwen shape the fp16 group-128 scales alone put the packed head above
    the pages' 25-27% band; the format arithmetic is checked against the array sizes."""
    qwen = oracle.packed_bytes(151936, 4096, 512, 64, 128, 128)
    parts = oracle.component_bytes(151936, 4096, 512, 64, 128, 128)
    assert parts["q"] == 151936 * 4096 // 2 and parts["L"] == 151936 * 512 * 5 // 8
    assert qwen == 382204416
    assert oracle.packed_bytes(262144, 2560, 384, 64, 128, 128) == 427920640


# --------------------------------------------------------- LSE / argmax / CE
def test_lse_argmax_ce_against_scipy_and_loops():
    rng = np.random.default_rng(31)
    y = rng.standard_normal((4, 257)) * 7
    y[2, 10] = y[2, 200] = y[2].max() + 1.0       # tie: lowest index wins
    targets = np.array([0, 5, 200, 256])
    lse, am, ce = oracle.lse_argmax_ce(y, targets)
    np.testing.assert_allclose(lse, scipy.special.logsumexp(y, axis=1), rtol=1e-14)
    for t in range(4):
        row = list(y[t])
        best = max(range(len(row)), key=lambda i: (row[i], -i))
        assert am[t] == best
        m = max(row)
        loop_lse = m + math.log(math.fsum(math.exp(v - m) for v in row))
        assert abs(ce[t] - (loop_lse - row[targets[t]])) <= 1e-12 * max(1.0, abs(loop_lse))
    assert am[2] == 10


def test_tolerance_formula():
    h_bits = gen.f32_to_bf16_bits(np.array([[3.0, 4.0]], np.float32))
    tol = oracle.tolerance(h_bits, np.array([0.5, 2.0]))
    np.testing.assert_allclose(tol, [[2e-3 * 5 * 0.5, 2e-3 * 5 * 2.0]])


# ------------------------------------------------------------ planted mistakes
def _mutant_group_index(comp, g, g_B, rows):
    # wrong: scale index j % (d/g) instead of j // g
    Rh = oracle.dequantize(comp["R"], comp["s_R"], None)
    Bh = oracle.dequantize(comp["B"], comp["s_B"], g_B)
    Lh = oracle.dequantize(comp["L"][rows], comp["s_L"][rows], None)
    s = oracle.fp16_decode(comp["s_res"][rows])
    d = comp["q"].shape[1]
    Qh = comp["q"][rows].astype(np.float64) * np.tile(s, (1, g))[:, :d]
    Ah = oracle.dequantize(comp["A"][rows], comp["s_A"][rows], None)
    return Lh @ Rh + Qh + Ah @ Bh


def _mutant_drop_correction(comp, g, g_B, rows):
    Rh = oracle.dequantize(comp["R"], comp["s_R"], None)
    Lh = oracle.dequantize(comp["L"][rows], comp["s_L"][rows], None)
    Qh = oracle.dequantize(comp["q"][rows], comp["s_res"][rows], g)
    return Lh @ Rh + Qh


def _mutant_sign(comp, g, g_B, rows):
    Rh = oracle.dequantize(comp["R"], comp["s_R"], None)
    Bh = oracle.dequantize(comp["B"], comp["s_B"], g_B)
    Lh = oracle.dequantize(comp["L"][rows], comp["s_L"][rows], None)
    Qh = oracle.dequantize(comp["q"][rows], comp["s_res"][rows], g)
    Ah = oracle.dequantize(comp["A"][rows], comp["s_A"][rows], None)
    return Lh @ Rh - Qh + Ah @ Bh


@pytest.mark.parametrize("mutant", [_mutant_group_index, _mutant_drop_correction, _mutant_sign])
def test_planted_forward_mistakes_are_caught(monkeypatch, mutant):
    from oracle import archead_oracle as ao
    monkeypatch.setattr(ao, "w_hat_rows", mutant)
    comp = _tiny_components()
    h_bits, _ = gen.random_hidden(32, 2, seed=12)
    y, _ = ao.logits(comp, 16, 8, h_bits)
    exact = _exact_logits(comp, h_bits, 16, 8, ("core", "res", "corr"))
    worst = max(abs(y[t, v] - float(exact[t][v])) / abs(float(exact[t][v]))
                for t in range(2) for v in range(3))
    assert worst > 1e-6


def test_planted_mapback_mistake_is_caught():
    """Using T_p instead of T_p^{-1} in the map-back of Eq. 5 misses the Eckart-Young optimum."""
    E, T_p, T_inv, r = _ey_case(9)
    U, S, Vt = oracle.truncated_svd(E @ T_p, r)
    wrong = oracle.metric_objective(E, U * S, Vt @ T_p, T_p)
    Et = E @ T_p
    ev = np.sort(np.linalg.eigvalsh(Et.T @ Et))[::-1]
    assert wrong > np.sum(ev[r:]) * (1 + 1e-6)


# ------------------------------------------------------------- sampling
def test_philox4x64_matches_numpys_bit_generator():
    """The oracle's Philox4x64-10 (written from its definition) against numpy's
    Philox bit generator, which increments its 256-bit counter before each block."""
    rng = np.random.default_rng(5)
    for _ in range(6):
        c0, c1, c2 = (int(x) for x in rng.integers(1, 2**63, size=3, dtype=np.int64))
        k = rng.integers(0, 2**63, size=2, dtype=np.int64).astype(np.uint64) * np.uint64(2) + np.uint64(1)
        bg = np.random.Philox(counter=np.array([c0 - 1, c1, c2, 0], dtype=np.uint64), key=k)
        ref = bg.random_raw(4)
        got = oracle.philox4x64(c0, c1, c2, 0, k[0], k[1])
        assert [int(x) for x in got] == [int(x) for x in ref]


def test_gumbel_max_draws_follow_softmax():
    """40000 seeded draws over six logits: chi-square against softmax(y / tau)."""
    y = np.array([0.3, -1.2, 2.0, 0.5, 0.0, 1.1])
    tau, T = 0.8, 40000
    idx, _ = oracle.sample_gumbel(np.tile(y, (T, 1)), tau, seed=1234567, offset=10)
    p = np.exp(y / tau - (y / tau).max())
    p /= p.sum()
    counts = np.bincount(idx, minlength=y.size)
    chi2 = float((((counts - T * p) ** 2) / (T * p)).sum())
    assert chi2 < 20.5   # 99.9 % point of chi-square with 5 degrees of freedom


def test_gumbel_sampling_invariants():
    rng = np.random.default_rng(9)
    y = rng.normal(size=(50, 300)) * 3
    a, _ = oracle.sample_gumbel(y, 0.7, seed=42, offset=1000)
    b, _ = oracle.sample_gumbel(y + 7.25, 0.7, seed=42, offset=1000)       # softmax is shift invariant
    assert np.array_equal(a, b)
    c, _ = oracle.sample_gumbel(y, 1e-4, seed=42, offset=1000)              # tau -> 0: the argmax
    assert np.array_equal(c, np.argmax(y, axis=1))
    d, _ = oracle.sample_gumbel(y[:, 100:], 0.7, seed=42, offset=1000, row0=100)   # global rows
    assert np.all((d >= 100) & (d < 300))
    g = oracle.gumbel_noise(42, np.arange(3, dtype=np.uint64), np.arange(8, dtype=np.uint64))
    assert np.all(np.isfinite(g))


def test_build_properties_hold_for_the_oracle_build():
    """The sampled-row properties the full-size GPU build is held to hold for
    a head the oracle builds (so the bounds are the construction's, not the
    GPU's)."""
    from parity import check_build_properties
    V, d = 4096, 1024
    W, H, _, _ = gen.dense_head_inputs(n_calib=8192, V=V, d=d, seed_cfg=7)
    b = oracle.build_packed_head(W, H, r_c=128, r_r=16, g=128, g_B=128)
    comps = {k: v for k, v in b.items() if not k.startswith("_")}
    rows = np.random.default_rng(3).choice(V, 256, replace=False)
    check_build_properties(W[rows], comps, rows, b["_T_p"], 128, 128, oracle.fp16_decode, oracle.dequantize)
    # a transposed core (A_c from the wrong side) must fail them
    bad = dict(comps, R=np.ascontiguousarray(comps["R"][::-1]))
    with pytest.raises(AssertionError):
        check_build_properties(W[rows], bad, rows, b["_T_p"], 128, 128, oracle.fp16_decode, oracle.dequantize)
