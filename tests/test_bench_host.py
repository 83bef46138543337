"""Host-side helpers of bench.py that need no GPU: the parity summary of a
timed run against the oracle, the CPU-baseline sample sizing and the split of
an oracle call into fixed and per-row time."""
import dataclasses

import numpy as np

import archead_inputs as gen
import bench
import oracle

SHAPE = gen.HeadShape(3000, 512, 64, 16, 128, 128)


def _case(T=3):
    comps = gen.random_components(SHAPE, 3)
    h_bits, _ = gen.random_hidden(SHAPE.d, T, 4, V=SHAPE.V)
    y, rowmax = oracle.logits(comps, SHAPE.g, SHAPE.g_B, h_bits)
    return comps, h_bits, y, rowmax


def test_parity_of_exact_outputs_and_a_planted_wrong_argmax():
    comps, h_bits, y, rowmax = _case()
    lse, am, _ = oracle.lse_argmax_ce(y)
    gpu = dict(logits=y.copy(), lse=lse.copy(), argmax=am.copy())
    p = bench.oracle_parity(oracle, SHAPE, h_bits, y, rowmax, gpu)
    assert p["rows"] == SHAPE.V and p["tokens"] == 3
    assert p["logits_max_err_over_tol"] == 0.0 and p["lse_max_err_over_tol"] == 0.0
    assert p["argmax_mismatches"] == 0
    gpu["argmax"][1] = (am[1] + 7) % SHAPE.V        # far from the maximum: beyond any tie
    gpu["argmax"][2] = -1                           # out of range
    assert bench.oracle_parity(oracle, SHAPE, h_bits, y, rowmax, gpu)["argmax_mismatches"] == 2


def test_parity_on_a_row_sample_compares_logits_only():
    comps, h_bits, y, rowmax = _case()
    n = 1000
    gpu = dict(logits=y.copy(), lse=None, argmax=np.argmax(y, axis=1).astype(np.int32))
    gpu["logits"][0, 5] += 10.0 * oracle.tolerance(h_bits, rowmax)[0, 5]
    p = bench.oracle_parity(oracle, SHAPE, h_bits, y[:, :n], rowmax[:n], gpu)
    assert p["rows"] == n and "argmax_mismatches" not in p
    assert 9.0 < p["logits_max_err_over_tol"] < 11.0
    p = bench.oracle_parity(oracle, SHAPE, h_bits, y[:, :n], rowmax[:n], dict(logits=None, argmax=gpu["argmax"]))
    assert "note" in p


def test_cpu_baseline_takes_the_whole_small_head_and_reports_parity(monkeypatch):
    comps, h_bits, y, rowmax = _case()
    lse, am, _ = oracle.lse_argmax_ce(y)
    monkeypatch.setattr(bench, "CPU_SAMPLE_SECONDS", 2.0)
    wl = dataclasses.replace(bench.workload(3, 2)[0], shape=SHAPE)
    cpu, parity = bench.cpu_baseline(3, wl, 3, comps, h_bits, dict(logits=None, lse=lse, argmax=am))
    assert cpu["kind"] == "oracle" and cpu["value"] > 0 and f"{SHAPE.V} of {SHAPE.V}" in cpu["sample"]
    assert "scaled" not in cpu["sample"]
    assert parity["argmax_mismatches"] == 0 and parity["lse_max_err_over_tol"] < 1e-6


def test_oracle_call_model_splits_fixed_and_per_row_time():
    comps, h_bits, _, _ = _case(T=1)
    t_fixed, t_row = bench.oracle_call_model(oracle, comps, SHAPE, h_bits, small=256, large=2048)
    assert t_fixed >= 0.0 and t_row > 0.0


def test_randomized_build_flops_add_the_sketch_products():
    """The randomised SVD's sketch is r + oversample columns, rounded up to a
    multiple of 64 above 64 and capped at d; each factorisation adds
    power_iters + 2 products G Q (2 d^2 k flops each) and two d x k x k ones."""
    assert bench.sketch_cols(4096, 512, 32) == 576
    assert bench.sketch_cols(4096, 64, 32) == 128
    assert bench.sketch_cols(256, 8, 0) == 8
    assert bench.sketch_cols(256, 240, 64) == 256
    V, d, r_c, r_r, N = 151936, 4096, 512, 64, 16384
    exact = bench.build_flops(V, d, r_c, r_r, N)
    rand = bench.build_flops(V, d, r_c, r_r, N, svd="randomized", oversample=32, power_iters=2)
    extra = sum(2 * d * d * k * 4 + 4 * d * k * k for k in (576, 128))
    assert rand - exact == extra
    # the default bench line: ~8.02 TFLOP of dense products
    assert abs(rand / 1e12 - 8.02) < 0.01
