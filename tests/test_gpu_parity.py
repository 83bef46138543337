"""GPU parity: the CUDA path against the float64 CPU oracle, element by element.

Every call goes through the C ABI of libarchead.so (via the ctypes binding).
Inputs are the seeded synthetic workloads of archead_inputs; expected values
come only from oracle/.  Rules (tests/parity.py): per-logit tolerance
2e-3 * ||h_t|| * max_j |W_hat[v, j]|, LSE within the row's largest tolerance,
CE within twice that, argmax exact unless the oracle's gap is within tolerance.
"""
import numpy as np
import pytest
import torch

import archead_inputs as gen
import oracle
from parity import check_argmax, check_argmax_exact, check_lse_ce, check_logits

pytestmark = pytest.mark.gpu

QWEN = (151936, 4096, 512, 64, 128, 128)
GEMMA = (262144, 2560, 384, 64, 128, 128)


@pytest.fixture(scope="module")
def qoh():
    import quantized_output_head_b200 as m
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return m


def _dev_hidden(h_bits):
    return torch.from_numpy(h_bits.view(np.int16)).cuda()


def _oracle(comps, shape, h_bits):
    y, rowmax = oracle.logits(comps, shape[4], shape[5], h_bits)
    return y, oracle.tolerance(h_bits, rowmax)


# ------------------------------------------------------------- config 1
@pytest.fixture(scope="module")
def cfg1(qoh):
    W, H, h_bits, targets = gen.dense_head_inputs()
    built = oracle.build_packed_head(W, H, r_c=32, r_r=8, g=64, g_B=64, p=0.75, lam=1e-2)
    comps = {k: v for k, v in built.items() if not k.startswith("_")}
    shape = (1024, 256, 32, 8, 64, 64)
    head = qoh.PackedHead(*shape, comps)
    y, tol = _oracle(comps, shape, h_bits)
    return head, h_bits, targets, y, tol


def test_cfg1_logits_and_argmax(cfg1):
    head, h_bits, _, y, tol = cfg1
    lg, am = head.logits(_dev_hidden(h_bits))
    check_logits(lg.cpu().numpy(), y, tol)
    check_argmax(am.cpu().numpy(), y, tol)


def test_cfg1_fused_epilogue(cfg1):
    head, h_bits, targets, y, tol = cfg1
    lse, am, ce = head.lse_argmax(_dev_hidden(h_bits), torch.from_numpy(targets))
    check_lse_ce(lse.cpu().numpy(), ce.cpu().numpy(), y, tol, targets)
    check_argmax(am.cpu().numpy(), y, tol)


def test_cfg1_host_buffer_entry_matches_device_entry(cfg1):
    head, h_bits, targets, y, tol = cfg1
    lse_d, am_d, ce_d = head.lse_argmax(_dev_hidden(h_bits), torch.from_numpy(targets))
    lse_h, am_h, ce_h = head.lse_argmax_host(h_bits, targets)
    assert np.array_equal(lse_h, lse_d.cpu().numpy())
    assert np.array_equal(am_h, am_d.cpu().numpy())
    assert np.array_equal(ce_h, ce_d.cpu().numpy())


def test_cfg1_host_logits_entry_matches_device_entry(cfg1):
    """archead_logits_host (host buffers in and out) gives the device entry's
    logits and argmax bit for bit, and both outputs are optional."""
    head, h_bits, _, y, tol = cfg1
    lg_d, am_d = head.logits(_dev_hidden(h_bits))
    lg_h, am_h = head.logits_host(h_bits)
    assert np.array_equal(lg_h, lg_d.cpu().numpy())
    assert np.array_equal(am_h, am_d.cpu().numpy())
    check_logits(lg_h, y, tol)
    only_am = head.logits_host(h_bits, out=(None, np.empty(h_bits.shape[0], np.int32)))[1]
    assert np.array_equal(only_am, am_d.cpu().numpy())
    with pytest.raises(Exception):
        head.logits_host(h_bits, out=(None, None))


def _pinned(a):
    t = torch.from_numpy(np.ascontiguousarray(a)).pin_memory()
    return t, t.numpy()


def test_cfg1_host_entries_replay_with_pinned_buffers(cfg1):
    """Pinned host buffers take the captured-sequence path (a capture on the
    first call, a replay after it): new inputs in the same buffers give the
    device entry points' results bit for bit, twice in a row, for both
    host-buffer entry points and their prepared forms."""
    head, h_bits, targets, y, tol = cfg1
    T = h_bits.shape[0]
    _, hh = _pinned(h_bits.view(np.int16))
    _, th = _pinned(targets)
    keep = [_pinned(np.zeros((T, head.V), np.float32)), _pinned(np.zeros(T, np.int32)),
            _pinned(np.zeros(T, np.float32)), _pinned(np.zeros(T, np.int32)), _pinned(np.zeros(T, np.float32))]
    lg, am, lse, am2, ce = [k[1] for k in keep]
    logits_call = head.prepare_logits_host(hh, (lg, am))
    lse_call = head.prepare_lse_argmax_host(hh, th, (lse, am2, ce))
    rng = np.random.default_rng(3)
    for rep in range(3):
        src = h_bits if rep == 0 else np.roll(h_bits, rep, axis=1)   # new inputs into the same buffers
        hh.view(np.uint16)[:] = src
        th[:] = rng.integers(0, head.V, size=T, dtype=np.int32)
        logits_call()
        lse_call()
        lg_d, am_d = head.logits(_dev_hidden(src))
        lse_d, am2_d, ce_d = head.lse_argmax(_dev_hidden(src), torch.from_numpy(th.copy()))
        assert np.array_equal(lg, lg_d.cpu().numpy()) and np.array_equal(am, am_d.cpu().numpy())
        assert np.array_equal(lse, lse_d.cpu().numpy()) and np.array_equal(am2, am2_d.cpu().numpy())
        assert np.array_equal(ce, ce_d.cpu().numpy())
    # the unprepared forms with the same pinned buffers replay the same sequences
    head.logits_host(hh, (lg, am))
    assert np.array_equal(lg, lg_d.cpu().numpy())


# ------------------------------------------------ Qwen-shaped head (2, 3, 5)
@pytest.fixture(scope="module")
def qwen(qoh):
    shape, _, _, comps = gen.make_workload(2)
    head = qoh.PackedHead(*shape.as_tuple(), comps)
    h1, t1 = gen.draw_activations(4096, 1, shape.V, 2)
    h64, t64 = gen.draw_activations(4096, 64, shape.V, 3)
    h5, t5 = gen.draw_activations(4096, 4096, shape.V, 5)
    stacked = np.concatenate([h1, h64], axis=0)
    y, tol = _oracle(comps, QWEN, stacked)
    return dict(head=head, comps=comps, h1=h1, t1=t1, h64=h64, t64=t64, h5=h5, t5=t5,
                y1=y[:1], tol1=tol[:1], y64=y[1:65], tol64=tol[1:65])


def test_qwen_decode_T1_logits_argmax(qwen):
    head = qwen["head"]
    lg, am = head.logits(_dev_hidden(qwen["h1"]))
    check_logits(lg.cpu().numpy(), qwen["y1"], qwen["tol1"])
    check_argmax(am.cpu().numpy(), qwen["y1"], qwen["tol1"])


def test_qwen_decode_T1_fused(qwen):
    head = qwen["head"]
    lse, am, ce = head.lse_argmax(_dev_hidden(qwen["h1"]), torch.from_numpy(qwen["t1"]))
    check_lse_ce(lse.cpu().numpy(), ce.cpu().numpy(), qwen["y1"], qwen["tol1"], qwen["t1"])
    check_argmax(am.cpu().numpy(), qwen["y1"], qwen["tol1"])


@pytest.mark.parametrize("T", sorted(set(gen.SWEEP_T) | {9, 16, 17}))
def test_qwen_decode_sweep_fused(qwen, T):
    """Config 3's token counts, plus the dispatch boundary: up to 8 tokens take
    one decode launch, 9 and more the tensor-core kernel."""
    head = qwen["head"]
    assert head.forward_kernel(T) == ("decode" if T <= 8 else "tensor_core")
    h, tg = qwen["h64"][:T], qwen["t64"][:T]
    lse, am, ce = head.lse_argmax(_dev_hidden(h), torch.from_numpy(tg))
    y, tol = qwen["y64"][:T], qwen["tol64"][:T]
    check_lse_ce(lse.cpu().numpy(), ce.cpu().numpy(), y, tol, tg)
    check_argmax(am.cpu().numpy(), y, tol)


def test_qwen_decode_T64_logits(qwen):
    head = qwen["head"]
    lg, am = head.logits(_dev_hidden(qwen["h64"]))
    check_logits(lg.cpu().numpy(), qwen["y64"], qwen["tol64"])
    check_argmax(am.cpu().numpy(), qwen["y64"], qwen["tol64"])


def test_qwen_prefill_T4096_every_token_and_T512_logits(qwen):
    """Config 5 at full size: LSE, CE and argmax of all 4096 tokens (32 token
    tiles of the tensor-core launch) over the whole vocabulary, and every logit
    of a 512-token call (four token tiles), against the oracle.  The oracle runs
    on batches of 1024 tokens to bound host memory."""
    head = qwen["head"]
    h5, t5 = qwen["h5"], qwen["t5"]
    assert head.forward_kernel(4096) == "tensor_core" and head.forward_kernel(512) == "tensor_core"
    lse, am, ce = head.lse_argmax(_dev_hidden(h5), torch.from_numpy(t5))
    lse, am, ce = lse.cpu().numpy(), am.cpu().numpy(), ce.cpu().numpy()
    lg512, am512 = head.logits(_dev_hidden(h5[:512]))
    lg512, am512 = lg512.cpu().numpy(), am512.cpu().numpy()
    for b0 in range(0, 4096, 1024):
        sl = slice(b0, b0 + 1024)
        y, tol = _oracle(qwen["comps"], QWEN, h5[sl])
        check_lse_ce(lse[sl], ce[sl], y, tol, t5[sl])
        check_argmax(am[sl], y, tol)
        if b0 == 0:
            check_logits(lg512, y[:512], tol[:512])
            check_argmax(am512, y[:512], tol[:512])
        del y, tol


def test_qwen_calls_are_deterministic(qwen):
    head = qwen["head"]
    hd = _dev_hidden(qwen["h64"][:8])
    a = head.lse_argmax(hd)
    b = head.lse_argmax(hd)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_qwen_status_clean(qwen):
    head = qwen["head"]
    head.lse_argmax(_dev_hidden(qwen["h1"]), torch.from_numpy(qwen["t1"]))
    assert head.status(head.workspace(1)) == 0


@pytest.mark.parametrize("variant", sorted(gen.BASELINE_SHAPES))
def test_qwen_storage_matched_baselines(qoh, variant):
    """The pages' comparison heads (plain group-INT4; core + residual) on both kernels, every logit."""
    shape = gen.BASELINE_SHAPES[variant]
    comps = gen.draw_components(shape, 2)
    head = qoh.PackedHead(*shape.as_tuple(), comps)
    h_bits, _ = gen.draw_activations(shape.d, 20, shape.V, 3)
    y, tol = _oracle(comps, shape.as_tuple(), h_bits)
    for T in (1, 20):
        assert head.forward_kernel(T) == ("decode" if T == 1 else "tensor_core")
        lg, am = head.logits(_dev_hidden(h_bits[:T]))
        check_logits(lg.cpu().numpy(), y[:T], tol[:T])
        check_argmax(am.cpu().numpy(), y[:T], tol[:T])


# ------------------------------------------------------------- config 4
@pytest.fixture(scope="module")
def gemma(qoh):
    shape, h, tg, comps = gen.make_workload(4)
    head = qoh.PackedHead(*shape.as_tuple(), comps)
    y, tol = _oracle(comps, GEMMA, h)
    return head, h, tg, y, tol


def test_gemma_decode_T16_fused_ce(gemma):
    head, h, tg, y, tol = gemma
    lse, am, ce = head.lse_argmax(_dev_hidden(h), torch.from_numpy(tg))
    check_lse_ce(lse.cpu().numpy(), ce.cpu().numpy(), y, tol, tg)
    check_argmax(am.cpu().numpy(), y, tol)


def test_gemma_decode_T16_logits(gemma):
    head, h, tg, y, tol = gemma
    lg, am = head.logits(_dev_hidden(h))
    check_logits(lg.cpu().numpy(), y, tol)


# ------------------------------------------------ ragged and edge shapes
SMALL = [
    # V,    d,   r_c, r_r, g,   g_B, T
    (1000, 320, 32, 8, 64, 64, 3),       # ragged vocabulary tail (not a multiple of 16)
    (1003, 320, 100, 40, 16, 10, 9),     # ragged ranks, g = 16, g_B not a power of two, two launches
    (16, 64, 0, 0, 64, 1, 1),            # residual only, one m-tile
    (47, 128, 64, 32, 128, 128, 17),     # one 128-row tile, mostly past the vocabulary (tensor-core path)
    (4099, 512, 64, 64, 256, 32, 8),     # group of 256 spans a whole residual warp
    (2048, 1024, 512, 64, 512, 128, 5),  # group larger than a warp's columns
]


@pytest.mark.parametrize("V,d,r_c,r_r,g,g_B,T", SMALL)
def test_small_shapes(qoh, V, d, r_c, r_r, g, g_B, T):
    shape = (V, d, r_c, r_r, g, g_B)
    comps = gen.random_components(gen.HeadShape(*shape), seed=V + d + T)
    h_bits, tg = gen.random_hidden(d, T, seed=T + 7, V=V)
    head = qoh.PackedHead(*shape, comps)
    y, tol = _oracle(comps, shape, h_bits)
    lg, am = head.logits(_dev_hidden(h_bits))
    check_logits(lg.cpu().numpy(), y, tol)
    check_argmax(am.cpu().numpy(), y, tol)
    lse, am2, ce = head.lse_argmax(_dev_hidden(h_bits), torch.from_numpy(tg))
    check_lse_ce(lse.cpu().numpy(), ce.cpu().numpy(), y, tol, tg)
    assert np.array_equal(am.cpu().numpy(), am2.cpu().numpy())


# Calls of >= 9 tokens take the tensor-core kernel when g_B is a multiple of 64.
SMALL_TC = [
    # V,    d,   r_c, r_r, g,   g_B, T
    (1000, 320, 32, 8, 64, 64, 17),       # ragged vocabulary, one 32-column correction chunk
    (2000, 256, 0, 0, 16, 64, 33),        # residual only, g = 16, ragged token tile
    (1500, 512, 64, 0, 32, 64, 130),      # no correction, g = 32, two token tiles
    (4099, 512, 128, 64, 256, 128, 40),   # g = 256, last 128-row tile nearly empty
    (300, 128, 64, 32, 128, 128, 200),    # three 128-row tiles, the last partial
    (777, 192, 64, 64, 64, 64, 9),        # fewest tokens of the tensor-core path, odd k-step count
    (777, 192, 64, 64, 64, 64, 8),        # most tokens of the decode kernel (one launch)
    (1003, 320, 100, 40, 16, 10, 20),     # g_B = 10: 9+ tokens through the decode kernel (three launches)
]


@pytest.mark.parametrize("V,d,r_c,r_r,g,g_B,T", SMALL_TC)
def test_small_shapes_many_tokens(qoh, V, d, r_c, r_r, g, g_B, T):
    test_small_shapes(qoh, V, d, r_c, r_r, g, g_B, T)


@pytest.mark.parametrize("T", [5, 24])   # the decode kernel, then the tensor-core kernel
def test_vocab_shards_merge_to_the_whole_head(qoh, T):
    """Three vocabulary shards of one head, merged, against the unsharded head and the oracle."""
    shape = (1000, 256, 32, 8, 64, 64)
    comps = gen.random_components(gen.HeadShape(*shape), seed=321)
    h_bits, targets = gen.random_hidden(256, T, seed=322, V=shape[0])
    hd, tg = _dev_hidden(h_bits), torch.from_numpy(targets)
    y, tol = _oracle(comps, shape, h_bits)
    whole = qoh.PackedHead(*shape, comps)
    lse_w, am_w, ce_w = whole.lse_argmax(hd, tg)
    parts = []
    for r in range(3):
        v0, v1 = qoh.shard_rows(shape[0], 3, r)
        head = qoh.PackedHead(v1 - v0, *shape[1:], qoh.shard_components(comps, v0, v1))
        head.set_vocab_shard(v0, shape[0])
        p = head.shard_partials(hd, tg)
        parts.append(p)
        # the shard's own statistics: global argmax inside its rows, target logit only when it holds the target
        pc = p.cpu().numpy()
        am = pc[:, 2].view(np.int32)
        assert np.all((am >= v0) & (am < v1))
        inside = (targets >= v0) & (targets < v1)
        assert np.all(np.isnan(pc[~inside, 3]))
        np.testing.assert_allclose(pc[inside, 3], y[np.arange(T)[inside], targets[inside]],
                                   atol=float(tol.max()), rtol=0)
        np.testing.assert_allclose(pc[:, 1], y[:, v0:v1].max(axis=1), atol=float(tol.max()), rtol=0)
    with pytest.raises(qoh.ArcheadError):
        head.set_vocab_shard(8, shape[0])               # shards start on 16-row boundaries
    lse, am, ce = qoh.merge_shards(torch.stack(parts))
    check_lse_ce(lse.cpu().numpy(), ce.cpu().numpy(), y, tol, targets)
    check_argmax(am.cpu().numpy(), y, tol)
    np.testing.assert_allclose(lse.cpu().numpy(), lse_w.cpu().numpy(), atol=float(tol.max()), rtol=0)
    np.testing.assert_allclose(ce.cpu().numpy(), ce_w.cpu().numpy(), atol=2 * float(tol.max()), rtol=0)


def _check_samples(got, y, tol, temperature, seed, offset):
    """Sampled ids against the oracle's Gumbel-max picks: equal, or the oracle's
    perturbed values of the two rows within the logit tolerance / temperature
    (plus the fp32 rounding of the Gumbel draw)."""
    want, z = oracle.sample_gumbel(y, temperature, seed, offset)
    for t, (a, b) in enumerate(zip(np.asarray(got), want)):
        if a == b:
            continue
        assert 0 <= a < y.shape[1], f"sample[{t}] = {a} out of range"
        gap = z[t, b] - z[t, a]
        assert gap <= max(tol[t, a], tol[t, b]) / temperature + 1e-4, f"sample[{t}]: gpu {a}, oracle {b}, gap {gap:.3g}"


@pytest.mark.parametrize("T", [5, 20])   # one and three decode launches
def test_sampling_matches_oracle(qoh, T):
    shape = (1000, 256, 32, 8, 64, 64)
    comps = gen.random_components(gen.HeadShape(*shape), seed=77)
    h_bits, _ = gen.random_hidden(256, T, seed=78, V=shape[0])
    head = qoh.PackedHead(*shape, comps)
    y, tol = _oracle(comps, shape, h_bits)
    for temperature, seed, offset in ((0.7, 12345, 0), (1.5, 2**40 + 3, 2**33 + 7)):
        s1, lse, am = head.sample(_dev_hidden(h_bits), temperature, seed, offset)
        _check_samples(s1.cpu().numpy(), y, tol, temperature, seed, offset)
        check_lse_ce(lse.cpu().numpy(), None, y, tol)
        check_argmax(am.cpu().numpy(), y, tol)
        s2, _, _ = head.sample(_dev_hidden(h_bits), temperature, seed, offset)
        assert torch.equal(s1, s2)                      # counter-based: reproducible
    a, _, _ = head.sample(_dev_hidden(h_bits), 1.0, 1, 0)
    b, _, _ = head.sample(_dev_hidden(h_bits), 1.0, 1, 1000)
    assert not torch.equal(a, b)                        # another counter range draws other noise


@pytest.mark.parametrize("T", [5, 20])   # one and three decode launches
def test_sampling_across_vocabulary_shards(qoh, T):
    """Three vocabulary shards' sampling pairs, merged, draw exactly what the
    unsharded head draws (the noise follows the global row); each shard's
    pair is the best perturbed logit of its own rows."""
    shape = (1000, 256, 32, 8, 64, 64)
    comps = gen.random_components(gen.HeadShape(*shape), seed=88)
    h_bits, _ = gen.random_hidden(256, T, seed=89, V=shape[0])
    hd = _dev_hidden(h_bits)
    whole = qoh.PackedHead(*shape, comps)
    for temperature, seed, offset in ((0.7, 4242, 0), (1.3, 2**41 + 5, 2**35 + 1)):
        want, _, _ = whole.sample(hd, temperature, seed, offset)
        parts = []
        for r in range(3):
            v0, v1 = qoh.shard_rows(shape[0], 3, r)
            head = qoh.PackedHead(v1 - v0, *shape[1:], qoh.shard_components(comps, v0, v1))
            head.set_vocab_shard(v0, shape[0])
            p = head.sample_partials(hd, temperature, seed, offset)
            rows = p[:, 1].contiguous().view(torch.int32).cpu().numpy()
            assert np.all((rows >= v0) & (rows < v1))
            own, _, _ = head.sample(hd, temperature, seed, offset)
            np.testing.assert_array_equal(rows, own.cpu().numpy())   # the shard's own draw over its rows
            parts.append(p)
        got = qoh.merge_sample_shards(torch.stack(parts))
        assert torch.equal(got, want)


def test_sampling_frequencies_follow_softmax(qoh):
    """One token repeated 16384 times over a 64-row head: chi-square of the GPU's
    draws against softmax(y / tau) of the oracle's logits."""
    shape = (64, 64, 16, 8, 16, 16)
    comps = gen.random_components(gen.HeadShape(*shape), seed=5)
    h1, _ = gen.random_hidden(64, 1, seed=6, V=64)
    y, _ = _oracle(comps, shape, h1)
    tau, n = 0.9, 16384
    head = qoh.PackedHead(*shape, comps)
    got, _, _ = head.sample(_dev_hidden(np.repeat(h1, n, axis=0)), tau, seed=99, offset=0)
    p = np.exp(y[0] / tau - (y[0] / tau).max())
    p /= p.sum()
    counts = np.bincount(got.cpu().numpy(), minlength=64)
    keep = n * p >= 5                                   # chi-square cells with enough expected draws
    rest = counts[~keep].sum(), n * p[~keep].sum()
    obs = np.append(counts[keep], rest[0])
    exp = np.append(n * p[keep], rest[1])
    chi2 = float(((obs - exp) ** 2 / np.maximum(exp, 1e-12)).sum())
    assert chi2 < 110.0   # well above the 99.9 % point for <= 64 cells


def test_qwen_sampling_T1(qwen):
    head = qwen["head"]
    s, lse, am = head.sample(_dev_hidden(qwen["h1"]), 0.8, seed=2024, offset=5)
    _check_samples(s.cpu().numpy(), qwen["y1"], qwen["tol1"], 0.8, 2024, 5)
    check_argmax(am.cpu().numpy(), qwen["y1"], qwen["tol1"])


def test_zero_residual_and_correction_is_core_product(qoh):
    shape = (512, 256, 64, 32, 64, 64)
    comps = gen.random_components(gen.HeadShape(*shape), seed=99)
    comps["q"][:] = 0
    comps["A"][:] = 0
    h_bits, _ = gen.random_hidden(256, 4, seed=98)
    head = qoh.PackedHead(*shape, comps)
    lg, _ = head.logits(_dev_hidden(h_bits))
    h = oracle.bf16_decode(h_bits)
    Rh = oracle.dequantize(comps["R"], comps["s_R"], None)
    Lh = oracle.dequantize(comps["L"], comps["s_L"], None)
    ref = (h @ Rh.T) @ Lh.T
    _, rowmax = oracle.logits(comps, 64, 64, h_bits)
    check_logits(lg.cpu().numpy(), ref, oracle.tolerance(h_bits, rowmax))


def test_bad_target_gives_nan_and_status(qoh):
    shape = (64, 64, 16, 8, 16, 16)
    comps = gen.random_components(gen.HeadShape(*shape), seed=3)
    head = qoh.PackedHead(*shape, comps)
    h_bits, _ = gen.random_hidden(64, 2, seed=4)
    ws = head.workspace(2)
    head.status(ws, clear=True)
    lse, am, ce = head.lse_argmax(_dev_hidden(h_bits), torch.tensor([5, 64], dtype=torch.int32))
    ce = ce.cpu().numpy()
    assert np.isfinite(ce[0]) and np.isnan(ce[1])
    assert head.status(ws, clear=True) == qoh.STATUS_BAD_TARGET
    assert head.status(ws) == 0


def test_forward_argument_errors(qoh):
    shape = (64, 64, 16, 8, 16, 16)
    head = qoh.PackedHead(*shape, gen.random_components(gen.HeadShape(*shape), seed=5))
    h = torch.zeros((2, 64), dtype=torch.bfloat16, device="cuda")
    ws = head.workspace(2)
    lse = torch.empty(2, device="cuda")
    am = torch.empty(2, dtype=torch.int32, device="cuda")
    with pytest.raises(qoh.ArcheadError) as e:
        head.lse_argmax_into(h[:0], None, lse, am, None, ws)
    assert e.value.status == qoh.ARCHEAD_EINVAL
    with pytest.raises(qoh.ArcheadError) as e:
        head.lse_argmax_into(h, None, lse, am, None, ws[:64])
    assert e.value.status == qoh.ARCHEAD_ENOMEM
    big = torch.zeros(3 * 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(qoh.ArcheadError) as e:
        head.lse_argmax_into(big[1:129].view(2, 64), None, lse, am, None, ws)
    assert e.value.status == qoh.ARCHEAD_EALIGN


# ------------------------------------------- argmax ties and extreme tokens
def _tie_head(gen_seed, V, d, T, h_bits, spacing):
    """Components where, for token t, rows b_t - spacing < b_t < b_t + spacing
    are identical copies of a row whose residual codes follow the sign of h_t
    (so its logit is the row maximum by a wide margin).  The copies sit at the
    same position modulo `spacing` (a multiple of 16, the m-tile height, or of
    128, the tensor-core tile height), in different tiles, so both kernels
    compute bit-identical logits for them and the lowest index must win."""
    shape = (V, d, 32, 8, 64, 64)
    comps = gen.random_components(gen.HeadShape(*shape), seed=gen_seed)
    h = oracle.bf16_decode(h_bits)
    triples = []
    step = (V - 2 * spacing - 16) // T
    for t in range(T):
        b = spacing + 8 + step * t + t % 16
        rows = (b - spacing, b, b + spacing)
        assert rows[0] >= 0 and rows[2] < V
        comps["q"][b] = np.where(h[t] >= 0, 7, -8).astype(np.int8)
        comps["s_res"][b] = gen.f64_to_fp16_bits(np.full(d // 64, 0.006))   # two standard deviations
        for v in (rows[0], rows[2]):
            for k in ("L", "s_L", "q", "s_res", "A", "s_A"):
                comps[k][v] = comps[k][b]
        triples.append(rows)
    assert len({v for r in triples for v in r}) == 3 * T   # the triples of different tokens never meet
    return shape, comps, triples


@pytest.mark.parametrize("T,spacing", [(5, 16), (5, 2368), (24, 128), (24, 1280)])
def test_argmax_ties_resolve_to_lowest_index(qoh, T, spacing):
    """Equal maxima in different m-tiles / 128-row tiles / blocks: argmax must be
    exactly the lowest index on both entry points (5 tokens: decode kernel,
    24 tokens: tensor-core kernel; spacing 2368 = 148 m-tiles puts two copies in
    the same decode block)."""
    V, d = 7000, 256
    h_bits, targets = gen.random_hidden(d, T, seed=41 + T, V=V)
    shape, comps, triples = _tie_head(40 + T, V, d, T, h_bits, spacing)
    head = qoh.PackedHead(*shape, comps)
    assert head.forward_kernel(T) == ("decode" if T <= 8 else "tensor_core")
    y, tol = _oracle(comps, shape, h_bits)
    lowest = np.array([r[0] for r in triples])
    # the construction: the oracle's maximum is the triple, by more than the tolerance
    _, am_ref, _ = oracle.lse_argmax_ce(y)
    assert np.array_equal(am_ref, lowest)
    for t, rows in enumerate(triples):
        rest = np.delete(y[t], rows)
        assert y[t, rows[0]] - rest.max() > 4 * tol[t].max()
    lg, am = head.logits(_dev_hidden(h_bits))
    lg = lg.cpu().numpy()
    for t, rows in enumerate(triples):   # the copies are bit-identical on the GPU too
        assert lg[t, rows[0]] == lg[t, rows[1]] == lg[t, rows[2]]
    check_logits(lg, y, tol)
    check_argmax_exact(am.cpu().numpy(), lowest)
    lse, am2, ce = head.lse_argmax(_dev_hidden(h_bits), torch.from_numpy(targets))
    check_argmax_exact(am2.cpu().numpy(), lowest, "argmax (fused epilogue)")
    check_lse_ce(lse.cpu().numpy(), ce.cpu().numpy(), y, tol, targets)


@pytest.mark.parametrize("T,kernel", [(5, "decode"), (24, "tensor_core")])
def test_activation_splits_with_uneven_columns(qoh, T, kernel):
    """Column ranges of h under powers of two of their own: on the tensor-core
    path the activation kernel splits d over 8 blocks of 128 columns at this
    shape and the last split rescales the others to the token's exponent; on
    the decode path each residual warp scales its own 256 columns (warps past
    d have none).  Tokens whose columns are zero outside one split, 2^40
    larger or 2^-40 smaller in one split, or zero but for one entry, against
    the oracle."""
    shape = (3000, 1024, 64, 16, 64, 64)
    comps = gen.random_components(gen.HeadShape(*shape), seed=616)
    h_bits, targets = gen.random_hidden(1024, T, seed=617, V=shape[0])
    h = gen.bf16_bits_to_f32(h_bits).copy()
    h[0, 128:] = 0.0                                  # only the first split
    h[1, :896] = 0.0                                  # only the last split
    h[2, 384:512] *= np.float32(2.0 ** 40)            # one split far above the rest
    h[3, 640:768] *= np.float32(2.0 ** -40)           # one split far below the rest
    h[4, :] = 0.0
    h[4, 700] = np.float32(3.0)                       # one entry in the sixth split
    h_bits = gen.f32_to_bf16_bits(h)
    assert np.array_equal(gen.bf16_bits_to_f32(h_bits), h)   # the scaling is exact in bf16
    head = qoh.PackedHead(*shape, comps)
    assert head.forward_kernel(T) == kernel
    y, tol = _oracle(comps, shape, h_bits)
    lg, am = head.logits(_dev_hidden(h_bits))
    lse, am2, ce = head.lse_argmax(_dev_hidden(h_bits), torch.from_numpy(targets))
    check_logits(lg.cpu().numpy(), y, tol)
    check_argmax(am.cpu().numpy(), y, tol)
    check_argmax(am2.cpu().numpy(), y, tol)
    check_lse_ce(lse.cpu().numpy(), ce.cpu().numpy(), y, tol, targets)
    assert head.status(head.workspace(T)) == 0


@pytest.mark.parametrize("T", [5, 24])   # decode kernel, tensor-core kernel
def test_zero_and_extreme_magnitude_tokens(qoh, T):
    """Token 0 all zero (every logit exactly 0: argmax 0, LSE = log V), token 1
    scaled by 2^64, token 2 by 2^-60 (bf16 exact), the rest ordinary."""
    shape = (3000, 256, 32, 8, 64, 64)
    comps = gen.random_components(gen.HeadShape(*shape), seed=606)
    h_bits, targets = gen.random_hidden(256, T, seed=607, V=shape[0])
    h = gen.bf16_bits_to_f32(h_bits).copy()
    h[0] = 0.0
    h[1] *= np.float32(2.0 ** 64)
    h[2] *= np.float32(2.0 ** -60)
    h_bits = gen.f32_to_bf16_bits(h)
    assert np.array_equal(gen.bf16_bits_to_f32(h_bits), h)   # the scaling is exact in bf16
    head = qoh.PackedHead(*shape, comps)
    y, tol = _oracle(comps, shape, h_bits)
    lg, am = head.logits(_dev_hidden(h_bits))
    lg, am = lg.cpu().numpy(), am.cpu().numpy()
    lse, am2, ce = head.lse_argmax(_dev_hidden(h_bits), torch.from_numpy(targets))
    lse, am2, ce = lse.cpu().numpy(), am2.cpu().numpy(), ce.cpu().numpy()
    # the zero token: exact zeros, every row tied, so the lowest index
    assert np.all(lg[0] == 0.0)
    assert am[0] == 0 and am2[0] == 0
    np.testing.assert_allclose(lse[0], np.log(shape[0]), rtol=1e-6)
    np.testing.assert_allclose(ce[0], np.log(shape[0]), rtol=1e-6)
    # every other token within the tolerance (which scales with ||h_t||)
    check_logits(lg[1:], y[1:], tol[1:])
    check_argmax(am[1:], y[1:], tol[1:])
    check_argmax(am2[1:], y[1:], tol[1:])
    check_lse_ce(lse[1:], ce[1:], y[1:], tol[1:], targets[1:])
    assert head.status(head.workspace(T)) == 0
