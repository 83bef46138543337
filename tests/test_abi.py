"""The C-ABI library loads, exports every symbol include/archead.h declares,
and its host-only logic (byte counts, argument checks) behaves.  No GPU."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "archead.h")


def _load_build_module():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_archead_build", os.path.join(ROOT, "quantized_output_head_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.fixture(scope="module")
def qoh():
    _load_build_module().build()
    import quantized_output_head_b200 as m
    return m


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"ARCHEAD_API\s+[\w\s\*]*?\b(archead_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_symbols()
    for must in ("archead_pack_load", "archead_logits", "archead_logits_lse_argmax"):
        assert must in names


def test_library_exports_every_declared_symbol(qoh):
    names = declared_symbols()
    lib = ctypes.CDLL(qoh.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", qoh.LIB_PATH], capture_output=True, text=True).stdout
    exported = sorted(set(re.findall(r"\bT (archead_\w+)", out)))
    assert exported == names
    assert sorted(qoh.EXPORTED) == names


BUILD_HEADER = os.path.join(ROOT, "include", "archead_build.h")


def test_builder_library_exports_every_declared_symbol(qoh):
    import quantized_output_head_b200.builder as bld
    text = open(BUILD_HEADER).read()
    names = sorted(set(re.findall(r"ARCHEAD_API\s+[\w\s\*]*?\b(archead_\w+)\s*\(", text)))
    assert "archead_build_head" in names
    out = subprocess.run(["nm", "-D", "--defined-only", bld.BUILD_LIB_PATH], capture_output=True, text=True).stdout
    assert sorted(set(re.findall(r"\bT (archead_\w+)", out))) == names
    assert sorted(bld.EXPORTED_BUILD) == names


def test_builder_argument_checks_need_no_gpu(qoh):
    """Bad arguments are refused on the host, before any CUDA call."""
    import ctypes as ct
    import quantized_output_head_b200.builder as bld
    lib = bld._blib
    assert lib.archead_build_quantize(None, 4, 64, 4, 0, None, None, None) == -1
    assert b"null" in lib.archead_build_last_error()
    fake = ct.c_void_p(256)                  # never dereferenced: the checks fail first
    assert lib.archead_build_quantize(fake, 4, 64, 6, 0, fake, fake, None) == -1
    assert lib.archead_build_quantize(fake, 4, 64, 4, 24, fake, fake, None) == -1
    assert lib.archead_build_metric(0, 16, fake, 0.01, 0.75, fake, fake, fake, 1 << 20, None) == -1
    assert lib.archead_build_metric(64, 16, fake, -1.0, 0.75, fake, fake, fake, 1 << 20, None) == -1
    bad = [qoh.ArcheadDesc(1024, 256, 300, 8, 64, 64),    # r_c > min(V, d)
           qoh.ArcheadDesc(1024, 256, 32, 8, 48, 64),     # g does not divide d
           qoh.ArcheadDesc(0, 256, 0, 0, 64, 64)]
    for desc in bad:
        assert lib.archead_build_workspace_bytes(ct.byref(desc), 4096) == 0
        assert lib.archead_build_head(ct.byref(desc), fake, fake, 4096, 0.01, 0.75, None, fake, 1 << 20, None) == -1


SHAPES = [
    (1024, 256, 32, 8, 64, 64),
    (151936, 4096, 512, 64, 128, 128),
    (262144, 2560, 384, 64, 128, 128),
    (1000, 320, 0, 0, 16, 1),
    (17, 320, 100, 3, 64, 10),
]


@pytest.mark.parametrize("shape", SHAPES)
def test_packed_bytes_matches_oracle(qoh, shape):
    assert qoh.archead_packed_bytes(*shape) == oracle.packed_bytes(*shape)


@pytest.mark.parametrize("shape", SHAPES)
def test_arena_holds_payload(qoh, shape):
    arena = qoh.archead_arena_bytes(*shape)
    assert arena >= qoh.archead_packed_bytes(*shape)
    assert arena % 256 == 0


def test_arena_padding_small_at_qwen_shape(qoh):
    shape = (151936, 4096, 512, 64, 128, 128)
    assert qoh.archead_arena_bytes(*shape) - qoh.archead_packed_bytes(*shape) < 4096


@pytest.mark.parametrize("shape", [
    (0, 256, 32, 8, 64, 64),      # V < 1
    (16, 100, 8, 8, 4, 4),        # d not a multiple of 64
    (16, 256, 8, 8, 48, 64),      # g not a power of two
    (16, 256, 8, 8, 8, 64),       # g < 16
    (16, 256, 8, 8, 64, 7),       # g_B does not divide d
    (16, 256, -1, 8, 64, 64),     # negative rank
])
def test_unsupported_shapes_report_zero(qoh, shape):
    assert qoh.archead_packed_bytes(*shape) == 0
    assert qoh.archead_arena_bytes(*shape) == 0


def _host_components(V, d, r_c, r_r, g, g_B):
    import archead_inputs as gen
    return gen.random_components(gen.HeadShape(V, d, r_c, r_r, g, g_B), 5)


def _pack_load_raw(qoh, shape, comps, arena_ptr=4096, arena_bytes=1 << 30):
    desc = qoh.ArcheadDesc(*shape)
    keep = {k: np.ascontiguousarray(v) for k, v in comps.items()}
    hc = qoh.ArcheadHostComponents(**{k: v.ctypes.data for k, v in keep.items()})
    h = ctypes.c_void_p()
    return qoh._lib.archead_pack_load(ctypes.byref(desc), ctypes.byref(hc), arena_ptr, arena_bytes, None,
                                      ctypes.byref(h))


def test_pack_load_rejects_out_of_range_codes(qoh):
    shape = (32, 64, 8, 4, 16, 16)
    c = _host_components(*shape)
    c["q"][3, 5] = 8                       # INT4 residual range is [-8, 7]
    assert _pack_load_raw(qoh, shape, c) == qoh.ARCHEAD_EINVAL
    c = _host_components(*shape)
    c["L"][0, 0] = -17                     # INT5 core range is [-16, 15]
    assert _pack_load_raw(qoh, shape, c) == qoh.ARCHEAD_EINVAL


def test_pack_load_rejects_non_finite_scales(qoh):
    shape = (32, 64, 8, 4, 16, 16)
    c = _host_components(*shape)
    c["s_res"][1, 1] = 0x7C00              # +inf in fp16
    assert _pack_load_raw(qoh, shape, c) == qoh.ARCHEAD_EINVAL
    c = _host_components(*shape)
    c["s_B"][0, 0] = 0x7E00                # NaN
    assert _pack_load_raw(qoh, shape, c) == qoh.ARCHEAD_EINVAL


def test_pack_load_argument_checks(qoh):
    shape = (32, 64, 8, 4, 16, 16)
    c = _host_components(*shape)
    assert _pack_load_raw(qoh, shape, c, arena_ptr=4096 + 16) == qoh.ARCHEAD_EALIGN
    assert _pack_load_raw(qoh, shape, c, arena_bytes=16) == qoh.ARCHEAD_ENOMEM
    assert _pack_load_raw(qoh, (32, 60, 8, 4, 16, 16), c) == qoh.ARCHEAD_EUNSUP
    assert qoh._lib.archead_pack_load(None, None, None, 0, None, None) == qoh.ARCHEAD_EINVAL


def test_forward_rejects_null_handle(qoh):
    L = qoh._lib
    assert L.archead_logits(None, 4096, 1, 4096, None, 4096, 1 << 20, None) == qoh.ARCHEAD_EINVAL
    assert L.archead_logits_lse_argmax(None, 4096, 1, None, 4096, 4096, None, 4096, 1 << 20, None) == \
        qoh.ARCHEAD_EINVAL
    assert L.archead_workspace_bytes(None, 4) == 0
    assert L.archead_forward_kernel(None, 4) == -1
    assert L.archead_status_string(qoh.ARCHEAD_EUNSUP) == b"unsupported shape or device"


def test_sampling_and_shard_calls_refuse_bad_arguments_on_the_host(qoh):
    """These checks return before any CUDA call or handle use (no GPU here)."""
    import ctypes as ct
    L = qoh._lib
    fake = 4096                                  # never dereferenced: the checks fail first
    for temp in (0.0, -1.0, float("inf"), float("nan")):
        assert L.archead_sample(fake, fake, 1, temp, 1, 0, fake, None, None, fake, 1 << 20, None) == \
            qoh.ARCHEAD_EINVAL
    assert L.archead_sample(fake, fake, 1, 1.0, 1, 0, None, None, None, fake, 1 << 20, None) == qoh.ARCHEAD_EINVAL
    assert L.archead_sample(fake, fake, 1, 1.0, 1, 0, fake + 2, None, None, fake, 1 << 20, None) == \
        qoh.ARCHEAD_EALIGN
    assert L.archead_set_vocab_shard(None, 0, 10) == qoh.ARCHEAD_EINVAL
    assert L.archead_shard_partials(fake, fake, 1, None, None, fake, 1 << 20, None) == qoh.ARCHEAD_EINVAL
    assert L.archead_shard_partials(fake, fake, 1, None, fake + 4, fake, 1 << 20, None) == qoh.ARCHEAD_EALIGN
    assert L.archead_merge_shards(None, 2, 1, fake, fake, fake, None) == qoh.ARCHEAD_EINVAL
    assert L.archead_merge_shards(fake, 0, 1, fake, fake, fake, None) == qoh.ARCHEAD_EINVAL
    assert L.archead_merge_shards(fake, 2, 0, fake, fake, fake, None) == qoh.ARCHEAD_EINVAL
    assert L.archead_merge_shards(fake, 2, 1, None, None, None, None) == qoh.ARCHEAD_EINVAL
    assert L.archead_merge_shards(fake + 4, 2, 1, fake, fake, fake, None) == qoh.ARCHEAD_EALIGN
    for temp in (0.0, float("inf")):
        assert L.archead_sample_partials(fake, fake, 1, temp, 1, 0, fake, fake, 1 << 20, None) == qoh.ARCHEAD_EINVAL
    assert L.archead_sample_partials(fake, fake, 1, 1.0, 1, 0, None, fake, 1 << 20, None) == qoh.ARCHEAD_EINVAL
    assert L.archead_sample_partials(fake, fake, 1, 1.0, 1, 0, fake + 4, fake, 1 << 20, None) == qoh.ARCHEAD_EALIGN
    assert L.archead_merge_sample_shards(None, 2, 1, fake, None) == qoh.ARCHEAD_EINVAL
    assert L.archead_merge_sample_shards(fake, 0, 1, fake, None) == qoh.ARCHEAD_EINVAL
    assert L.archead_merge_sample_shards(fake, 2, 1, None, None) == qoh.ARCHEAD_EINVAL
    assert L.archead_merge_sample_shards(fake + 4, 2, 1, fake, None) == qoh.ARCHEAD_EALIGN
    status = ct.c_uint32(0)
    assert L.archead_workspace_status(None, 0, None, ct.byref(status)) == qoh.ARCHEAD_EINVAL
    assert L.archead_workspace_status(fake + 16, 0, None, ct.byref(status)) == qoh.ARCHEAD_EALIGN


def test_builder_svd_options_are_checked_first(qoh):
    """Bad randomised-SVD options: the binding refuses an unknown method, and
    the library returns EINVAL before it touches a pointer or the GPU."""
    import ctypes as ct
    import quantized_output_head_b200.builder as bld
    with pytest.raises(ValueError):
        bld.svd_opts("approximate")
    fake = 4096                                   # never dereferenced: the option check fails first
    desc = bld._desc(1024, 256, 32, 8, 64, 64)
    comps = bld.ArcheadDeviceComponents(*([fake] * 10))
    for method, oversample, iters in ((7, 8, 2), (bld.ARCHEAD_SVD_RANDOMIZED, -1, 2),
                                      (bld.ARCHEAD_SVD_RANDOMIZED, 8, 65)):
        opts = bld.ArcheadSvdOpts(method, oversample, iters, 1)
        assert bld._blib.archead_build_head_svd(ct.byref(desc), fake, fake, 16, 0.01, 0.75, ct.byref(opts),
                                                ct.byref(comps), fake, 1 << 20, None) == qoh.ARCHEAD_EINVAL
        assert bld._blib.archead_build_correction_svd(ct.byref(desc), fake, fake, fake, ct.byref(opts), fake, fake,
                                                      fake, fake, fake, 1 << 20, None) == qoh.ARCHEAD_EINVAL


def test_builder_binding_refuses_host_or_wrongly_typed_tensors(qoh):
    """The construction binding checks its tensors before it calls the library."""
    import torch
    import quantized_output_head_b200.builder as bld
    with pytest.raises(ValueError):
        bld.quantize(torch.zeros(4, 64, dtype=torch.float64), 4, 16)          # host tensor
    with pytest.raises(ValueError):
        bld.metric(torch.zeros(64, 32, dtype=torch.float64), 0.01, 0.75)      # fp64, host
    with pytest.raises(ValueError):
        bld.build_head(torch.zeros(32, 64), torch.zeros(16, 64), 4, 2, 16, 16)
