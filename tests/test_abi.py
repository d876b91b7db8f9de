"""The C ABI library loads, exports every symbol include/bq.h declares, and
rejects bad arguments on the host before touching the GPU (no compute here)."""

import ctypes
import os
import re

import numpy as np

import pytest

from rotation_bit_quantization_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "bq.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(bq_\w+)\s*\(", text)))


def test_header_declares_the_entry_points():
    syms = declared_symbols()
    for name in ("bq_butterfly_fwd", "bq_butterfly_inv", "bq_butterfly_bwd", "bq_transform_quantize",
                 "bq_weight_rotate_pack"):
        assert name in syms
    assert set(syms) == set(_lib.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
    out = os.popen(f"nm -D --defined-only {_lib.LIB_PATH}").read()
    for name in declared_symbols():
        assert re.search(rf"\bT {name}\b", out), name


def test_status_strings(lib):
    assert _lib.status_string(0) == "ok"
    assert "invalid" in _lib.status_string(1)
    assert _lib.status_string(99) == "unknown status"


def test_table_sizes(lib):
    assert lib.bq_table_floats(4096) > 2 * 12 * 4096
    assert lib.bq_table_floats(3) == 0
    assert lib.bq_table_floats(8192) == 0          # above the supported width
    assert lib.bq_table_floats(1) == 0


def test_workspace_size(lib):
    ws = lib.bq_butterfly_bwd_workspace_size(4096, 32, 65536)
    assert ws >= 32 * 24576 * 4
    assert lib.bq_butterfly_bwd_workspace_size(4096, 0, 10) == 0
    assert lib.bq_butterfly_bwd_workspace_size(4096, 129, 10) == 0
    assert lib.bq_butterfly_bwd_workspace_size(5000, 2, 10) == 0


def _layer(n, m, r, table=16, O=None):
    return _lib.BQLayer(n, m, r, table, O)


FAKE = 0x10000  # 16-byte aligned, never dereferenced: validation fails first or nothing is launched


@pytest.mark.parametrize("layer,why", [
    (_layer(4096, 4096, 1, table=None), "null table"),
    (_layer(4096, 4096, 1, table=FAKE + 4), "misaligned table"),
    (_layer(4095, 4095, 1, table=FAKE), "m not a power of two"),
    (_layer(8192, 8192, 1, table=FAKE), "m too large"),
    (_layer(4096, 1024, 5, table=FAKE), "n != m*r"),
    (_layer(5120, 1024, 5, table=FAKE), "r > 1 without O"),
    (_layer(1024, 1024, 1, table=FAKE, O=FAKE), "O given with r == 1"),
    (_layer(9 * 1024, 1024, 9, table=FAKE, O=FAKE), "r too large"),
])
def test_fwd_rejects_bad_layers(lib, layer, why):
    st = lib.bq_butterfly_fwd(ctypes.byref(layer), FAKE, 0, FAKE, 0, 4, None)
    assert st == _lib.BQ_ERR_INVALID_ARG, why


def test_fwd_rejects_bad_buffers(lib):
    good = _layer(256, 256, 1, table=FAKE)
    assert lib.bq_butterfly_fwd(ctypes.byref(good), None, 0, FAKE, 0, 4, None) == _lib.BQ_ERR_INVALID_ARG
    assert lib.bq_butterfly_fwd(ctypes.byref(good), FAKE + 8, 0, FAKE, 0, 4, None) == _lib.BQ_ERR_INVALID_ARG
    assert lib.bq_butterfly_fwd(ctypes.byref(good), FAKE, 7, FAKE, 0, 4, None) == _lib.BQ_ERR_INVALID_ARG
    assert lib.bq_butterfly_fwd(ctypes.byref(good), FAKE, 0, FAKE, 1, 4, None) == _lib.BQ_ERR_INVALID_ARG  # alias, dtypes differ
    assert lib.bq_butterfly_fwd(ctypes.byref(good), FAKE, 0, FAKE, 0, -1, None) == _lib.BQ_ERR_INVALID_ARG
    assert lib.bq_butterfly_fwd(ctypes.byref(good), None, 0, None, 0, 0, None) == _lib.BQ_OK   # empty: no launch
    assert lib.bq_butterfly_inv(None, FAKE, 0, FAKE, 0, 4, None) == _lib.BQ_ERR_INVALID_ARG


@pytest.mark.parametrize("bits,group,ok", [(3, 128, False), (4, 48, False), (4, 100, False), (2, 512, False),
                                           (4, 96, False), (4, 0, False)])
def test_quantize_rejects_bad_settings(lib, bits, group, ok):
    good = _layer(4096, 4096, 1, table=FAKE)
    st = lib.bq_transform_quantize(ctypes.byref(good), FAKE, 0, 8, bits, group, FAKE, FAKE, FAKE, None)
    assert st == _lib.BQ_ERR_INVALID_ARG
    st = lib.bq_weight_rotate_pack(ctypes.byref(good), FAKE, 0, 8, bits, group, FAKE, FAKE, FAKE, None)
    assert st == _lib.BQ_ERR_INVALID_ARG


def test_quantize_rejects_null_outputs(lib):
    good = _layer(4096, 4096, 1, table=FAKE)
    assert lib.bq_transform_quantize(ctypes.byref(good), FAKE, 0, 8, 4, 128, None, FAKE, FAKE, None) == 1
    assert lib.bq_transform_quantize(ctypes.byref(good), FAKE, 0, 8, 4, 128, FAKE, FAKE + 2, FAKE, None) == 1
    assert lib.bq_transform_quantize(ctypes.byref(good), FAKE, 0, 0, 4, 128, None, None, None, None) == 0


def test_wait_faults_rejects_null_before_any_cuda_call(lib):
    assert lib.bq_wait_faults(None, 0, None) == _lib.BQ_ERR_INVALID_ARG
    assert lib.bq_wait_faults(None, 1, None) == _lib.BQ_ERR_INVALID_ARG


def test_bwd_rejects_bad_arguments(lib):
    L = (_lib.BQLayer * 2)(_layer(64, 64, 1, table=FAKE), _layer(64, 64, 1, table=FAKE))
    ws = lib.bq_butterfly_bwd_workspace_size(64, 2, 10)
    args = [FAKE, 0, FAKE, 0, FAKE, FAKE, FAKE, 10, FAKE]
    assert lib.bq_butterfly_bwd(L, 2, *args, ws - 1, None) == _lib.BQ_ERR_WORKSPACE
    assert lib.bq_butterfly_bwd(L, 0, *args, ws, None) == _lib.BQ_ERR_INVALID_ARG
    assert lib.bq_butterfly_bwd(None, 2, *args, ws, None) == _lib.BQ_ERR_INVALID_ARG
    bad = list(args); bad[4] = None
    assert lib.bq_butterfly_bwd(L, 2, *bad, ws, None) == _lib.BQ_ERR_INVALID_ARG
    mixed = (_lib.BQLayer * 2)(_layer(64, 64, 1, table=FAKE), _layer(32, 32, 1, table=FAKE))
    assert lib.bq_butterfly_bwd(mixed, 2, *args, ws, None) == _lib.BQ_ERR_INVALID_ARG
    kron = (_lib.BQLayer * 1)(_layer(320, 64, 5, table=FAKE, O=FAKE))
    assert lib.bq_butterfly_bwd(kron, 1, *args, ws, None) == _lib.BQ_ERR_UNSUPPORTED


@pytest.mark.parametrize("layer,status", [
    (_layer(64, 64, 0, table=FAKE), _lib.BQ_ERR_INVALID_ARG),          # r = 0
    (_layer(64 * 9, 64, 9, table=FAKE, O=FAKE), _lib.BQ_ERR_INVALID_ARG),  # r above the limit
    (_layer(320, 64, 5, table=FAKE, O=FAKE), _lib.BQ_ERR_UNSUPPORTED),  # a valid composite: no backward
    (_layer(320, 64, 5, table=FAKE), _lib.BQ_ERR_INVALID_ARG),          # r > 1 without O
    (_layer(64, 64, 1, table=FAKE, O=FAKE), _lib.BQ_ERR_INVALID_ARG),   # O with r == 1
    (_layer(64, 64, 1, table=FAKE + 4), _lib.BQ_ERR_INVALID_ARG),       # misaligned table
])
def test_both_backward_entry_points_reject_bad_layers_alike(lib, layer, status):
    """The allocation-free backward validates its layers exactly as bq_butterfly_bwd does."""
    L = (_lib.BQLayer * 1)(layer)
    args = [FAKE, 0, FAKE, 0, FAKE, FAKE, FAKE, 10]
    ws = 1 << 30
    assert lib.bq_butterfly_bwd(L, 1, *args, FAKE, ws, None) == status
    assert lib.bq_butterfly_bwd_noalloc(L, 1, *args, None) == status


def test_noalloc_rejects_what_does_not_fit_its_scratch(lib):
    # 86 layers of width 4096 need more than the 8 MiB of fixed scratch even at one
    # token chunk per layer (98,304 bytes of partials each); nothing is launched
    L = (_lib.BQLayer * 86)(*[_layer(4096, 4096, 1, table=FAKE) for _ in range(86)])
    args = [FAKE, 0, FAKE, 0, FAKE, FAKE, FAKE, 10]
    assert lib.bq_butterfly_bwd_noalloc(L, 86, *args, None) == _lib.BQ_ERR_WORKSPACE
    assert lib.bq_butterfly_bwd_noalloc(L, 0, *args, None) == _lib.BQ_ERR_INVALID_ARG


def test_precompute_rejects_bad_width(lib):
    assert lib.bq_precompute_cs(FAKE, 12, FAKE, None) == _lib.BQ_ERR_INVALID_ARG
    assert lib.bq_precompute_cs(None, 16, FAKE, None) == _lib.BQ_ERR_INVALID_ARG
    assert lib.bq_precompute_cs(FAKE, 16, FAKE + 4, None) == _lib.BQ_ERR_INVALID_ARG


def test_binding_fails_loudly_without_library(tmp_path):
    saved = _lib._lib
    try:
        _lib._lib = None
        with pytest.raises(ImportError):
            _lib.load(str(tmp_path / "missing.so"))
    finally:
        _lib._lib = saved


@pytest.mark.parametrize("bits,group,eps", [(3, 128, 1e-4), (4, 96, 1e-4), (4, 32, 1e-4), (2, 128, 0.0),
                                            (2, 128, 1.0), (2, 128, float("nan"))])
def test_uniformity_rejects_bad_settings(lib, bits, group, eps):
    st = lib.bq_uniformity_loss(FAKE, 4, 4096, bits, group, eps, FAKE, FAKE, FAKE, None)
    assert st == _lib.BQ_ERR_INVALID_ARG


def test_uniformity_rejects_bad_buffers(lib):
    assert lib.bq_uniformity_loss(None, 4, 4096, 4, 128, 1e-4, FAKE, FAKE, FAKE, None) == _lib.BQ_ERR_INVALID_ARG
    assert lib.bq_uniformity_loss(FAKE, 4, 4096, 4, 128, 1e-4, None, FAKE, FAKE, None) == _lib.BQ_ERR_INVALID_ARG
    assert lib.bq_uniformity_loss(FAKE + 4, 4, 4096, 4, 128, 1e-4, FAKE, FAKE, FAKE, None) == _lib.BQ_ERR_INVALID_ARG
    assert lib.bq_uniformity_loss(FAKE, 4, 4000, 4, 128, 1e-4, FAKE, FAKE, FAKE, None) == _lib.BQ_ERR_INVALID_ARG
    assert lib.bq_uniformity_loss(FAKE, -1, 4096, 4, 128, 1e-4, FAKE, FAKE, FAKE, None) == _lib.BQ_ERR_INVALID_ARG
    assert lib.bq_uniformity_loss(FAKE, 0, 4096, 4, 128, 1e-4, FAKE, FAKE, FAKE, None) == _lib.BQ_OK  # nothing to do


def test_angle_sgd_rejects_bad_arguments(lib):
    assert lib.bq_angle_sgd(None, FAKE, 8, 0.1, None) == _lib.BQ_ERR_INVALID_ARG
    assert lib.bq_angle_sgd(FAKE, FAKE, -1, 0.1, None) == _lib.BQ_ERR_INVALID_ARG
    assert lib.bq_angle_sgd(FAKE, FAKE, 8, float("nan"), None) == _lib.BQ_ERR_INVALID_ARG
    assert lib.bq_angle_sgd(FAKE, FAKE, 0, 0.1, None) == _lib.BQ_OK


def test_reconstruction_rejects_bad_arguments(lib):
    assert lib.bq_reconstruction_workspace_size(256, 16, 8, 2, 64) > 0
    assert lib.bq_reconstruction_workspace_size(250, 16, 8, 2, 64) == 0      # not a power of two
    assert lib.bq_reconstruction_workspace_size(256, 0, 8, 2, 64) == 0
    assert lib.bq_reconstruction_workspace_size(256, 16, 8, 3, 64) == 0
    assert lib.bq_reconstruction_workspace_size(256, 16, 8, 2, 48) == 0
    good = _lib.BQLayer(256, 256, 1, FAKE, None)
    kron = _lib.BQLayer(256 * 3, 256, 3, FAKE, FAKE)
    args = (FAKE, 16, FAKE, 8, 2, 64, FAKE, FAKE, FAKE)
    assert lib.bq_reconstruction_loss(ctypes.byref(good), *args, 16, None) == _lib.BQ_ERR_WORKSPACE
    assert lib.bq_reconstruction_loss(ctypes.byref(kron), *args, 1 << 30, None) == _lib.BQ_ERR_UNSUPPORTED
    assert lib.bq_reconstruction_loss(None, *args, 1 << 30, None) == _lib.BQ_ERR_INVALID_ARG


def test_w2a16_rejects_bad_arguments(lib):
    ok = (FAKE, 16, 256, FAKE, FAKE, FAKE, 128, 2, 64, FAKE, _lib.BQ_F32, None, 0, None, None)

    def call(**kw):
        names = ("x", "tokens", "n", "codes", "scale", "zero", "out_features", "bits", "group", "out", "out_t",
                 "ws", "ws_bytes", "status", "stream")
        args = dict(zip(names, ok))
        args.update(kw)
        return lib.bq_w2a16_gemm(*[args[k] for k in names])

    bad = _lib.BQ_ERR_INVALID_ARG
    assert call(n=200) == bad                  # not a multiple of 64
    assert call(bits=3) == bad
    assert call(group=32) == bad
    assert call(n=320, group=128) == bad       # group does not divide n
    assert call(out_t=7) == bad
    assert call(x=None) == bad
    assert call(x=FAKE + 8) == bad             # misaligned activations
    assert call(codes=FAKE + 4) == bad
    assert call(tokens=-1) == bad
    assert call(tokens=0) == _lib.BQ_OK        # nothing to do, nothing launched
    assert call(out_features=0) == _lib.BQ_OK
    assert call(ws=FAKE + 16, ws_bytes=1 << 20) == bad      # workspace not 256-byte aligned
    assert lib.bq_w2a16_gemm_workspace_size(0, 4096, 128) == 0
    assert lib.bq_w2a16_gemm_workspace_size(16, 4000, 128) == 0
    assert lib.bq_w2a16_gemm_workspace_size(17, 4000, 128) == 0
    assert lib.bq_w2a16_linear_workspace_size(4096, 3, 0) == 4096 * 3 * 2
    assert lib.bq_w2a16_linear_workspace_size(256, 1, 0) == 512
    layer = _lib.BQLayer(256, 256, 1, FAKE, None)
    assert lib.bq_w2a16_linear(ctypes.byref(layer), FAKE, 0, 4, FAKE, FAKE, FAKE, 128, 2, 64, FAKE, 0, FAKE, 16,
                               None, None) == _lib.BQ_ERR_WORKSPACE
    assert lib.bq_w2a16_linear(ctypes.byref(layer), FAKE, 0, 4, FAKE, FAKE, FAKE, 128, 2, 64, FAKE, 0, FAKE + 16,
                               1 << 20, None, None) == bad


def test_hadamard_preset_rejects_bad_arguments(lib):
    assert lib.bq_precompute_hadamard(4095, None, FAKE, None, None) == _lib.BQ_ERR_INVALID_ARG
    assert lib.bq_precompute_hadamard(8192, None, FAKE, None, None) == _lib.BQ_ERR_INVALID_ARG
    assert lib.bq_precompute_hadamard(4096, None, None, None, None) == _lib.BQ_ERR_INVALID_ARG
    assert lib.bq_precompute_hadamard(4096, None, FAKE + 4, None, None) == _lib.BQ_ERR_INVALID_ARG
    assert lib.bq_precompute_hadamard(4096, None, FAKE, FAKE + 2, None) == _lib.BQ_ERR_INVALID_ARG


class _FakeCudaTensor:
    """Stands in for a CUDA tensor in the host-side error-path tests (no device needed)."""

    def __init__(self, shape, dtype):
        self.shape, self.dtype = shape, dtype
        self.is_cuda = True

    def is_contiguous(self):
        return True

    def data_ptr(self):
        return FAKE

    def numel(self):
        return int(np.prod(self.shape))

    def element_size(self):
        return 1


class _Stream:
    cuda_stream = 0


def test_binding_maps_a_failing_launch_to_an_exception(lib, monkeypatch):
    """A launch error (a fake cudaErrorMemoryAllocation reported by the library as
    BQ_ERR_CUDA) reaches the caller as BQError with that status and its name, and a
    rejected argument as BQ_ERR_INVALID_ARG: the binding never swallows a status."""
    import torch

    class FakeLib:
        def __getattr__(self, name):
            return getattr(lib, name)

        def bq_w2a16_gemm(self, *args):
            return _lib.BQ_ERR_CUDA

        def bq_uniformity_loss(self, *args):
            return _lib.BQ_ERR_INVALID_ARG

    monkeypatch.setattr(_lib, "_lib", FakeLib())
    x = _FakeCudaTensor((16, 256), torch.bfloat16)
    c = _FakeCudaTensor((128, 64), torch.uint8)
    s = _FakeCudaTensor((128, 4), torch.int16)
    out = _FakeCudaTensor((16, 128), torch.float32)
    with pytest.raises(_lib.BQError) as e:
        _lib.bq_w2a16_gemm(x, c, s, s, 2, 64, out, stream=_Stream())
    assert e.value.status == _lib.BQ_ERR_CUDA and "cuda" in str(e.value).lower()
    y = _FakeCudaTensor((4, 256), torch.float32)
    kl = _FakeCudaTensor((4, 2), torch.float32)
    with pytest.raises(_lib.BQError) as e:
        _lib.bq_uniformity_loss(y, 4, 128, 1e-4, kl, stream=_Stream())
    assert e.value.status == _lib.BQ_ERR_INVALID_ARG


def test_binding_rejects_host_tensors():
    import torch
    with pytest.raises(ValueError):
        _lib._dev(torch.zeros(4), "x")


def test_zero_rows_launch_nothing(lib):
    """Zero rows (tokens, features, count) return BQ_OK once the other arguments are
    valid, with NULL data pointers: nothing is launched (this runs without a GPU).
    The backward needs at least one token."""
    layer = ctypes.byref(_layer(4096, 4096, 1, table=FAKE))
    OK, BAD = _lib.BQ_OK, _lib.BQ_ERR_INVALID_ARG
    assert lib.bq_butterfly_fwd(layer, None, _lib.BQ_BF16, None, _lib.BQ_F32, 0, None) == OK
    assert lib.bq_butterfly_inv(layer, None, _lib.BQ_F32, None, _lib.BQ_BF16, 0, None) == OK
    assert lib.bq_butterfly_fwd(layer, None, 7, None, _lib.BQ_F32, 0, None) == BAD        # bad dtype first
    assert lib.bq_transform_quantize(layer, None, _lib.BQ_BF16, 0, 4, 128, None, None, None, None) == OK
    assert lib.bq_transform_quantize(layer, None, _lib.BQ_BF16, 0, 3, 128, None, None, None, None) == BAD
    assert lib.bq_weight_rotate_pack(layer, None, _lib.BQ_BF16, 0, 2, 128, None, None, None, None) == OK
    assert lib.bq_uniformity_loss(None, 0, 4096, 4, 128, 1e-4, None, None, None, None) == OK
    assert lib.bq_angle_sgd(None, None, 0, 0.1, None) == OK
    assert lib.bq_w2a16_gemm(None, 0, 4096, None, None, None, 11008, 2, 128, None, _lib.BQ_BF16, None, 0, None,
                             None) == OK
    assert lib.bq_w2a16_gemm(None, 16, 4096, None, None, None, 0, 2, 128, None, _lib.BQ_BF16, None, 0, None,
                             None) == OK
    assert lib.bq_w2a16_linear(layer, None, _lib.BQ_BF16, 0, None, None, None, 11008, 2, 128, None, _lib.BQ_BF16,
                               None, 0, None, None) == OK
    assert lib.bq_w2a16_linear(layer, None, _lib.BQ_BF16, 0, None, None, None, 11008, 3, 128, None, _lib.BQ_BF16,
                               None, 0, None, None) == BAD
    bwd_layers = (_lib.BQLayer * 1)(_layer(4096, 4096, 1, table=FAKE))
    assert lib.bq_butterfly_bwd(bwd_layers, 1, FAKE, _lib.BQ_BF16, FAKE, _lib.BQ_BF16, FAKE, FAKE, FAKE, 0, FAKE,
                                1 << 20, None) == BAD


def test_cuda_error_accessors(lib):
    """The library's own CUDA runtime error is readable through the ABI (host only)."""
    assert lib.bq_cuda_error_string(0) == b"no error"
    assert isinstance(lib.bq_cuda_error_string(2), bytes) and lib.bq_cuda_error_string(2)
    assert isinstance(int(lib.bq_cuda_last_error()), int)


def test_w2a16_workspace_plan(lib):
    """Host-side plan of the W2A16 GEMM (148 SMs when no device answers, the B200's
    count): no workspace for 1-8 tokens (the decode kernel) or once the output tiles
    fill the SMs; a split-K workspace of float32 partial rows in between, sized in
    whole 128-feature tiles; 0 for invalid shapes."""
    n, out = 4096, 11008
    f_tiles = (out + 127) // 128
    for t in range(1, 9):
        assert lib.bq_w2a16_gemm_workspace_size(t, n, out) == 0
    for t in (9, 16, 64, 128):
        ws = lib.bq_w2a16_gemm_workspace_size(t, n, out)
        ntok = max(16, (t + 15) // 16 * 16)
        assert ws > 0 and ws % (f_tiles * 128 * ntok * 4) == 0
        ksplit = ws // (f_tiles * 128 * ntok * 4)
        assert 2 <= ksplit <= n // 64 // 4                  # at least 4 K stages per slice
    assert lib.bq_w2a16_gemm_workspace_size(2048, n, out) == 0   # 688 tiles >= 148 SMs
    assert lib.bq_w2a16_gemm_workspace_size(0, n, out) == 0
    assert lib.bq_w2a16_gemm_workspace_size(17, 100, out) == 0   # n not a multiple of 64
    assert lib.bq_w2a16_linear_workspace_size(n, 32, out) >= 32 * n * 2 + lib.bq_w2a16_gemm_workspace_size(32, n, out)


def test_block_transform_rejects_bad_arguments(lib):
    f = lib.bq_block_transform_quantize
    assert lib.bq_block_table_bytes(4096, 32) == 4096 * 32 * 2
    assert lib.bq_block_table_bytes(100, 32) == 0 and lib.bq_block_table_bytes(4096, 8) == 0
    assert lib.bq_block_prepare(FAKE, 100, 32, FAKE, None) == _lib.BQ_ERR_INVALID_ARG
    assert lib.bq_block_prepare(FAKE, 128, 32, FAKE + 4, None) == _lib.BQ_ERR_INVALID_ARG
    args = dict(table=FAKE, C=256, G=32, x=FAKE, rows=4, fmt=_lib.BQ_BLOCK_MXFP4, gscale=1.0, y=None, yt=0,
                codes=FAKE, scales=FAKE, status=None)

    def call(**kw):
        a = dict(args, **kw)
        return f(a["table"], a["C"], a["G"], a["x"], a["rows"], a["fmt"], a["gscale"], a["y"], a["yt"], a["codes"],
                 a["scales"], a["status"], None)

    assert call(fmt=_lib.BQ_BLOCK_NVFP4) == _lib.BQ_ERR_INVALID_ARG            # NVFP4 needs G = 16
    assert call(G=16, fmt=_lib.BQ_BLOCK_INT4) == _lib.BQ_ERR_INVALID_ARG       # INT4 needs G = 32
    assert call(C=96) == _lib.BQ_ERR_INVALID_ARG
    assert call(rows=-1) == _lib.BQ_ERR_INVALID_ARG
    assert call(codes=None) == _lib.BQ_ERR_INVALID_ARG
    assert call(x=FAKE + 8) == _lib.BQ_ERR_INVALID_ARG
    assert call(fmt=_lib.BQ_BLOCK_NONE) == _lib.BQ_ERR_INVALID_ARG             # no y
    assert call(fmt=_lib.BQ_BLOCK_NONE, y=FAKE, yt=7) == _lib.BQ_ERR_INVALID_ARG
    assert call(G=16, fmt=_lib.BQ_BLOCK_NVFP4, gscale=0.0) == _lib.BQ_ERR_INVALID_ARG
    assert call(fmt=9) == _lib.BQ_ERR_INVALID_ARG
    assert call(rows=0, table=None, x=None) == _lib.BQ_OK                      # empty: nothing launched
