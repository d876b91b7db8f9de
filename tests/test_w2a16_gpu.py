"""Parity of the W2A16 consumer GEMM (bq_w2a16_gemm, bq_w2a16_linear) with the float64
oracle.

Tolerance, derived from the arithmetic: the dequantized weight and the products are
exact (bf16 x bf16 fits float32), so the only error is the float32 accumulation.  A
tensor-core K = 16 step adds its products into the accumulator with one rounding
of at most one float32 ulp, so over K / 16 steps
    |out - exact| <= (K / 16 + 1) * 2^-23 * sum_k |x_k w_k|;
a bfloat16 output adds its round-to-nearest error, 2^-8 of the value."""

import numpy as np
import pytest

from oracle import butterfly as ob
from oracle import w2a16 as ow
from rotation_bit_quantization_b200 import workloads as wl
from tests import helpers as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bq():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import rotation_bit_quantization_b200 as bq_mod
    from rotation_bit_quantization_b200 import build
    build.build()
    bq_mod.load()
    return bq_mod


def _dev_weights(codes, s16, z16):
    torch = H.torch()
    return (torch.from_numpy(np.ascontiguousarray(codes)).cuda(),
            torch.from_numpy(np.ascontiguousarray(s16).view(np.int16)).cuda(),
            torch.from_numpy(np.ascontiguousarray(z16).view(np.int16)).cuda())


def _gemm(bq, xb, codes, s16, z16, bits, group, bf16_out, split=True):
    torch = H.torch()
    x = H.dev_bf16_bits(xb)
    c, s, z = _dev_weights(codes, s16, z16)
    out = torch.empty((xb.shape[0], codes.shape[0]), dtype=torch.bfloat16 if bf16_out else torch.float32,
                      device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = None
    if split:
        nbytes = bq.bq_w2a16_gemm_workspace_size(xb.shape[0], xb.shape[1], codes.shape[0])
        ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device="cuda")
    bq.bq_w2a16_gemm(x, c, s, z, bits, group, out, workspace=ws, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return H.host(out)


def _as_f64(host_out, bf16_out):
    return (wl.f32_from_bf16_bits(host_out) if bf16_out else host_out).astype(np.float64)


def _assert_close(got, ref, sum_abs, n, bf16_out):
    tol = (n / 16 + 1) * 2.0 ** -23 * sum_abs
    if bf16_out:
        tol = tol * 1.01 + 2.0 ** -8 * np.abs(ref) + 1e-38
    err = np.abs(got - ref)
    worst = np.unravel_index(np.argmax(err - tol), err.shape)
    assert np.all(err <= tol), f"at {worst}: err {err[worst]:.3e} > tol {tol[worst]:.3e}"
    return float((err / np.maximum(sum_abs, 1e-300)).max())


def _inputs(seed, tokens, n, out, bits, group):
    rng = np.random.default_rng(seed)
    xb = wl.bf16_bits_from_f32((rng.standard_normal((tokens, n)) * 0.5).astype(np.float32))
    codes, s16, z16 = wl.packed_weights(rng, out, n, bits, group)
    return xb, codes, s16, z16


@pytest.mark.parametrize("tokens,n,out,bits,group,bf16_out", [
    (1, 256, 128, 2, 64, False),          # one token, one tile
    (100, 1024, 200, 2, 128, False),      # ragged tokens and features (partial 32-column chunk)
    (300, 4096, 384, 4, 128, True),       # two token tiles, INT4, bf16 out
    (512, 2048, 1000, 4, 256, False),     # last feature tile 104 wide
    (257, 512, 136, 2, 64, True),         # one token past a tile
    (64, 512, 130, 4, 64, False),         # features not a multiple of 8: scalar stores
    (1024, 1024, 6144, 2, 128, True),     # 192 tiles: CTAs run more than one tile
])
def test_gemm_matches_oracle(bq, tokens, n, out, bits, group, bf16_out):
    xb, codes, s16, z16 = _inputs(tokens * 7 + out + bits, tokens, n, out, bits, group)
    got = _as_f64(_gemm(bq, xb, codes, s16, z16, bits, group, bf16_out), bf16_out)
    ref, sum_abs = ow.w2a16_gemm(wl.f32_from_bf16_bits(xb), codes, s16, z16, bits, group)
    rel = _assert_close(got, ref, sum_abs, n, bf16_out)
    if not bf16_out:
        assert rel < 2.0 ** -16            # the typical float32 error is far inside the bound


@pytest.mark.parametrize("tokens,n,out,bits,group", [
    (4, 256, 128, 2, 64),        # one 32-token chunk
    (100, 1024, 200, 2, 128),    # 4 chunks of a 112-token tile, ragged features
    (200, 512, 264, 4, 256),     # 7 chunks: six parked in tensor memory, one in registers
    (257, 512, 136, 2, 64),      # a full tile (eight chunks) and a one-token tile
    (300, 1024, 130, 4, 128),    # features not a multiple of 8: scalar stores
])
def test_gemm_bf16_unsplit_drained_epilogue(bq, tokens, n, out, bits, group):
    """bfloat16 output without a K split: the epilogue drains the accumulator (bf16
    pairs, chunks 0-5 in spare tensor-memory columns, 6-7 in registers) before the
    transposed stores.  Each output is the float32 result rounded once, so it equals
    the float32-output run rounded to bfloat16."""
    xb, codes, s16, z16 = _inputs(tokens * 5 + out + bits, tokens, n, out, bits, group)
    got = _gemm(bq, xb, codes, s16, z16, bits, group, True, split=False)
    f32 = _gemm(bq, xb, codes, s16, z16, bits, group, False, split=False)
    assert np.array_equal(got, wl.bf16_bits_from_f32(f32.astype(np.float32)))
    ref, sum_abs = ow.w2a16_gemm(wl.f32_from_bf16_bits(xb), codes, s16, z16, bits, group)
    _assert_close(_as_f64(got, True), ref, sum_abs, n, True)


@pytest.mark.parametrize("tokens,out,bits,group", [(1, 11008, 2, 128), (16, 11008, 2, 128), (7, 4096, 4, 128),
                                                  (40, 1000, 2, 64), (100, 2048, 4, 256), (2, 1000, 4, 64),
                                                  (3, 130, 2, 256), (4, 4096, 4, 128), (1, 200, 4, 128),
                                                  (9, 1001, 2, 64), (17, 700, 4, 128), (8, 24, 2, 256)])
def test_gemm_decode_sizes(bq, tokens, out, bits, group):
    """Few tokens: 1-8 tokens run on the decode kernel (warp-level MMAs on weights
    expanded in registers), more split K over the SMs and add the slices in a fixed
    order; either way the result matches the oracle, repeats bitwise, and agrees with
    the unsplit kernel to float32 summation order."""
    n = 4096
    xb, codes, s16, z16 = _inputs(tokens + out + 3 * bits, tokens, n, out, bits, group)
    torch = H.torch()
    assert (bq.bq_w2a16_gemm_workspace_size(tokens, n, out) > 0) == (tokens > 8)
    got = _as_f64(_gemm(bq, xb, codes, s16, z16, bits, group, False), False)
    again = _as_f64(_gemm(bq, xb, codes, s16, z16, bits, group, False), False)
    assert np.array_equal(got, again)
    ref, sum_abs = ow.w2a16_gemm(wl.f32_from_bf16_bits(xb), codes, s16, z16, bits, group)
    rel = _assert_close(got, ref, sum_abs, n, False)
    assert rel < 2.0 ** -16
    unsplit = _as_f64(_gemm(bq, xb, codes, s16, z16, bits, group, False, split=False), False)
    _assert_close(unsplit, ref, sum_abs, n, False)
    bf = _as_f64(_gemm(bq, xb, codes, s16, z16, bits, group, True), True)
    _assert_close(bf, ref, sum_abs, n, True)


def test_gemm_full_layer_sampled_tokens_and_determinism(bq):
    """The LLaMA-2-7B MLP shape (2048 x 4096 activations, 11008 x 4096 INT2 g128
    weights, 688 tiles, several per CTA): sampled tokens against the oracle, and two
    runs bitwise equal."""
    xb, codes, s16, z16, bits, group = wl.w2a16_4096()
    got = _gemm(bq, xb, codes, s16, z16, bits, group, True)
    again = _gemm(bq, xb, codes, s16, z16, bits, group, True)
    assert np.array_equal(got, again)
    rows = np.random.default_rng(1).choice(xb.shape[0], 48, replace=False)
    rows = np.unique(np.concatenate([rows, [0, xb.shape[0] - 1]]))
    ref, sum_abs = ow.w2a16_gemm(wl.f32_from_bf16_bits(xb[rows]), codes, s16, z16, bits, group)
    _assert_close(_as_f64(got[rows], True), ref, sum_abs, 4096, True)


def test_gemm_zero_tokens_is_a_no_op(bq):
    torch = H.torch()
    x = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    c, s, z = _dev_weights(*wl.packed_weights(np.random.default_rng(0), 128, 256, 2, 64))
    out = torch.full((0, 128), 7.0, dtype=torch.float32, device="cuda")
    bq.bq_w2a16_gemm(x, c, s, z, 2, 64, out)
    torch.cuda.synchronize()


def test_linear_is_forward_then_gemm_and_matches_oracle(bq):
    torch = H.torch()
    m, tokens, out, bits, group = 4096, 300, 256, 2, 128
    rng = np.random.default_rng(21)
    theta = wl.uniform_angles(rng, m)
    x = (rng.standard_normal((tokens, m)) * 0.5).astype(np.float32)
    codes, s16, z16 = wl.packed_weights(rng, out, m, bits, group)
    layer = bq.Layer(H.dev_f32(theta))
    xd = H.dev_f32(x)
    c, s, z = _dev_weights(codes, s16, z16)
    ws = torch.empty(bq.bq_w2a16_linear_workspace_size(m, tokens, out), dtype=torch.uint8, device="cuda")
    y = torch.empty((tokens, out), dtype=torch.float32, device="cuda")
    bq.bq_w2a16_linear(layer, xd, c, s, z, bits, group, y, ws)
    # the same two steps called separately
    xt = torch.empty((tokens, m), dtype=torch.bfloat16, device="cuda")
    bq.bq_butterfly_fwd(layer, xd, xt)
    y2 = torch.empty_like(y)
    gws = torch.empty(max(bq.bq_w2a16_gemm_workspace_size(tokens, m, out), 256), dtype=torch.uint8, device="cuda")
    bq.bq_w2a16_gemm(xt, c, s, z, bits, group, y2, workspace=gws)
    torch.cuda.synchronize()
    assert torch.equal(y, y2)
    # oracle: Q x in float64 rounded to bf16; the GPU's bf16 rotated activations may sit
    # one bf16 ulp (2^-7 relative) and the float32 bound (2e-5 ||x||) away from it
    xr = ow.bf16_round(ob.forward(theta, x.astype(np.float64)).astype(np.float32)).astype(np.float64)
    ref, sum_abs = ow.w2a16_gemm(xr, codes, s16, z16, bits, group)
    w_abs = np.abs(ow.dequantize_bf16(codes, s16, z16, bits, group, m)).astype(np.float64).sum(axis=1)
    tol = (m / 16 + 1) * 2.0 ** -23 * sum_abs + 2.0 ** -7 * sum_abs \
        + H.F32_TOL * np.linalg.norm(x, axis=1)[:, None] * w_abs[None, :]
    assert np.all(np.abs(H.host(y).astype(np.float64) - ref) <= tol)


def test_quantized_layer_end_to_end_reproduces_the_float_layer(bq):
    """y = W x = (W Q^T)(Q x): rotate-pack W on the GPU, then bq_w2a16_linear on the raw
    activations.  The result equals the oracle's exact product of the same bf16 operands
    (the bound above), and differs from the float layer W x only by the weight
    quantization: |y - W x| <= sum_k |x~_k| s_k / 2 (each weight within half a step of
    its code), plus the bf16 rounding of the operands."""
    torch = H.torch()
    m, tokens, out, bits, group = 4096, 64, 512, 4, 128
    rng = np.random.default_rng(31)
    theta = wl.uniform_angles(rng, m)
    w = (rng.standard_normal((out, m)) * 0.02).astype(np.float32)
    x = (rng.standard_normal((tokens, m)) * 0.5).astype(np.float32)
    layer = bq.Layer(H.dev_f32(theta))
    codes, scale, zero = bq.quant_outputs(out, m, bits, group, "cuda")
    bq.bq_weight_rotate_pack(layer, H.dev_f32(w), bits, group, codes, scale, zero)
    y = torch.empty((tokens, out), dtype=torch.float32, device="cuda")
    ws = torch.empty(bq.bq_w2a16_linear_workspace_size(m, tokens, out), dtype=torch.uint8, device="cuda")
    bq.bq_w2a16_linear(layer, H.dev_f32(x), codes, scale, zero, bits, group, y, ws)
    torch.cuda.synchronize()
    got = H.host(y).astype(np.float64)
    exact = x.astype(np.float64) @ w.astype(np.float64).T
    xt = ob.forward(theta, x.astype(np.float64))
    s = H.host(scale).view(np.uint16).view(np.float16).astype(np.float64)       # (out, m/group)
    step = np.repeat(s, group, axis=1)                                          # per weight
    qerr = np.abs(xt) @ (step / 2).T + 2.0 ** -7 * (np.abs(xt) @ np.abs(ob.forward(theta, w.astype(np.float64))).T)
    assert np.all(np.abs(got - exact) <= qerr * 1.05 + 1e-4)
    # and the quantized layer is much closer to W x than a zero output would be
    assert np.linalg.norm(got - exact) < 0.2 * np.linalg.norm(exact)
