"""Pins of the W2A16 GEMM oracle (oracle/w2a16.py) against what fixes it from
outside: the library's float32 -> bfloat16 conversion, an exact integer
evaluation of the dequantized product, a layer whose weights the quantizer
reproduces exactly (so the GEMM must equal x W^T), and planted mistakes."""

import numpy as np
import pytest

from oracle import quant as oq
from oracle import w2a16 as ow


def test_bf16_round_matches_library_conversion():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * np.float32(1e3),
        (rng.standard_normal(2000) * 1e-38).astype(np.float32),           # subnormals
        np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8), 3.3895314e38, 3.4e38,
                  np.inf, -np.inf, 0.0, -0.0, 2.0 ** -133], dtype=np.float32),
    ]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    got = ow.bf16_round(x)
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))
    assert np.isnan(ow.bf16_round(np.array([np.nan], dtype=np.float32)))[0]


def _integer_case(rng, tokens, n, out, bits, group):
    """Codes, fp16 power-of-two scales, zero points and small integer activations,
    with the product evaluated exactly in integers."""
    qmax = 2 ** bits - 1
    q = rng.integers(0, qmax + 1, size=(out, n)).astype(np.uint8)
    z = rng.integers(0, qmax + 1, size=(out, n // group))
    e = rng.integers(0, 9, size=(out, n // group))                        # s = 2^-e
    s16 = (2.0 ** -e).astype(np.float16).view(np.uint16)
    z16 = z.astype(np.float16).view(np.uint16)
    x = rng.integers(-128, 129, size=(tokens, n)).astype(np.int64)
    # sum_g 2^(8 - e_og) sum_{k in g} x_k (q_ok - z_og), an exact integer, then / 2^8
    d = q.astype(np.int64).reshape(out, n // group, group) - z[..., None]
    per_group = np.einsum("tgk,ogk->tog", x.reshape(tokens, n // group, group), d)
    exact = (per_group * (2 ** (8 - e))[None]).sum(axis=-1)
    return x, oq.pack(q, bits), s16, z16, exact / 256.0


@pytest.mark.parametrize("bits,group", [(2, 64), (2, 128), (4, 128), (4, 256)])
def test_gemm_matches_exact_integer_evaluation(bits, group):
    rng = np.random.default_rng(bits * 1000 + group)
    x, codes, s16, z16, exact = _integer_case(rng, 7, 512, 9, bits, group)
    out, sum_abs = ow.w2a16_gemm(x.astype(np.float32), codes, s16, z16, bits, group)
    assert np.array_equal(out, exact)
    assert np.all(sum_abs >= np.abs(out))


def test_gemm_of_an_exactly_quantizable_layer_is_the_plain_product():
    """W = (q - z) s with every group holding levels 0 and qmax: the quantizer
    returns q, s and z themselves, and (q - z) s is a bfloat16 value, so the
    GEMM of the packed weights is x W^T."""
    rng = np.random.default_rng(5)
    bits, group, n, out = 2, 128, 1024, 24
    qmax = 2 ** bits - 1
    q = rng.integers(0, qmax + 1, size=(out, n))
    q[:, ::group] = 0
    q[:, 1::group] = qmax
    z = rng.integers(0, qmax + 1, size=(out, n // group))
    s = 2.0 ** -rng.integers(2, 7, size=(out, n // group))
    w = ((q.reshape(out, n // group, group) - z[..., None]) * s[..., None]).reshape(out, n).astype(np.float32)
    codes, s16, z16 = oq.quantize_pack(w, bits, group)
    x = ow.bf16_round(rng.standard_normal((5, n)).astype(np.float32))
    got, _ = ow.w2a16_gemm(x, codes, s16, z16, bits, group)
    assert np.array_equal(got, x.astype(np.float64) @ w.astype(np.float64).T)


def test_planted_unpack_order_and_zero_sign_are_caught(monkeypatch):
    rng = np.random.default_rng(11)
    bits, group = 2, 64
    x, codes, s16, z16, exact = _integer_case(rng, 3, 256, 4, bits, group)
    # a planted mistake in the oracle: codes read from the top bits of each byte down
    real_unpack = oq.unpack

    def reversed_unpack(packed, b, n):
        c = real_unpack(packed, b, n)
        per = 8 // b
        return c.reshape(c.shape[0], -1, per)[..., ::-1].reshape(c.shape)

    monkeypatch.setattr(oq, "unpack", reversed_unpack)
    bad, _ = ow.w2a16_gemm(x.astype(np.float32), codes, s16, z16, bits, group)
    assert not np.array_equal(bad, exact)
    monkeypatch.setattr(oq, "unpack", real_unpack)
    # a planted mistake: the zero point added instead of subtracted
    real_deq = oq.dequantize

    def plus_zero(cd, sc, zr, g):
        return real_deq(cd, sc, zr, g) + 2 * real_deq(np.zeros_like(cd), sc, zr, g) * -1.0

    monkeypatch.setattr(oq, "dequantize", plus_zero)
    bad, _ = ow.w2a16_gemm(x.astype(np.float32), codes, s16, z16, bits, group)
    assert not np.array_equal(bad, exact)
