"""Out-of-bounds write checks that need no memory checker: every output of every
entry point is allocated between two 4 KiB guard bands filled with a sentinel byte,
the call runs on ragged shapes, and the bands must be untouched afterwards.  Inputs
must be unchanged too."""

import numpy as np
import pytest

from rotation_bit_quantization_b200 import workloads as wl
from tests import helpers as H

pytestmark = pytest.mark.gpu

PAD = 4096
SENTINEL = 0xA5


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


class Guarded:
    """A device tensor of `shape`/`dtype` with sentinel-filled bands on both sides; `shift`
    moves its start by that many bytes (to test outputs that meet only the documented
    minimum alignment)."""

    def __init__(self, shape, dtype, shift=0):
        torch = H.torch()
        nbytes = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        self.nbytes = nbytes
        self.lo = PAD + shift
        self.buf = torch.full((2 * PAD + nbytes + shift,), SENTINEL, dtype=torch.uint8, device="cuda")
        self.t = self.buf[self.lo:self.lo + nbytes].view(dtype).view(shape)

    def check(self, name):
        b = self.buf.cpu().numpy()
        assert np.all(b[:self.lo] == SENTINEL), f"{name}: write before the buffer"
        assert np.all(b[self.lo + self.nbytes:] == SENTINEL), f"{name}: write past the end"


def _snap(*ts):
    return [t.clone() for t in ts]


def _same(before, after):
    torch = H.torch()
    return all(torch.equal(a, b) for a, b in zip(before, after))


@pytest.mark.parametrize("m,r,rows", [(4096, 1, 3), (4096, 1, 449), (1024, 5, 5), (256, 1, 7), (64, 3, 9)])
def test_transform_and_inverse_stay_in_bounds(bq, m, r, rows):
    torch = H.torch()
    rng = np.random.default_rng(m + r + rows)
    theta = wl.uniform_angles(rng, m)
    O = None if r == 1 else H.dev_f32(wl.random_orthogonal(rng, r))
    layer = bq.Layer(H.dev_f32(theta), O)
    n = m * r
    x = H.dev_f32(rng.standard_normal((rows, n)).astype(np.float32))
    xb = x.to(torch.bfloat16)
    keep = _snap(x, xb)
    for dt in (torch.float32, torch.bfloat16):
        for src in (x, xb):
            y = Guarded((rows, n), dt)
            bq.bq_butterfly_fwd(layer, src, y.t)
            z = Guarded((rows, n), dt)
            bq.bq_butterfly_inv(layer, src, z.t)
            torch.cuda.synchronize()
            y.check("forward output")
            z.check("inverse output")
    assert _same(keep, (x, xb))


@pytest.mark.parametrize("m,r,rows,bits,group", [(4096, 1, 5, 4, 128), (4096, 1, 300, 2, 64), (1024, 5, 3, 4, 128),
                                                 (1024, 1, 7, 2, 32), (256, 1, 2, 4, 256)])
def test_quantize_and_pack_stay_in_bounds(bq, m, r, rows, bits, group):
    torch = H.torch()
    rng = np.random.default_rng(m + rows + bits)
    theta = wl.uniform_angles(rng, m)
    O = None if r == 1 else H.dev_f32(wl.random_orthogonal(rng, r))
    layer = bq.Layer(H.dev_f32(theta), O)
    n = m * r
    if n % group:
        pytest.skip("group does not divide n")
    x = H.dev_f32(rng.standard_normal((rows, n)).astype(np.float32)).to(torch.bfloat16)
    keep = _snap(x)
    fns = [bq.bq_transform_quantize] + ([bq.bq_weight_rotate_pack] if r == 1 else [])
    for fn in fns:
        c = Guarded((rows, n * bits // 8), torch.uint8)
        s = Guarded((rows, n // group), torch.int16)
        z = Guarded((rows, n // group), torch.int16)
        fn(layer, x, bits, group, c.t, s.t, z.t)
        torch.cuda.synchronize()
        c.check("codes")
        s.check("scales")
        z.check("zero points")
    assert _same(keep, (x,))


@pytest.mark.parametrize("m,layers,tokens", [(4096, 2, 37), (256, 3, 5), (4096, 1, 1)])
def test_backward_stays_in_bounds(bq, m, layers, tokens):
    torch = H.torch()
    rng = np.random.default_rng(m + layers + tokens)
    Ls = [bq.Layer(H.dev_f32(wl.uniform_angles(rng, m))) for _ in range(layers)]
    x = H.dev_f32(rng.standard_normal((layers, tokens, m)).astype(np.float32)).to(torch.bfloat16)
    dy = H.dev_f32(rng.standard_normal((layers, tokens, m)).astype(np.float32))
    keep = _snap(x, dy)
    L = m.bit_length() - 1
    y = Guarded((layers, tokens, m), torch.bfloat16)
    dx = Guarded((layers, tokens, m), torch.float32)
    dth = Guarded((layers, L * m // 2), torch.float32)
    ws = Guarded((bq.bq_butterfly_bwd_workspace_size(m, layers, tokens),), torch.uint8)
    bq.bq_butterfly_bwd(Ls, x, y.t, dy, dx.t, dth.t, ws.t)
    torch.cuda.synchronize()
    for g, nm in ((y, "Y"), (dx, "dX"), (dth, "dtheta"), (ws, "workspace")):
        g.check(nm)
    assert _same(keep, (x, dy))


def test_calibration_losses_stay_in_bounds(bq):
    torch = H.torch()
    rng = np.random.default_rng(5)
    rows, n, bits, group = 13, 1024, 4, 128
    y = H.dev_f32(rng.standard_normal((rows, n)).astype(np.float32))
    keep = _snap(y)
    kl = Guarded((rows, n // group), torch.float32)
    dy = Guarded((rows, n), torch.float32)
    loss = Guarded((1,), torch.float32)
    bq.bq_uniformity_loss(y, bits, group, 1e-4, kl.t, dy.t, loss.t)
    torch.cuda.synchronize()
    for g, nm in ((kl, "kl"), (dy, "dL/dY"), (loss, "loss")):
        g.check(nm)
    assert _same(keep, (y,))
    m, out, T = 256, 40, 24
    theta = H.dev_f32(wl.uniform_angles(rng, m))
    layer = bq.Layer(theta)
    w = H.dev_f32((rng.standard_normal((out, m)) * 0.02).astype(np.float32))
    x = H.dev_f32(rng.standard_normal((T, m)).astype(np.float32))
    keep = _snap(w, x, theta)
    dth = Guarded((8 * m // 2,), torch.float32)
    rl = Guarded((1,), torch.float32)
    ws = Guarded((bq.bq_reconstruction_workspace_size(m, out, T, 2, 64),), torch.uint8)
    bq.bq_reconstruction_loss(layer, w, x, 2, 64, dth.t, rl.t, ws.t)
    torch.cuda.synchronize()
    for g, nm in ((dth, "dtheta"), (rl, "loss"), (ws, "workspace")):
        g.check(nm)
    assert _same(keep, (w, x, theta))


@pytest.mark.parametrize("tokens,out,bits,split", [(100, 200, 2, False), (100, 200, 2, True), (7, 130, 4, True),
                                                   (300, 384, 4, False), (1, 1000, 2, True)])
def test_w2a16_stays_in_bounds(bq, tokens, out, bits, split):
    torch = H.torch()
    rng = np.random.default_rng(tokens + out)
    n, group = 1024, 128
    x = H.dev_f32(rng.standard_normal((tokens, n)).astype(np.float32)).to(torch.bfloat16)
    codes, s16, z16 = wl.packed_weights(rng, out, n, bits, group)
    c = torch.from_numpy(codes).cuda()
    s = torch.from_numpy(s16.view(np.int16)).cuda()
    z = torch.from_numpy(z16.view(np.int16)).cuda()
    keep = _snap(x, c, s, z)
    for dt in (torch.float32, torch.bfloat16):
        o = Guarded((tokens, out), dt)
        ws = None
        if split:
            ws = Guarded((max(256, bq.bq_w2a16_gemm_workspace_size(tokens, n, out)),), torch.uint8)
        st = Guarded((1,), torch.int32)
        st.t.zero_()
        bq.bq_w2a16_gemm(x, c, s, z, bits, group, o.t, workspace=None if ws is None else ws.t, status=st.t)
        torch.cuda.synchronize()
        o.check("output")
        st.check("status")
        assert int(st.t.item()) == 0
        if ws is not None:
            ws.check("workspace")
    assert _same(keep, (x, c, s, z))


def test_hadamard_preset_stays_in_bounds(bq):
    torch = H.torch()
    m = 1024
    L = 10
    table = Guarded((bq.load().bq_table_floats(m),), torch.float32)
    theta = Guarded((L, m // 2), torch.float32)
    k = torch.randint(0, 4, (L, m // 2), dtype=torch.uint8, device="cuda")
    import ctypes
    from rotation_bit_quantization_b200 import _lib
    st = bq.load().bq_precompute_hadamard(m, ctypes.c_void_p(k.data_ptr()), ctypes.c_void_p(table.t.data_ptr()),
                                          ctypes.c_void_p(theta.t.data_ptr()), None)
    assert st == _lib.BQ_OK
    torch.cuda.synchronize()
    table.check("table")
    theta.check("angles")


@pytest.mark.parametrize("rows,C", [(1, 64), (131, 320), (300, 4096)])
@pytest.mark.parametrize("shift", [0, 16])
def test_block_transform_stays_in_bounds(bq, rows, C, shift):
    """All block formats and both unquantized outputs on ragged rows, a last unit of one
    64-channel sub-tile (C = 320), and outputs shifted to the documented minimum alignment
    (codes 16 bytes, scales 2 bytes), which the kernel's wide stores must detect."""
    torch = H.torch()
    rng = np.random.default_rng(rows + C + shift)
    x = H.dev_bf16_bits(wl.bf16_bits_from_f32(rng.standard_normal((rows, C)).astype(np.float32)))
    keep = _snap(x)
    for fmt, G in (("mxfp4", 32), ("nvfp4", 16), ("int4", 32), ("none", 16), ("none", 32)):
        Tb = wl.block_transforms(C, G, 3)
        bt = bq.BlockTransform(H.dev_bf16_bits(Tb.reshape(-1, G)).view(Tb.shape))
        st = Guarded((1,), torch.int32)
        st.t.zero_()
        if fmt == "none":
            for dt in (torch.float32, torch.bfloat16):
                y = Guarded((rows, C), dt, shift)
                bq.bq_block_transform_quantize(bt, x, "none", y=y.t, status=st.t)
                torch.cuda.synchronize()
                y.check(f"block output {dt}")
        else:
            c = Guarded((rows, C // 2), torch.uint8, shift)
            sc = Guarded((rows, C // G), torch.int16 if fmt == "int4" else torch.uint8, 2 if shift else 0)
            bq.bq_block_transform_quantize(bt, x, fmt, c.t, sc.t, gscale=0.5, status=st.t)
            torch.cuda.synchronize()
            c.check(f"{fmt} codes")
            sc.check(f"{fmt} scales")
        st.check("status")
        assert int(st.t.item()) == 0
    assert _same(keep, (x,))
