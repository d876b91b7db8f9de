"""bq_butterfly_bwd_noalloc: the backward for callers that cannot allocate device
memory (another framework owns the allocator, a real-time loop must not block in
it, or the device memory is all reserved by a pool).  Its scratch is a fixed
array inside the library, so its results must match the workspace version.

Collected last on purpose: if it fails, a run that stops at the first failure
has already run every other test.  Self-contained, so it also passes alone in a
fresh process.
"""

import ctypes

import numpy as np
import pytest

from oracle import butterfly as ob
from rotation_bit_quantization_b200 import _lib
from rotation_bit_quantization_b200 import workloads as wl


def test_rejects_more_than_fits_without_touching_the_gpu():
    # 86 layers of width 4096 need 86 * 24576 * 4 bytes of partial sums even with one
    # token chunk per layer: more than the 8 MiB scratch.  Validation fails first.
    from rotation_bit_quantization_b200 import build
    build.build()
    lib = _lib.load()
    fake = 0x10000
    layers = (_lib.BQLayer * 86)(*[_lib.BQLayer(4096, 4096, 1, fake, None) for _ in range(86)])
    st = lib.bq_butterfly_bwd_noalloc(layers, 86, fake, 0, fake, 0, fake, fake, fake, 10, None)
    assert st == _lib.BQ_ERR_WORKSPACE
    layers85 = (_lib.BQLayer * 85)(*[_lib.BQLayer(4096, 4096, 1, fake, None) for _ in range(85)])
    assert lib.bq_butterfly_bwd_noalloc(layers85, 85, None, 0, fake, 0, fake, fake, fake, 10, None) == \
        _lib.BQ_ERR_INVALID_ARG


@pytest.mark.gpu
def test_noalloc_matches_workspace_backward_twice():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import rotation_bit_quantization_b200 as bq
    from rotation_bit_quantization_b200 import build
    build.build()
    bq.load()

    m, nl, rows = 4096, 3, 257
    rng = np.random.default_rng(2024)
    thetas = [wl.uniform_angles(rng, m) for _ in range(nl)]
    x = (rng.standard_t(3, (nl, rows, m)) * 0.5).astype(np.float32)
    dy = rng.standard_normal((nl, rows, m)).astype(np.float32)
    layers = [bq.Layer(torch.from_numpy(t).cuda()) for t in thetas]
    xd, dyd = torch.from_numpy(x).cuda(), torch.from_numpy(dy).cuda()

    def outputs():
        return (torch.empty((nl, rows, m), dtype=torch.float32, device="cuda"),
                torch.empty((nl, rows, m), dtype=torch.float32, device="cuda"),
                torch.empty((nl, 12 * m // 2), dtype=torch.float32, device="cuda"))

    y0, dx0, th0 = outputs()
    ws = torch.empty(bq.bq_butterfly_bwd_workspace_size(m, nl, rows), dtype=torch.uint8, device="cuda")
    bq.bq_butterfly_bwd(layers, xd, y0, dyd, dx0, th0, ws)
    torch.cuda.synchronize()

    results = []
    for _ in range(2):
        y1, dx1, th1 = outputs()
        bq.bq_butterfly_bwd_noalloc(layers, xd, y1, dyd, dx1, th1)
        torch.cuda.synchronize()
        assert torch.equal(y1, y0) and torch.equal(dx1, dx0)
        results.append(th1.cpu().numpy())
    assert np.array_equal(results[0], results[1])          # deterministic across calls
    ref = th0.cpu().numpy()
    for l in range(nl):
        A = ob.backward_abs_scale(thetas[l], x[l].astype(np.float64), dy[l].astype(np.float64)).ravel()
        bound = 2e-4 * A + 1e-6 * A.max()
        assert np.all(np.abs(results[0][l] - ref[l]) <= bound)


@pytest.mark.gpu
@pytest.mark.parametrize("nl,rows", [(40, 64), (128, 24)])
def test_noalloc_generic_width_with_fewer_chunks(nl, rows):
    """Width 2048 (the general backward kernel) with many layers: the default chunk count
    does not fit the fixed scratch, so the allocation-free call sums dtheta over fewer,
    larger token chunks (40 layers: 4 chunks instead of 15; 128 layers: 1 instead of 5).
    y and dx stay bitwise equal to the workspace version; dtheta stays within the
    oracle-scaled bound and is reproducible across calls."""
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import rotation_bit_quantization_b200 as bq
    from rotation_bit_quantization_b200 import build
    build.build()
    bq.load()

    m = 2048
    rng = np.random.default_rng(nl * 1000 + rows)
    thetas = [wl.uniform_angles(rng, m) for _ in range(nl)]
    x = (rng.standard_t(3, (nl, rows, m)) * 0.5).astype(np.float32)
    dy = rng.standard_normal((nl, rows, m)).astype(np.float32)
    layers = [bq.Layer(torch.from_numpy(t).cuda()) for t in thetas]
    xd, dyd = torch.from_numpy(x).cuda(), torch.from_numpy(dy).cuda()
    L = 11

    def outputs():
        return (torch.empty((nl, rows, m), dtype=torch.float32, device="cuda"),
                torch.empty((nl, rows, m), dtype=torch.float32, device="cuda"),
                torch.empty((nl, L * m // 2), dtype=torch.float32, device="cuda"))

    assert bq.bq_butterfly_bwd_workspace_size(m, nl, rows) > (8 << 20)   # the default plan does not fit
    y0, dx0, th0 = outputs()
    ws = torch.empty(bq.bq_butterfly_bwd_workspace_size(m, nl, rows), dtype=torch.uint8, device="cuda")
    bq.bq_butterfly_bwd(layers, xd, y0, dyd, dx0, th0, ws)
    torch.cuda.synchronize()
    results = []
    for _ in range(2):
        y1, dx1, th1 = outputs()
        bq.bq_butterfly_bwd_noalloc(layers, xd, y1, dyd, dx1, th1)
        torch.cuda.synchronize()
        assert torch.equal(y1, y0) and torch.equal(dx1, dx0)
        results.append(th1.cpu().numpy())
    assert np.array_equal(results[0], results[1])
    ref = th0.cpu().numpy()
    for l in (0, nl // 2, nl - 1):
        A = ob.backward_abs_scale(thetas[l], x[l].astype(np.float64), dy[l].astype(np.float64)).ravel()
        bound = 2e-4 * A + 1e-6 * A.max()
        assert np.all(np.abs(results[0][l] - ref[l]) <= bound)
        _, _, dth = ob.backward(thetas[l], x[l].astype(np.float64), dy[l].astype(np.float64))
        assert np.all(np.abs(results[0][l] - dth.ravel()) <= bound)
