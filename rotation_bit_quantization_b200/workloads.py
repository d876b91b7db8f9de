"""Seeded synthetic inputs for the butterfly transform + quantize path.

This module only draws random numbers and rounds them to the storage dtypes
(float32 -> bfloat16 round-to-nearest-even).  It holds none of the method's
arithmetic, so the CUDA path and the float64 oracle can both consume it.

The workloads stand in for LLaMA-2-7B / 13B layers (hidden sizes 4096 and
5120; explainer article, section "butterfly"), whose weights and calibration
data are not available here.  Outlier channels follow the layer-dependent tail
patterns the explainer article describes (section "why fixed rotation fails":
attention layers have a positive tail, early MLP layers a negative tail).

Seeds: ``numpy.random.default_rng([cfg, stream])`` with stream 0 = angles,
1 = X, 2 = W, 3 = O, 4 = dY, 5 = outlier channels; the tiny case draws its
angles from ``default_rng(0)``.  The backward workload draws per layer from
``[5, layer, stream]`` (host) or from a seeded ``torch.Generator`` (device).
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

TWO_PI = 2.0 * np.pi


# ----------------------------------------------------------------------------
# storage-dtype helpers (input preparation, not part of the method)
# ----------------------------------------------------------------------------

def bf16_bits_from_f32(a) -> np.ndarray:
    """float32 -> bfloat16 bit patterns (uint16), round to nearest even; NaN stays NaN."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    rounding = ((u >> 16) & 1) + 0x7FFF
    out = ((u + rounding) >> 16).astype(np.uint16)
    nan = np.isnan(a)
    if nan.any():
        out[nan] = 0x7FC0
    return out


def f32_from_bf16_bits(b) -> np.ndarray:
    """bfloat16 bit patterns -> float32 (exact widening)."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def uniform_angles(rng, m: int) -> np.ndarray:
    """Angles ~ U[-pi, pi) drawn in float64 and stored as float32, shape (log2 m, m/2)."""
    L = m.bit_length() - 1
    t = rng.uniform(-np.pi, np.pi, size=(L, m // 2))
    return t.astype(np.float32)


def random_orthogonal(rng, r: int) -> np.ndarray:
    """Dense r x r orthogonal matrix: QR of a seeded N(0,1) matrix, column signs so diag(R) > 0.

    Returned as float32 (the shared input); its orthogonality holds to float32
    rounding, which both sides see identically.
    """
    a = rng.standard_normal((r, r))
    q, rr = np.linalg.qr(a)
    q = q * np.sign(np.diag(rr))[None, :]
    return q.astype(np.float32)


def student_t(rng, nu: float, shape) -> np.ndarray:
    return rng.standard_t(nu, size=shape)


# ----------------------------------------------------------------------------
# workloads
# ----------------------------------------------------------------------------

@dataclass
class Workload:
    """One seeded problem instance.  Arrays are host numpy arrays.

    theta: float32 (log2 m, m/2); O: float32 (r, r) or None; x: float32 or
    bf16 bits (rows, n); w likewise; dy: float32; bits/group: quantizer
    settings of the fused call (None when the workload has no quantizer).
    """
    name: str
    m: int
    r: int
    theta: np.ndarray
    O: np.ndarray | None = None
    x: np.ndarray | None = None
    x_dtype: str = "f32"          # "f32" or "bf16" (then x holds uint16 bit patterns)
    w: np.ndarray | None = None
    w_dtype: str = "f32"
    dy: np.ndarray | None = None
    bits: int | None = None
    group: int | None = None
    meta: dict = field(default_factory=dict)

    @property
    def n(self) -> int:
        return self.m * self.r


def _outlier_channels(rng, n, k):
    return np.sort(rng.choice(n, size=k, replace=False))


def tiny(rows_x: int = 64, rows_w: int = 128) -> Workload:
    """n = 256: 8 stages, 1024 angles U[-pi,pi) (seed 0); X fp32 N(0,1) with 3 channels x20;
    W fp32 N(0, 0.02); weight side 2-bit RTN in groups of 64."""
    n = 256
    theta = uniform_angles(np.random.default_rng(0), n)
    rx = np.random.default_rng([1, 1])
    x = rx.standard_normal((rows_x, n))
    ch = _outlier_channels(np.random.default_rng([1, 5]), n, 3)
    x[:, ch] *= 20.0
    w = np.random.default_rng([1, 2]).normal(0.0, 0.02, (rows_w, n))
    return Workload("tiny n=256", n, 1, theta, x=x.astype(np.float32), x_dtype="f32",
                    w=w.astype(np.float32), w_dtype="f32", bits=2, group=64,
                    meta={"outlier_channels": ch.tolist()})


def act_4096(rows: int = 2048, seed_offset: int = 0) -> Workload:
    """LLaMA-2-7B activation shape: n = 4096, X rows x 4096 bf16 = 0.5 * t(nu=3) with 8 fixed
    channels set to +50*|value| (positive tail); fused Qx + INT4 RTN in groups of 128."""
    n = 4096
    theta = uniform_angles(np.random.default_rng([2, 0]), n)
    x = 0.5 * student_t(np.random.default_rng([2, 1, seed_offset]), 3.0, (rows, n))
    ch = _outlier_channels(np.random.default_rng([2, 5]), n, 8)
    x[:, ch] = 50.0 * np.abs(x[:, ch])
    return Workload(f"act n=4096 rows={rows}", n, 1, theta, x=bf16_bits_from_f32(x.astype(np.float32)),
                    x_dtype="bf16", bits=4, group=128, meta={"outlier_channels": ch.tolist()})


def weight_4096(rows: int = 11008) -> Workload:
    """W2A16 weight side: W rows x 4096 bf16 N(0, 0.02) with round(1% of 4096) = 41 columns x10;
    W <- W Q^T, then 2-bit RTN in groups of 128 along the input dimension."""
    n = 4096
    theta = uniform_angles(np.random.default_rng([3, 0]), n)
    w = np.random.default_rng([3, 2]).normal(0.0, 0.02, (rows, n))
    ch = _outlier_channels(np.random.default_rng([3, 5]), n, 41)
    w[:, ch] *= 10.0
    return Workload(f"weight n=4096 rows={rows}", n, 1, theta, w=bf16_bits_from_f32(w.astype(np.float32)),
                    w_dtype="bf16", bits=2, group=128, meta={"outlier_channels": ch.tolist()})


def act_5120(rows: int = 8192) -> Workload:
    """LLaMA-2-13B shape: n = 5120, Q = B_1024 (x) O_5; X rows x 5120 bf16 = t(nu=3) with 10
    channels set to -50*|value| (negative tail); fused transform + INT4 RTN in groups of 128."""
    m, r = 1024, 5
    theta = uniform_angles(np.random.default_rng([4, 0]), m)
    O = random_orthogonal(np.random.default_rng([4, 3]), r)
    n = m * r
    x = student_t(np.random.default_rng([4, 1]), 3.0, (rows, n))
    ch = _outlier_channels(np.random.default_rng([4, 5]), n, 10)
    x[:, ch] = -50.0 * np.abs(x[:, ch])
    return Workload(f"act n=5120 rows={rows}", m, r, theta, O=O, x=bf16_bits_from_f32(x.astype(np.float32)),
                    x_dtype="bf16", bits=4, group=128, meta={"outlier_channels": ch.tolist()})


def backward_layer_host(layer: int, tokens: int, m: int = 4096) -> Workload:
    """One layer of the calibration-backward workload, drawn on the host (small token counts):
    X tokens x m bf16 t(nu=3), dY N(0,1) fp32, angles U[-pi,pi) of that layer."""
    theta = uniform_angles(np.random.default_rng([5, layer, 0]), m)
    x = student_t(np.random.default_rng([5, layer, 1]), 3.0, (tokens, m))
    dy = np.random.default_rng([5, layer, 4]).standard_normal((tokens, m))
    return Workload(f"bwd layer {layer} tokens={tokens}", m, 1, theta,
                    x=bf16_bits_from_f32(x.astype(np.float32)), x_dtype="bf16",
                    dy=dy.astype(np.float32))


def _layer_ids(layers):
    return list(range(layers)) if isinstance(layers, (int, np.integer)) else [int(l) for l in layers]


def backward_angles(layers, m: int = 4096) -> np.ndarray:
    """Per-layer angles of the backward workload, float32 (len, log2 m, m/2), for layers
    0..layers-1 (an int) or the given layer indices; layer l's angles depend on l only."""
    return np.stack([uniform_angles(np.random.default_rng([5, l, 0]), m) for l in _layer_ids(layers)])


def shard_layers(num_layers: int, world: int, rank: int):
    """Layer indices of one rank when the backward's independent layers are split across
    ranks: rank r takes layers r, r + world, r + 2 world, ..."""
    if world <= 0 or not (0 <= rank < world) or num_layers < 0:
        raise ValueError("bad world/rank/layers")
    return list(range(rank, num_layers, world))


def backward_inputs_device(layers, tokens: int, m: int, device, seed: int = 5):
    """Device-resident X (len, tokens, m) bf16 and dY (len, tokens, m) fp32 for layers
    0..layers-1 (an int) or the given layer indices, drawn with a seeded torch.Generator
    per layer (layer l's draws depend on seed and l only, so a rank holding a subset of
    the layers draws exactly those layers of the full workload); t(nu=3) =
    z / sqrt(chi2_3 / 3) built from normal draws.

    Used where host generation of ~50 GB is impractical; callers copy the layers
    they check back to the host.
    """
    import torch

    ids = _layer_ids(layers)
    gen = torch.Generator(device=device)
    x = torch.empty((len(ids), tokens, m), dtype=torch.bfloat16, device=device)
    dy = torch.empty((len(ids), tokens, m), dtype=torch.float32, device=device)
    for k, l in enumerate(ids):
        gen.manual_seed(seed * 1_000_003 + l)
        z = torch.randn((tokens, m), generator=gen, device=device)
        c = torch.randn((3, tokens, m), generator=gen, device=device).square_().sum(0).div_(3.0).sqrt_()
        x[k].copy_(z.div_(c))
        del z, c
        dy[k].normal_(generator=gen)
    return x, dy


def shard_rows(total_rows: int, world: int, rank: int):
    """Contiguous row range [start, stop) of one rank when rows are split across ranks."""
    if world <= 0 or not (0 <= rank < world):
        raise ValueError("bad world/rank")
    base, extra = divmod(total_rows, world)
    start = rank * base + min(rank, extra)
    stop = start + base + (1 if rank < extra else 0)
    return start, stop


def packed_weights(rng, out_features: int, n: int, bits: int, group: int):
    """Random packed low-bit weights in the layout the weight quantizer writes: uniformly random
    code bytes (so every code is uniform over the 2^bits levels), fp16 scales log-uniform in
    [2^-9, 2^-5] (the step sizes of N(0, 0.02) rows spread over 3 to 15 levels) and zero points
    uniform over the levels.  Returns (codes uint8 [out][n*bits/8], scale16, zero16 uint16 bits)."""
    codes = rng.integers(0, 256, size=(out_features, n * bits // 8), dtype=np.uint8)
    g = n // group
    scale16 = (2.0 ** rng.uniform(-9.0, -5.0, size=(out_features, g))).astype(np.float16).view(np.uint16)
    zero16 = rng.integers(0, 2 ** bits, size=(out_features, g)).astype(np.float16).view(np.uint16)
    return codes, scale16, zero16


def w2a16_4096(tokens: int = 2048, out_features: int = 11008, seed: int = 6):
    """W2A16 layer of the LLaMA-2-7B MLP shape: rotated activations tokens x 4096 bf16
    (0.5 * t(nu=3), the act workload's distribution) and INT2 g128 weights of out_features rows.
    Returns (x bf16 bits, codes, scale16, zero16, bits, group)."""
    rng = np.random.default_rng([seed, 1])
    x = bf16_bits_from_f32((0.5 * student_t(rng, 3.0, (tokens, 4096))).astype(np.float32))
    codes, s16, z16 = packed_weights(np.random.default_rng([seed, 2]), out_features, 4096, 2, 128)
    return x, codes, s16, z16, 2, 128


def block_transforms(C: int, G: int, seed: int = 7) -> np.ndarray:
    """Seeded per-block G x G transforms, bf16 bits (C/G, G, G): identity plus N(0, 0.3^2/G)
    entries (well conditioned, not orthogonal), standing in for transforms built offline
    from calibration statistics."""
    rng = np.random.default_rng([7, seed, C, G])
    T = np.eye(G)[None] + 0.3 * rng.standard_normal((C // G, G, G)) / np.sqrt(G)
    return bf16_bits_from_f32(T.astype(np.float32))
