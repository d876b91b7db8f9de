"""ctypes binding of libbq.so: argument marshalling only.

Every function here has the name of the C entry point it calls (see
include/bq.h).  Tensors are torch CUDA tensors; their device pointers and the
current CUDA stream are passed through unchanged.  Nothing is computed on the
host: if libbq.so is missing or a call fails, an exception is raised (there is
no fallback path).
"""

from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libbq.so")

BQ_OK, BQ_ERR_INVALID_ARG, BQ_ERR_UNSUPPORTED, BQ_ERR_WORKSPACE, BQ_ERR_CUDA = range(5)
BQ_F32, BQ_BF16 = 0, 1
BQ_BLOCK_NONE, BQ_BLOCK_MXFP4, BQ_BLOCK_NVFP4, BQ_BLOCK_INT4 = range(4)
BLOCK_FORMATS = {"none": BQ_BLOCK_NONE, "mxfp4": BQ_BLOCK_MXFP4, "nvfp4": BQ_BLOCK_NVFP4, "int4": BQ_BLOCK_INT4}

EXPORTED = (
    "bq_table_floats",
    "bq_precompute_cs",
    "bq_precompute_hadamard",
    "bq_butterfly_fwd",
    "bq_butterfly_inv",
    "bq_butterfly_bwd_workspace_size",
    "bq_butterfly_bwd",
    "bq_butterfly_bwd_noalloc",
    "bq_transform_quantize",
    "bq_weight_rotate_pack",
    "bq_uniformity_loss",
    "bq_angle_sgd",
    "bq_reconstruction_workspace_size",
    "bq_reconstruction_loss",
    "bq_w2a16_gemm",
    "bq_w2a16_gemm_workspace_size",
    "bq_w2a16_linear_workspace_size",
    "bq_w2a16_linear",
    "bq_block_table_bytes",
    "bq_block_prepare",
    "bq_block_transform_quantize",
    "bq_status_string",
    "bq_cuda_last_error",
    "bq_wait_faults",
    "bq_cuda_error_string",
)


class BQLayer(ctypes.Structure):
    _fields_ = [("n", ctypes.c_int32), ("m", ctypes.c_int32), ("r", ctypes.c_int32),
                ("table", ctypes.c_void_p), ("O", ctypes.c_void_p)]


class BQError(RuntimeError):
    def __init__(self, name: str, status: int, text: str):
        super().__init__(f"{name} failed: status {status} ({text})")
        self.status = status


_lib = None


def load(path: str | None = None):
    """Load libbq.so (once).  Raises if the library has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    path = path or LIB_PATH
    if not os.path.exists(path):
        raise ImportError(f"libbq.so not found at {path}; build it with "
                          "`python -m rotation_bit_quantization_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    lp = ctypes.POINTER(BQLayer)
    sig = {
        "bq_table_floats": (sz, [i32]),
        "bq_precompute_cs": (i32, [vp, i32, vp, vp]),
        "bq_precompute_hadamard": (i32, [i32, vp, vp, vp, vp]),
        "bq_butterfly_fwd": (i32, [lp, vp, i32, vp, i32, i64, vp]),
        "bq_butterfly_inv": (i32, [lp, vp, i32, vp, i32, i64, vp]),
        "bq_butterfly_bwd_workspace_size": (sz, [i32, i32, i64]),
        "bq_butterfly_bwd": (i32, [lp, i32, vp, i32, vp, i32, vp, vp, vp, i64, vp, sz, vp]),
        "bq_butterfly_bwd_noalloc": (i32, [lp, i32, vp, i32, vp, i32, vp, vp, vp, i64, vp]),
        "bq_transform_quantize": (i32, [lp, vp, i32, i64, i32, i32, vp, vp, vp, vp]),
        "bq_weight_rotate_pack": (i32, [lp, vp, i32, i64, i32, i32, vp, vp, vp, vp]),
        "bq_uniformity_loss": (i32, [vp, i64, i32, i32, i32, ctypes.c_float, vp, vp, vp, vp]),
        "bq_angle_sgd": (i32, [vp, vp, i64, ctypes.c_float, vp]),
        "bq_reconstruction_workspace_size": (sz, [i32, i64, i64, i32, i32]),
        "bq_reconstruction_loss": (i32, [lp, vp, i64, vp, i64, i32, i32, vp, vp, vp, sz, vp]),
        "bq_w2a16_gemm": (i32, [vp, i64, i32, vp, vp, vp, i64, i32, i32, vp, i32, vp, sz, vp, vp]),
        "bq_w2a16_gemm_workspace_size": (sz, [i64, i32, i64]),
        "bq_w2a16_linear_workspace_size": (sz, [i32, i64, i64]),
        "bq_w2a16_linear": (i32, [lp, vp, i32, i64, vp, vp, vp, i64, i32, i32, vp, i32, vp, sz, vp, vp]),
        "bq_block_table_bytes": (sz, [i32, i32]),
        "bq_block_prepare": (i32, [vp, i32, i32, vp, vp]),
        "bq_block_transform_quantize": (i32, [vp, i32, i32, vp, i64, i32, ctypes.c_float, vp, i32, vp, vp, vp, vp]),
        "bq_status_string": (ctypes.c_char_p, [i32]),
        "bq_cuda_last_error": (i32, []),
        "bq_wait_faults": (i32, [ctypes.POINTER(i32), i32, vp]),
        "bq_cuda_error_string": (ctypes.c_char_p, [i32]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().bq_status_string(status).decode()


def _check(name: str, status: int):
    if status != BQ_OK:
        text = status_string(status)
        if status == BQ_ERR_CUDA:  # which CUDA call failed, from the library's own runtime
            code = int(load().bq_cuda_last_error())
            if code:
                text += f"; CUDA error {code}: {load().bq_cuda_error_string(code).decode()}"
        raise BQError(name, status, text)


# ----------------------------------------------------------------------------- marshalling helpers

def _torch():
    import torch
    return torch


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.float32:
        return BQ_F32
    if t.dtype == torch.bfloat16:
        return BQ_BF16
    raise TypeError(f"unsupported dtype {t.dtype}: use float32 or bfloat16")


def _stream(stream=None):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dev(t, name):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


class Layer:
    """One layer's prepared transform: holds the device table (and O_r) alive.

    theta: float32 CUDA tensor of shape (log2 m, m/2); O: None or float32 CUDA
    tensor (r, r).  The table is filled by bq_precompute_cs on the current stream.
    """

    def __init__(self, theta, O=None, stream=None):
        torch = _torch()
        lib = load()
        _dev(theta, "theta")
        if theta.dtype != torch.float32 or theta.dim() != 2:
            raise ValueError("theta must be float32 of shape (log2 m, m/2)")
        self.m = int(theta.shape[1]) * 2
        self.r = 1 if O is None else int(O.shape[0])
        self.n = self.m * self.r
        floats = lib.bq_table_floats(self.m)
        if floats == 0:
            raise ValueError(f"unsupported butterfly width m={self.m}")
        self.theta = theta
        self.table = torch.empty(floats, dtype=torch.float32, device=theta.device)
        self.O = None if O is None else _dev(O, "O")
        bq_precompute_cs(theta, self.m, self.table, stream)
        self.c = BQLayer(self.n, self.m, self.r, self.table.data_ptr(),
                         None if self.O is None else self.O.data_ptr())

    @classmethod
    def hadamard(cls, m: int, quadrant=None, O=None, device="cuda", stream=None):
        """The Hadamard preset of width m (bq_precompute_hadamard): every angle pi/4, or
        pi/4 + k pi/2 with k from `quadrant` (uint8 CUDA tensor of shape (log2 m, m/2))."""
        torch = _torch()
        lib = load()
        L = m.bit_length() - 1
        if m < 2 or (1 << L) != m or lib.bq_table_floats(m) == 0:
            raise ValueError(f"unsupported butterfly width m={m}")
        if quadrant is not None:
            _dev(quadrant, "quadrant")
            if quadrant.dtype != torch.uint8 or quadrant.numel() != L * (m // 2):
                raise ValueError("quadrant must be uint8 with log2(m) * m/2 elements")
        self = cls.__new__(cls)
        self.m, self.r = m, 1 if O is None else int(O.shape[0])
        self.n = self.m * self.r
        self.theta = torch.empty((L, m // 2), dtype=torch.float32, device=device)
        self.table = torch.empty(lib.bq_table_floats(m), dtype=torch.float32, device=device)
        self.O = None if O is None else _dev(O, "O")
        _check("bq_precompute_hadamard", lib.bq_precompute_hadamard(m, _ptr(quadrant), _ptr(self.table),
                                                                    _ptr(self.theta), _stream(stream)))
        self.c = BQLayer(self.n, self.m, self.r, self.table.data_ptr(),
                         None if self.O is None else self.O.data_ptr())
        return self

    @property
    def fast_form(self) -> bool:
        """Whether the scaled two-FMA rotation form is in range for these angles (header flag)."""
        return bool(self.table[0].item() == 1.0)

    @property
    def fast_form_inverse(self) -> bool:
        """Whether the scaled form of the inverse is in range for these angles (header flag)."""
        return bool(self.table[3].item() == 1.0)


# ----------------------------------------------------------------------------- entry points

def bq_precompute_cs(theta, m: int, table, stream=None):
    _check("bq_precompute_cs", load().bq_precompute_cs(_ptr(theta), m, _ptr(table), _stream(stream)))


def bq_butterfly_fwd(layer: Layer, x, y, stream=None):
    _dev(x, "x"); _dev(y, "y")
    rows = x.numel() // layer.n
    _check("bq_butterfly_fwd", load().bq_butterfly_fwd(ctypes.byref(layer.c), _ptr(x), _dtype_code(x), _ptr(y),
                                                        _dtype_code(y), rows, _stream(stream)))
    return y


def bq_butterfly_inv(layer: Layer, y, x, stream=None):
    _dev(x, "x"); _dev(y, "y")
    rows = y.numel() // layer.n
    _check("bq_butterfly_inv", load().bq_butterfly_inv(ctypes.byref(layer.c), _ptr(y), _dtype_code(y), _ptr(x),
                                                        _dtype_code(x), rows, _stream(stream)))
    return x


def bq_butterfly_bwd_workspace_size(m: int, num_layers: int, rows_per_layer: int) -> int:
    return int(load().bq_butterfly_bwd_workspace_size(m, num_layers, rows_per_layer))


def bq_butterfly_bwd(layers, x, y, dy, dx, dtheta, workspace, stream=None):
    """x, y, dy, dx: (layers, rows, m); dtheta: (layers, log2 m * m/2) float32."""
    arr = (BQLayer * len(layers))(*[l.c for l in layers])
    for t, nm in ((x, "x"), (y, "y"), (dy, "dy"), (dx, "dx"), (dtheta, "dtheta"), (workspace, "workspace")):
        _dev(t, nm)
    rows = x.numel() // (len(layers) * layers[0].n)
    _check("bq_butterfly_bwd", load().bq_butterfly_bwd(arr, len(layers), _ptr(x), _dtype_code(x), _ptr(y),
                                                        _dtype_code(y), _ptr(dy), _ptr(dx), _ptr(dtheta), rows,
                                                        _ptr(workspace), workspace.numel() * workspace.element_size(),
                                                        _stream(stream)))


def bq_butterfly_bwd_noalloc(layers, x, y, dy, dx, dtheta, stream=None):
    """Like bq_butterfly_bwd, with the library's fixed device scratch instead of a workspace."""
    arr = (BQLayer * len(layers))(*[l.c for l in layers])
    for t, nm in ((x, "x"), (y, "y"), (dy, "dy"), (dx, "dx"), (dtheta, "dtheta")):
        _dev(t, nm)
    rows = x.numel() // (len(layers) * layers[0].n)
    _check("bq_butterfly_bwd_noalloc",
           load().bq_butterfly_bwd_noalloc(arr, len(layers), _ptr(x), _dtype_code(x), _ptr(y), _dtype_code(y),
                                           _ptr(dy), _ptr(dx), _ptr(dtheta), rows, _stream(stream)))


def _quant(name, layer, x, bits, group, codes, scale, zero, stream):
    _dev(x, "x"); _dev(codes, "codes"); _dev(scale, "scale"); _dev(zero, "zero")
    rows = x.numel() // layer.n
    fn = getattr(load(), name)
    _check(name, fn(ctypes.byref(layer.c), _ptr(x), _dtype_code(x), rows, bits, group, _ptr(codes), _ptr(scale),
                    _ptr(zero), _stream(stream)))
    return codes, scale, zero


def quant_outputs(rows: int, n: int, bits: int, group: int, device):
    """Allocate (codes uint8 [rows][n*bits/8], scale int16 [rows][n/group], zero int16 [rows][n/group])."""
    torch = _torch()
    codes = torch.empty((rows, n * bits // 8), dtype=torch.uint8, device=device)
    scale = torch.empty((rows, n // group), dtype=torch.int16, device=device)
    zero = torch.empty((rows, n // group), dtype=torch.int16, device=device)
    return codes, scale, zero


def bq_transform_quantize(layer: Layer, x, bits: int, group: int, codes, scale, zero, stream=None):
    return _quant("bq_transform_quantize", layer, x, bits, group, codes, scale, zero, stream)


def bq_weight_rotate_pack(layer: Layer, w, bits: int, group: int, codes, scale, zero, stream=None):
    return _quant("bq_weight_rotate_pack", layer, w, bits, group, codes, scale, zero, stream)


def bq_uniformity_loss(y, bits: int, group: int, eps: float, kl_group, dy=None, loss=None, stream=None):
    """y: float32 (rows, n); kl_group: float32 (rows, n/group); dy: float32 like y or None;
    loss: float32 tensor of one element or None."""
    _dev(y, "y"); _dev(kl_group, "kl_group")
    if dy is not None:
        _dev(dy, "dy")
    rows, n = y.shape
    _check("bq_uniformity_loss", load().bq_uniformity_loss(_ptr(y), rows, n, bits, group, float(eps), _ptr(kl_group),
                                                            _ptr(dy), _ptr(loss), _stream(stream)))
    return kl_group, dy, loss


def bq_wait_faults(clear: bool = False, stream=None) -> int:
    """The device's wait-fault word (0: no bounded wait of the m = 4096 kernels gave up);
    synchronises the stream, and resets the word when `clear`."""
    v = ctypes.c_int32(0)
    _check("bq_wait_faults", load().bq_wait_faults(ctypes.byref(v), 1 if clear else 0, _stream(stream)))
    return int(v.value)


def bq_angle_sgd(theta, dtheta, lr: float, stream=None):
    _dev(theta, "theta"); _dev(dtheta, "dtheta")
    _check("bq_angle_sgd", load().bq_angle_sgd(_ptr(theta), _ptr(dtheta), theta.numel(), float(lr), _stream(stream)))
    return theta


def bq_reconstruction_workspace_size(n: int, out_features: int, tokens: int, bits: int, group: int) -> int:
    return int(load().bq_reconstruction_workspace_size(n, out_features, tokens, bits, group))


def bq_reconstruction_loss(layer: Layer, w, x, bits: int, group: int, dtheta, loss, workspace, stream=None):
    """w: float32 (out_features, n); x: float32 (tokens, n); dtheta: float32 with log2(n)*n/2
    elements; loss: float32 tensor of one element; workspace: uint8 CUDA tensor."""
    for t, nm in ((w, "w"), (x, "x"), (dtheta, "dtheta"), (loss, "loss"), (workspace, "workspace")):
        _dev(t, nm)
    _check("bq_reconstruction_loss",
           load().bq_reconstruction_loss(ctypes.byref(layer.c), _ptr(w), w.shape[0], _ptr(x), x.shape[0], bits, group,
                                         _ptr(dtheta), _ptr(loss), _ptr(workspace),
                                         workspace.numel() * workspace.element_size(), _stream(stream)))
    return dtheta, loss


def bq_w2a16_gemm_workspace_size(tokens: int, n: int, out_features: int) -> int:
    return int(load().bq_w2a16_gemm_workspace_size(tokens, n, out_features))


def bq_w2a16_gemm(x, codes, scale, zero, bits: int, group: int, out, workspace=None, status=None, stream=None):
    """x: bfloat16 (tokens, n) rotated activations; codes/scale/zero: the packed weights of
    bq_weight_rotate_pack for (out_features, n); out: float32 or bfloat16 (tokens, out_features);
    workspace: None or a uint8 CUDA tensor of bq_w2a16_gemm_workspace_size bytes (split K);
    status: None or an int32 CUDA tensor of one element (zeroed by the caller)."""
    for t, nm in ((x, "x"), (codes, "codes"), (scale, "scale"), (zero, "zero"), (out, "out")):
        _dev(t, nm)
    for t, nm in ((workspace, "workspace"), (status, "status")):
        if t is not None:
            _dev(t, nm)
    tokens, n = x.shape
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("bq_w2a16_gemm",
           load().bq_w2a16_gemm(_ptr(x), tokens, n, _ptr(codes), _ptr(scale), _ptr(zero), codes.shape[0], bits,
                                group, _ptr(out), _dtype_code(out), _ptr(workspace), ws_bytes, _ptr(status),
                                _stream(stream)))
    return out


def bq_w2a16_linear_workspace_size(n: int, tokens: int, out_features: int) -> int:
    return int(load().bq_w2a16_linear_workspace_size(n, tokens, out_features))


def bq_w2a16_linear(layer: Layer, x, codes, scale, zero, bits: int, group: int, out, workspace, status=None,
                    stream=None):
    """Q x to bfloat16 in the workspace, then bq_w2a16_gemm; x: float32 or bfloat16 (tokens, n)."""
    for t, nm in ((x, "x"), (codes, "codes"), (scale, "scale"), (zero, "zero"), (out, "out"),
                  (workspace, "workspace")):
        _dev(t, nm)
    if status is not None:
        _dev(status, "status")
    tokens = x.numel() // layer.n
    _check("bq_w2a16_linear",
           load().bq_w2a16_linear(ctypes.byref(layer.c), _ptr(x), _dtype_code(x), tokens, _ptr(codes), _ptr(scale),
                                  _ptr(zero), codes.shape[0], bits, group, _ptr(out), _dtype_code(out),
                                  _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(status),
                                  _stream(stream)))
    return out


# ----------------------------------------------------------------------------- block transform + quantize

class BlockTransform:
    """Per-block G x G transforms of C channels, prepared for the fused kernel.

    T: bfloat16 CUDA tensor (C/G, G, G), T[b, o, k] mapping input channel b G + k to
    output channel b G + o.  The prepared table (bq_block_prepare) is kept alive here."""

    def __init__(self, T, stream=None):
        torch = _torch()
        lib = load()
        _dev(T, "T")
        if T.dtype != torch.bfloat16 or T.dim() != 3 or T.shape[1] != T.shape[2]:
            raise ValueError("T must be bfloat16 of shape (C/G, G, G)")
        self.G = int(T.shape[1])
        self.C = int(T.shape[0]) * self.G
        nbytes = lib.bq_block_table_bytes(self.C, self.G)
        if nbytes == 0:
            raise ValueError(f"unsupported block shape C={self.C}, G={self.G}")
        self.T = T
        self.table = torch.empty(nbytes // 2, dtype=torch.int16, device=T.device)
        _check("bq_block_prepare", lib.bq_block_prepare(_ptr(T), self.C, self.G, _ptr(self.table), _stream(stream)))


def block_outputs(rows: int, C: int, fmt: str, device):
    """Empty (codes, scales) tensors of a block-quantized batch."""
    torch = _torch()
    G = {"mxfp4": 32, "nvfp4": 16, "int4": 32}[fmt]
    codes = torch.empty((rows, C // 2), dtype=torch.uint8, device=device)
    scales = torch.empty((rows, C // G), dtype=torch.int16 if fmt == "int4" else torch.uint8, device=device)
    return codes, scales


def bq_block_transform_quantize(bt: BlockTransform, x, fmt: str, codes=None, scales=None, y=None, gscale: float = 1.0,
                                status=None, stream=None):
    """x: bfloat16 (rows, C).  fmt "mxfp4" / "nvfp4" / "int4" writes codes and scales (see
    block_outputs); "none" writes y (float32 or bfloat16, (rows, C))."""
    _dev(x, "x")
    rows = x.numel() // bt.C
    f = BLOCK_FORMATS[fmt]
    if f == BQ_BLOCK_NONE:
        _dev(y, "y")
        yt = _dtype_code(y)
    else:
        _dev(codes, "codes"); _dev(scales, "scales")
        yt = BQ_F32
    if status is not None:
        _dev(status, "status")
    _check("bq_block_transform_quantize",
           load().bq_block_transform_quantize(_ptr(bt.table), bt.C, bt.G, _ptr(x), rows, f, float(gscale), _ptr(y), yt,
                                              _ptr(codes), _ptr(scales), _ptr(status), _stream(stream)))
    return (y,) if f == BQ_BLOCK_NONE else (codes, scales)
