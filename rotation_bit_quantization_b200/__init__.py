"""B200-native learnable butterfly transform + low-bit quantization (ButterflyQuant hot path).

The compute path is libbq.so (hand-written CUDA for sm_100a, C ABI in
include/bq.h); this package only marshals arguments to it (``_lib``), builds it
(``build``) and draws seeded synthetic inputs (``workloads``).
"""

from ._lib import (  # noqa: F401
    BQError,
    BlockTransform,
    Layer,
    block_outputs,
    bq_block_transform_quantize,
    bq_butterfly_bwd,
    bq_butterfly_bwd_noalloc,
    bq_butterfly_bwd_workspace_size,
    bq_butterfly_fwd,
    bq_butterfly_inv,
    bq_precompute_cs,
    bq_transform_quantize,
    bq_weight_rotate_pack,
    bq_uniformity_loss,
    bq_angle_sgd,
    bq_reconstruction_loss,
    bq_reconstruction_workspace_size,
    bq_w2a16_gemm,
    bq_w2a16_gemm_workspace_size,
    bq_w2a16_linear,
    bq_w2a16_linear_workspace_size,
    bq_wait_faults,
    load,
    quant_outputs,
    status_string,
)
