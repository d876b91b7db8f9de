"""Plain float64 CPU oracle for the butterfly transform + low-bit quantization path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or link
this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code with the CUDA library (no kernels, headers, tables or helpers); the only
thing both sides consume is the seeded input generator module, which holds none
of the method's arithmetic.

What it computes, and where the method is stated:

* ``butterfly``  - the orthogonal butterfly transform Q built from Givens
  rotations with continuous angles (ButterflyQuant abstract, arXiv 2509.09679;
  explainer article, section "butterfly"), its inverse Q^T, the Kronecker
  composite B_m (x) O_r for widths that are not a power of two (explainer
  article, section "butterfly", last paragraph), and the backward pass
  (dX, dtheta) that gradient-based calibration needs (abstract: the continuous angles
  are learned by gradient descent).
* ``quant``      - per-group asymmetric round-to-nearest quantization with fp16
  scale and zero point and little-endian INT2/INT4 packing (2-bit weights:
  explainer article, section "training & results"; RTN block quantizer: WUSH
  technical summary, section 2 "method").  The pages give no formula; the
  readings taken are listed in the module docstring and in the design notes.

* ``calib``      - the calibration losses: the uniformity regulariser (the
  abstract names a uniformity regularisation of the transformed activations;
  explainer article, section "training & results": the KL divergence between the
  rotated activations' distribution and the uniform distribution over the
  quantization intervals) as a soft histogram over each group's RTN levels, its
  KL divergence to uniform and the gradient with respect to the activations;
  and the reconstruction loss of a quantized layer with a straight-through
  estimator.  The estimators and smoothing are readings listed in the module
  docstring.
* ``blockq``     - the block-wise transform of the WUSH workload (WUSH technical
  summary, section 2: per-block G x G linear transforms of the activations,
  fused with an AbsMax-scaled round-to-nearest block quantizer in FP or INT
  formats) and its MXFP4, NVFP4 and symmetric INT4 quantizers; pinned in
  ``tests/test_oracle_blockq_pins.py`` (dense block-diagonal product, exact
  rational E2M1 rounding, torch's FP8 E4M3 conversion, brute force, fixtures).
* ``w2a16``      - the W2A16 consumer GEMM (explainer article, section "training
  & results": 2-bit weights, 16-bit activations; abstract: y = (W Q^T)(Q x)):
  bfloat16 activations times the bfloat16-rounded dequantized codes, summed
  exactly in float64.

Parity status: every function here is pinned by an independent check in
``tests/test_oracle_pins.py`` (closed forms, the Hadamard special case against
``scipy.linalg.hadamard``, explicit dense stage matrices, ``numpy.kron``, finite
differences, brute-force quantizer search).  The stage order, Kronecker order,
quantizer details and packing layout are conventions the pages leave open;
those are pinned by convention plus self-consistency only.
"""

from . import butterfly, quant  # noqa: F401
