/*
 * bq.h - C ABI of libbq.so: the learnable orthogonal butterfly transform and
 * its fused low-bit quantization, hand-written CUDA for NVIDIA B200 (sm_100a).
 *
 * The method: ButterflyQuant (abstract, arXiv 2509.09679) rotates activations
 * and weights with the same orthogonal Q so that a linear layer is unchanged,
 * y = W x = (W Q^T)(Q x).  Q is a butterfly of Givens rotations with
 * continuous angles: log2(m) stages, stage s rotating the index pairs
 * (i, i + 2^s) with [[cos t, -sin t], [sin t, cos t]], m*log2(m)/2 angles in
 * total (abstract; explainer article, section "butterfly").  Widths that are
 * not a power of two use a Kronecker composite Q = B_m (x) O_r (explainer
 * article, section "butterfly").  The angles are learned by gradient descent
 * (abstract), which needs the backward pass exported here.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All data pointers are DEVICE pointers unless stated; the caller owns
 *    every buffer.  The library never allocates device memory and keeps no
 *    global state (the exceptions are the fixed scratch array of
 *    bq_butterfly_bwd_noalloc and the wait-fault word of bq_wait_faults);
 *    calls on different streams are independent.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Every call is asynchronous on that stream; an error status is
 *    returned before anything is launched when host-side validation fails.
 *  - The m = 4096, r = 1 kernels of bq_butterfly_fwd, bq_butterfly_inv,
 *    bq_transform_quantize and bq_weight_rotate_pack are launched with
 *    programmatic stream serialization: one may start its set-up while the
 *    previous kernel on the stream is still running, and it waits for that
 *    kernel to finish before it reads or writes any buffer, so the caller sees
 *    plain stream order.  A kernel the caller queues next on the stream starts
 *    early only if the caller launched it with that attribute, and must then
 *    call cudaGridDependencySynchronize before it reads these outputs.
 *  - Rows are contiguous and row-major: element (row, i) is at row*n + i.
 *  - Element index i = i1*r + i2 with i1 < m, i2 < r; B_m acts on i1, O_r on i2.
 *  - Angle layout: theta[s*(m/2) + p] for stage s < log2(m) and pair number
 *    p = ((i >> (s+1)) << s) | (i & (2^s - 1)) of the pair (i, i + 2^s).
 *  - Stage order: Q = B_{L-1} ... B_1 B_0 (stage 0, stride 1, acts first).
 *  - Data pointers must be 16-byte aligned; m must be a power of two in
 *    [2, 4096]; r in [1, 8]; n = m*r <= 16384.
 *  - Arithmetic is float32 (bf16 inputs are widened exactly; bf16 outputs are
 *    rounded to nearest even).
 *  - Zero rows (tokens, out_features, count) launch nothing and return BQ_OK
 *    once the other arguments are valid; the data pointers may then be NULL.
 *    The exceptions need at least one token: bq_butterfly_bwd,
 *    bq_butterfly_bwd_noalloc and bq_reconstruction_loss.
 *  - Errors: BQ_ERR_INVALID_ARG (bad sizes, null or misaligned pointers),
 *    BQ_ERR_UNSUPPORTED (valid request outside what this build implements),
 *    BQ_ERR_WORKSPACE (workspace too small), BQ_ERR_CUDA (a CUDA call or a
 *    launch failed).  The library carries its own CUDA runtime state, so its
 *    CUDA error is read with bq_cuda_last_error, not the caller's
 *    cudaGetLastError.  No entry point aborts, traps or asserts on the device.
 */
#ifndef BQ_H_
#define BQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BQ_OK = 0,
  BQ_ERR_INVALID_ARG = 1,
  BQ_ERR_UNSUPPORTED = 2,
  BQ_ERR_WORKSPACE = 3,
  BQ_ERR_CUDA = 4
} bq_status;

typedef enum { BQ_F32 = 0, BQ_BF16 = 1 } bq_dtype;

/* One layer's transform.  The struct itself lives in host memory; its
 * pointers are device pointers.
 *   n = m*r;  table: bq_table_floats(m) floats written by bq_precompute_cs for
 *   this layer's angles;  O: r*r float32 row-major orthogonal matrix, NULL
 *   iff r == 1 (O is an input of the composite, not a learned parameter). */
typedef struct {
  int32_t n, m, r;
  const float* table;
  const float* O;
} bq_layer;

/* Number of floats of the per-layer prepared table for width m (0 if m is
 * not a supported power of two). */
size_t bq_table_floats(int32_t m);

/* Angle preparation, once per layer (explainer article, section "butterfly":
 * the angles parameterise the Givens rotations).  Reads theta[log2(m)*(m/2)]
 * (device, float32) and writes `table` (device, bq_table_floats(m) floats):
 * cos/sin of every angle (float64 sincos rounded to float32) plus the derived
 * per-position coefficients and scales that the scaled-rotation kernels use.
 * The table must be rebuilt whenever theta changes. */
bq_status bq_precompute_cs(const float* theta, int32_t m, float* table, void* stream);

/* Hadamard presets: the table of the butterfly at the angles that make it a
 * Hadamard matrix (explainer article, section "butterfly": H_n is a butterfly
 * with particular angles; QuaRot's fixed and UniSVQ's randomized Hadamard
 * rotations are the baselines the pages compare with).  Angle (s, p) is
 * pi/4 + k pi/2 with k = quadrant[s*(m/2) + p] & 3 (quadrant: device bytes
 * [log2(m)*(m/2)], or NULL for k = 0 everywhere, which gives
 * Q = H_m diag(d) / sqrt(m) with d the Kronecker power of (1, -1)).  Every
 * entry of Q is +-1/sqrt(m).  cos and sin are taken as +-1/sqrt(2) exactly,
 * so the scaled-form coefficients are exactly +-1 and the output scale is
 * +-2^(-log2(m)/2) (a power of two for even log2 m).
 * theta: NULL, or device float32 [log2(m)*(m/2)] that receives the angles (a
 * starting point for calibration; bq_precompute_cs of them reproduces the
 * table up to float32 rounding of the angles). */
bq_status bq_precompute_hadamard(int32_t m, const uint8_t* quadrant, float* table, float* theta, void* stream);

/* y = Q x for every row (abstract: the activation side Q x).
 * x: rows*n elements of type xt; y: rows*n elements of type yt.  x == y is
 * allowed when xt == yt (each row is read completely before it is written). */
bq_status bq_butterfly_fwd(const bq_layer* layer, const void* x, bq_dtype xt,
                           void* y, bq_dtype yt, int64_t rows, void* stream);

/* x = Q^T y for every row: stages L-1 .. 0 with every angle negated, and O_r^T
 * for the composite (Q is orthogonal by construction, abstract).  Same layout
 * and aliasing rule as bq_butterfly_fwd. */
bq_status bq_butterfly_inv(const bq_layer* layer, const void* y, bq_dtype yt,
                           void* x, bq_dtype xt, int64_t rows, void* stream);

/* Bytes of workspace bq_butterfly_bwd needs for num_layers layers of width m
 * with rows_per_layer tokens each. */
size_t bq_butterfly_bwd_workspace_size(int32_t m, int32_t num_layers, int64_t rows_per_layer);

/* Backward for calibration (abstract: angles learned by gradient-based
 * optimisation), all layers in ONE launch.  For layer l with loss linear in
 * Y_l and upstream gradient dY_l:
 *   Y_l = Q_l X_l;  dX_l = Q_l^T dY_l;
 *   dtheta_l[s*(m/2)+p] = sum over tokens of (g_j v_i - g_i v_j), where v and g
 *   are the output and output-gradient of stage s at its pair (i, j).
 * layers: HOST array of num_layers (<= 128) descriptors, all with the same m
 *   and r == 1.
 * x: [num_layers][rows_per_layer][m] of type xt; y: same shape of type yt;
 * dy, dx: float32, same shape; dtheta: float32 [num_layers][log2(m)*(m/2)].
 * rows_per_layer >= 1.  The token reduction is deterministic (fixed-order
 * partial sums in `workspace`, reduced by the last block of each layer);
 * repeated calls give bitwise identical dtheta.  workspace: device, >= the size queried above,
 * 16-byte aligned; its contents on entry are irrelevant. */
bq_status bq_butterfly_bwd(const bq_layer* layers, int32_t num_layers,
                           const void* x, bq_dtype xt, void* y, bq_dtype yt,
                           const float* dy, float* dx, float* dtheta,
                           int64_t rows_per_layer, void* workspace,
                           size_t workspace_bytes, void* stream);

/* Size in bytes of the fixed device scratch that bq_butterfly_bwd_noalloc uses. */
#define BQ_NOALLOC_SCRATCH_BYTES (8u << 20)

/* bq_butterfly_bwd without a workspace argument, for callers that cannot
 * allocate device memory when they run the backward: code running while
 * another framework owns the device allocator, real-time loops that must not
 * block in an allocator, or processes whose device memory is fully reserved
 * by a pool.  The paper has no counterpart to this entry point.
 *
 * Arguments, results and the deterministic dtheta reduction are those of
 * bq_butterfly_bwd; y and dx are bitwise identical to it.  dtheta is summed
 * in possibly fewer, larger token chunks (so possibly in a different order):
 * the library's scratch is one file-scope device array of
 * BQ_NOALLOC_SCRATCH_BYTES bytes, which every GPU that loads the library
 * keeps until the process exits, and the chunk count is reduced until the
 * partial sums fit in it.  If even one chunk per layer does not fit
 * (num_layers * log2(m) * m/2 * 4 bytes + 512 > BQ_NOALLOC_SCRATCH_BYTES,
 * e.g. more than 85 layers of width 4096) it returns BQ_ERR_WORKSPACE and
 * launches nothing.  Nothing is allocated: no cudaMalloc, no cudaFree.
 * Fewer chunks also mean fewer CTAs: at width 4096 the scratch holds 85
 * (layer, chunk) slots, so at most 85 SMs work (32 layers get 64 CTAs, two
 * chunks per layer) and the call takes about 2.3 times as long as
 * bq_butterfly_bwd with a full-size workspace on a 148-SM B200.
 * The first call on a device looks up the array's device address (once per
 * device, with that device current); make that first call before any stream
 * capture.  Every call shares the one array and clears the part that must
 * start at zero itself; calls whose executions overlap on the GPU (different
 * streams, or concurrent host threads) race on it and must be serialised by
 * the caller. */
bq_status bq_butterfly_bwd_noalloc(const bq_layer* layers, int32_t num_layers,
                                   const void* x, bq_dtype xt, void* y, bq_dtype yt,
                                   const float* dy, float* dx, float* dtheta,
                                   int64_t rows_per_layer, void* stream);

/* Fused Q x followed by per-group asymmetric round-to-nearest quantization and
 * packing (2-bit weights: explainer article, section "training & results";
 * RTN block quantizer: WUSH technical summary, section 2).  Per group of
 * `group` contiguous outputs of a row (group divides n, group % 32 == 0):
 *   lo, hi = min, max;  scale16 = fp16_rn((hi - lo) / qmax);  s = scale16
 *   (s = 1 when hi == lo or scale16 == 0);  z = clamp(rint(-lo / s), 0, qmax);
 *   q = clamp(rint(y / s) + z, 0, qmax), rint half-to-even, IEEE float32
 *   division; qmax = 2^bits - 1.
 * The y quantized is bitwise the float32 output bq_butterfly_fwd produces.
 * codes: [rows][n*bits/8] bytes, lowest element in the lowest bits
 *   (INT4: q[2k] | q[2k+1] << 4; INT2: q[4k] | q[4k+1] << 2 | ...);
 * scale_f16, zero_f16: [rows][n/group] fp16 bit patterns.  bits: 2 or 4. */
bq_status bq_transform_quantize(const bq_layer* layer, const void* x, bq_dtype xt,
                                int64_t rows, int32_t bits, int32_t group,
                                uint8_t* codes, uint16_t* scale_f16,
                                uint16_t* zero_f16, void* stream);

/* Weight side of the invariance y = (W Q^T)(Q x) (abstract): row r of W Q^T
 * is Q w_r, so this rotates every row of W [out_features][n] and quantizes and
 * packs it exactly as bq_transform_quantize does (identical bits for identical
 * input); the W2A16 setting uses bits = 2. */
bq_status bq_weight_rotate_pack(const bq_layer* layer, const void* w, bq_dtype wt,
                                int64_t out_features, int32_t bits, int32_t group,
                                uint8_t* codes, uint16_t* scale_f16,
                                uint16_t* zero_f16, void* stream);

/* Uniformity regulariser of calibration and its gradient.  The angles are learned
 * with a loss that includes a uniformity regularisation of the rotated
 * activations (abstract): the KL divergence between their distribution and the
 * uniform distribution over the quantization intervals (explainer article,
 * section "training & results").  Per group of `group` contiguous values of a
 * row of y (float32, [rows][n], e.g. the output of bq_butterfly_fwd):
 *   s, z  the group's RTN scale and zero point (the rules of
 *         bq_transform_quantize), B = 2^bits levels;
 *   u     = y / s + z clamped to [0, 2^bits - 1], spread over its two nearest
 *         levels with the triangular kernel max(0, 1 - |u - c|);
 *   p_c   = mean over the group of those weights; p~ = (p + eps) / (1 + B eps);
 *   KL    = sum_c p~_c log(B p~_c).
 * kl_group: [rows][n/group] float32 per-group KL (device, written).
 * dy: [rows][n] float32 gradient of the mean KL over all groups with s and z held
 *   constant (zero where u is outside the open interval (0, 2^bits - 1)), or NULL.
 * loss: one float32, the mean KL over all groups (summed in a fixed order), or
 *   NULL.  bits: 2 or 4; group: 64, 128 or 256 dividing n; 0 < eps < 1.
 * y and dy must be 16-byte aligned.  Results are bitwise reproducible. */
bq_status bq_uniformity_loss(const float* y, int64_t rows, int32_t n, int32_t bits, int32_t group, float eps,
                             float* kl_group, float* dy, float* loss, void* stream);

/* One gradient step on the angles: theta[i] -= lr * dtheta[i] for i < count
 * (device float32 arrays; rebuild the layer's table with bq_precompute_cs
 * afterwards). */
bq_status bq_angle_sgd(float* theta, const float* dtheta, int64_t count, float lr, void* stream);

/* Bytes of workspace bq_reconstruction_loss needs (0 for unsupported sizes). */
size_t bq_reconstruction_workspace_size(int32_t n, int64_t out_features, int64_t tokens, int32_t bits,
                                        int32_t group);

/* Reconstruction loss of one linear layer under weight quantization, with a
 * straight-through estimator, and its gradient in the angles: the quantized
 * layer's output should match the original one (explainer article, section
 * "training & results"), through the invariance y = W x = (W Q^T)(Q x)
 * (abstract).  With V = W Q^T, W_hat = the dequantized bq_weight_rotate_pack
 * codes of W ((q - z) s), x~_t = Q x_t and r[t][o] = (W_hat x~_t)_o - (W x_t)_o:
 *   loss = (1/T) sum_t ||r_t||^2;
 *   dtheta = backward(x, (2/T) r W_hat) + backward(W, (2/T) r^T x~), taking
 *            dW_hat / dV as the identity (straight-through).
 * layer: r == 1 (n = m, a power of two).  w: [out_features][n] float32; x:
 * [tokens][n] float32 (device, 16-byte aligned).  dtheta: log2(n) * n/2 floats
 * (written); loss: one float (written).  workspace: device, 256-byte aligned,
 * >= bq_reconstruction_workspace_size(...).  bits / group: as for
 * bq_weight_rotate_pack.  Deterministic (fixed summation orders). */
bq_status bq_reconstruction_loss(const bq_layer* layer, const float* w, int64_t out_features, const float* x,
                                 int64_t tokens, int32_t bits, int32_t group, float* dtheta, float* loss,
                                 void* workspace, size_t workspace_bytes, void* stream);

/* W2A16 consumer GEMM on the tensor cores (tcgen05): the quantized layer of the
 * invariance y = W x = (W Q^T)(Q x) (abstract) with 2-bit weights and 16-bit
 * activations (explainer article, section "training & results": W2A16):
 *   out[t][o] = sum_k x[t][k] * bf16((q[o][k] - z[o][k / group]) * s[o][k / group])
 * where (q - z) s is formed exactly in float32 and rounded to nearest-even
 * bfloat16, products are exact and sums are float32.
 * x: [tokens][n] bfloat16, the rotated activations (e.g. bq_butterfly_fwd with
 *   yt = BQ_BF16); device, 16-byte aligned.
 * codes, scale_f16, zero_f16: the packed weights of bq_weight_rotate_pack for
 *   [out_features][n] (codes [out][n*bits/8] bytes, 16-byte aligned; scale and
 *   zero [out][n/group] fp16 bit patterns).  bits: 2, or 4 for W4A16.
 * group: 64, 128 or 256 dividing n; n: a multiple of 64.
 * out: [tokens][out_features] float32 (out_t = BQ_F32) or bfloat16 (BQ_BF16,
 *   rounded to nearest-even); device.
 * workspace: NULL, or device memory (256-byte aligned) of at least
 *   bq_w2a16_gemm_workspace_size(tokens, n, out_features) bytes.  With few
 *   output tiles (few tokens) the kernel splits K over more SMs and adds the
 *   slices' float32 partial sums in a fixed order (bitwise reproducible); without
 *   the workspace it does not split K (same results up to float32 summation
 *   order, slower for decode-sized token counts).  1-3 tokens (with n a multiple
 *   of 512 and tokens * n <= 16384) run on a CUDA-core kernel instead, with the
 *   same bf16 weights and float32 products; it needs no workspace.
 * status: NULL, or a device int32 the caller zeroes; the kernel ORs a nonzero
 *   code into it if one of its internal waits gave up after one second (the
 *   output is then incomplete): 1 the copy issuer waited for a free stage,
 *   2 a dequantizing thread for its copies, 4 the MMA issuer for its operands,
 *   8 the MMA issuer for the accumulator, 16 the epilogue for the accumulator,
 *   32 the final wait for copies or MMAs in flight.  Nothing is launched on
 *   invalid arguments; BQ_ERR_UNSUPPORTED if the driver's tensor-map encoder is
 *   unavailable. */
bq_status bq_w2a16_gemm(const void* x, int64_t tokens, int32_t n, const uint8_t* codes,
                        const uint16_t* scale_f16, const uint16_t* zero_f16, int64_t out_features,
                        int32_t bits, int32_t group, void* out, bq_dtype out_t, void* workspace,
                        size_t workspace_bytes, int32_t* status, void* stream);

/* Bytes of split-K workspace bq_w2a16_gemm uses for this shape on the current
 * device (0 when K is not split). */
size_t bq_w2a16_gemm_workspace_size(int64_t tokens, int32_t n, int64_t out_features);

/* Bytes of workspace bq_w2a16_linear needs: the bfloat16 rotated activations
 * plus the GEMM's split-K workspace. */
size_t bq_w2a16_linear_workspace_size(int32_t n, int64_t tokens, int64_t out_features);

/* The whole quantized layer from raw activations: x~ = Q x (bq_butterfly_fwd to
 * bfloat16 into the workspace), then bq_w2a16_gemm(x~, ...).  x: [tokens][n] of
 * dtype xt; workspace: device, 256-byte aligned, >= bq_w2a16_linear_workspace_size
 * (at least the activations' bytes, else BQ_ERR_WORKSPACE); other arguments as
 * for bq_w2a16_gemm. */
bq_status bq_w2a16_linear(const bq_layer* layer, const void* x, bq_dtype xt, int64_t tokens,
                          const uint8_t* codes, const uint16_t* scale_f16, const uint16_t* zero_f16,
                          int64_t out_features, int32_t bits, int32_t group, void* out, bq_dtype out_t,
                          void* workspace, size_t workspace_bytes, int32_t* status, void* stream);

/* ---------------------------------------------------------------------------
 * Block-wise transform fused with AbsMax block quantization (WUSH technical
 * summary, section 2 "method": per-block G x G linear transforms of the
 * activations, an AbsMax-scaled round-to-nearest block quantizer in FP and INT
 * formats; "implementation": the transform fused with activation quantization
 * on the GPU).  Per row and block b of G channels:
 *   y[b G + o] = sum_k T[b][o][k] x[b G + k]   (bf16 operands, float32 sums),
 * then one of:
 *   BQ_BLOCK_MXFP4 (G = 32): X = floor(log2 max|y|) - 2 clamped to [-127, 127]
 *     (-127 for an all-zero block), scale byte X + 127 (E8M0); codes
 *     E2M1(y / 2^X): magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6} as codes 0..7, sign
 *     in bit 3, round to nearest even, saturating at 6;
 *   BQ_BLOCK_NVFP4 (G = 16): scale = E4M3(max|y| / 6) (round to nearest even,
 *     saturating at 448), stored as its FP8 byte; codes E2M1(y / (scale *
 *     gscale)) with the product and the division in IEEE float32 (all +0
 *     when the scale is 0);
 *   BQ_BLOCK_INT4 (G = 32): scale16 = fp16(max|y| / 7) (1.0 for an all-zero or
 *     underflowing block), codes clamp(rint(y / scale), -7, 7) in IEEE float32,
 *     half to even, as 4-bit two's complement;
 *   BQ_BLOCK_NONE (G = 16 or 32): y itself, float32 or bfloat16.
 * Codes are [rows][C / 2] bytes, two per byte, lowest channel in the low nibble;
 * scales [rows][C / G] (bytes for MXFP4 and NVFP4, fp16 bits for INT4). */
typedef enum { BQ_BLOCK_NONE = 0, BQ_BLOCK_MXFP4 = 1, BQ_BLOCK_NVFP4 = 2, BQ_BLOCK_INT4 = 3 } bq_block_format;

/* Bytes of the prepared transform table for C channels in blocks of G (16 or 32);
 * 0 when C is not a positive multiple of 64 or G is not 16 or 32.  Host only. */
size_t bq_block_table_bytes(int32_t C, int32_t G);

/* Prepare the transform table from T: [C / G][G][G] bfloat16 (T[b][o][k] maps
 * input channel b G + k to output channel b G + o), device, 2-byte aligned; table:
 * device, 16-byte aligned, bq_block_table_bytes(C, G) bytes, written with each
 * 64-channel tile's blocks side by side (the layout the kernel copies).  Async. */
bq_status bq_block_prepare(const uint16_t* T, int32_t C, int32_t G, uint16_t* table, void* stream);

/* The fused block transform and quantization of x: [rows][C] bfloat16 (device,
 * 16-byte aligned).  table from bq_block_prepare with the same C and G; format
 * one of the above with its G; gscale > 0 (NVFP4 only).  BQ_BLOCK_NONE writes
 * y: [rows][C] of yt (16-byte aligned) and ignores codes / scales; the others
 * write codes (16-byte aligned) and scales (2-byte aligned).  status: NULL, or a
 * device int32 the caller zeroes; the kernel ORs a nonzero code into it if any
 * of its barrier waits gave up after one second (it then stops early and its
 * outputs are incomplete).  Runs on the tensor cores (tcgen05, operands copied
 * by the tensor memory accelerator).  Async. */
bq_status bq_block_transform_quantize(const uint16_t* table, int32_t C, int32_t G, const void* x, int64_t rows,
                                      bq_block_format format, float gscale, void* y, bq_dtype yt,
                                      uint8_t* codes, void* scales, int32_t* status, void* stream);

/* The library's last CUDA runtime error (a cudaError_t value, 0 for none),
 * cleared by the call: after BQ_ERR_CUDA it says which CUDA call or launch
 * failed.  Host only; launches nothing. */
int32_t bq_cuda_last_error(void);

/* The device's wait-fault word.  The m = 4096, r = 1 kernels of bq_butterfly_fwd,
 * bq_butterfly_inv, bq_transform_quantize and bq_weight_rotate_pack pass rows
 * between the warps of a row group through shared-memory barriers whose waits give
 * up after one second, so that a fault elsewhere cannot hold an SM; a wait that
 * gives up ORs 1 into this word of the library's memory on the current device
 * (those calls take no status word).  No correct launch sets it.
 * value: host int32 that receives the word; clear != 0 resets it to 0.
 * Synchronises `stream` (the word is read after the work queued before it).
 * Errors: BQ_ERR_INVALID_ARG for a NULL value (checked before any CUDA call),
 * BQ_ERR_CUDA if a copy or the synchronisation fails. */
bq_status bq_wait_faults(int32_t* value, int32_t clear, void* stream);

/* Static description of a cudaError_t value from bq_cuda_last_error. */
const char* bq_cuda_error_string(int32_t code);

/* Static, human-readable name of a status code. */
const char* bq_status_string(bq_status status);

#ifdef __cplusplus
}
#endif

#endif /* BQ_H_ */
