/*
 * libtpblock -- the Megatron column->row tensor-parallel transformer block on
 * one B200 (sm_100a): forward passes of the FFN block, the attention sub-layer
 * and the pre-LN layer, and the backward pass of the FFN block.
 *
 * Source of the method: "Tensor Parallelism > Combining Column and Row
 * Parallelism" (mbrenndoerfer.com), cited below as [TP-CR]:
 *   step 1  column-parallel W1: shard i computes Z_i = X W1_i, then GeLU(Z_i),
 *           with no communication;
 *   step 2  row-parallel W2: Y_i = GeLU(Z_i) W2_i, a partial sum over the
 *           full output;
 *   step 3  all-reduce: Y = sum_i Y_i;
 *   and the paragraphs on multi-head attention (QKV column-parallel by head
 *   group, output projection row-parallel), on feature reductions (LayerNorm
 *   needs the full row) and on the two reductions per layer with residual
 *   adds between the sub-layers.
 *
 * All t logical shards run on the one GPU; step 3 becomes an on-device
 * reduction in a fixed order (no atomics, bitwise reproducible).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Pointers are DEVICE pointers unless stated otherwise.  The caller owns
 *    every buffer, including the workspace; the library never allocates,
 *    frees or synchronises (except tp_get_device_status, which synchronises
 *    the given stream).
 *  - Matrices are row-major.  A tp_shard is a view {ptr, ld}: element (r, c)
 *    is at ptr + r*ld + c (ld in elements).  Shards may point into one big
 *    matrix (e.g. W1_i = W1 + i*f/t with ld = f) or into separate buffers.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL is the
 *    legacy default stream).  Launches go to that stream only.
 *  - Host validation runs before any launch.  On failure the call returns
 *    TP_ERR_INVALID_ARG or TP_ERR_UNSUPPORTED, launches nothing, and
 *    tp_last_error() describes the failed check.  A failed launch returns
 *    TP_ERR_CUDA.  A device-side wait that runs past its time limit makes the
 *    kernel stop, and tp_get_device_status() then returns TP_ERR_TIMEOUT.
 *  - bf16 paths: element type IEEE bfloat16, fp32 accumulation, results
 *    rounded to nearest even.  Every bf16 pointer must be 16-byte aligned,
 *    every ld a multiple of 8, and h, f/t and (heads/t)*d multiples of 64.
 *  - Stateless and thread-safe apart from the optional launch trace.
 */
#ifndef TPBLOCK_H
#define TPBLOCK_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define TP_API __attribute__((visibility("default")))
#else
#define TP_API
#endif

#define TP_MAX_SHARDS 16

typedef enum {
  TP_OK = 0,
  TP_ERR_INVALID_ARG = 1, /* null pointer, bad size, misaligned pointer or ld */
  TP_ERR_UNSUPPORTED = 2, /* valid but outside what the kernels implement */
  TP_ERR_WORKSPACE = 3,   /* workspace missing or smaller than *_workspace_bytes */
  TP_ERR_CUDA = 4,        /* a CUDA runtime call or launch failed */
  TP_ERR_TIMEOUT = 5,     /* a device wait ran out (reported by tp_get_device_status) */
  TP_ERR_RANGE = 6        /* an fp16 intermediate exceeded 65504 (reported by tp_get_device_status) */
} tp_status;

typedef enum { TP_BF16 = 0, TP_FP32 = 1, TP_FP16 = 2 } tp_dtype;

/* How step 3 (the all-reduce) is done on one device.
 * TP_REDUCE_FUSED:    one row-GEMM tile accumulates the K-slices of all t
 *                     shards into one fp32 accumulator, in a fixed order that
 *                     depends only on the tile's place in the schedule
 *                     (ascending or descending K, whichever starts on data
 *                     still in L2), and its epilogue adds the bias and the
 *                     residual.  The result is the same bits for every t.
 *                     A tile's place in the schedule, and the tile width
 *                     (256 or 512 columns, picked from the same count), depend
 *                     on the number of CTA pairs the device runs at once (74
 *                     on a 148-SM B200), so the bits are reproducible across
 *                     runs and processes on devices with the same SM count
 *                     (and the same TPB_GEMM_WIDE setting).
 * TP_REDUCE_PARTIALS: the row GEMM writes t fp32 partials Y_i [t, M, h] to the
 *                     workspace (TMA stores) and a reduce kernel sums them in
 *                     the order 0..t-1, then adds bias and residual.  With the
 *                     environment variable TPB_REDUCE_IN_GEMM=1 the sum is
 *                     taken inside the row GEMM instead: its last shard's
 *                     tiles add the stored partials 0..t-2 and their own
 *                     accumulator in the same order (same bits), overlapping
 *                     the reduction with the other tiles' multiplication. */
typedef enum { TP_REDUCE_FUSED = 0, TP_REDUCE_PARTIALS = 1 } tp_reduce_mode;

/* Element-wise nonlinearity of step 1: exact GeLU z*Phi(z) (erf form) or ReLU. */
typedef enum { TP_ACT_GELU = 0, TP_ACT_RELU = 1 } tp_activation;

/* A weight shard.  `dtype` is TP_BF16 (0, so a zeroed struct means bf16) or
 * TP_FP16; every shard of one weight has the same dtype.  In each tensor-core
 * GEMM the activation operand is produced in its weight's type: an fp16 W2
 * makes act(Z) fp16, an fp16 Wqkv makes the layer's LN1 output fp16, and so on.
 * fp16 has 3 more mantissa bits than bf16 at the same tensor-core rate, and
 * bf16 weights of ordinary magnitude convert to fp16 exactly; a bf16 caller
 * gets fp16 intermediates only by passing fp16 copies of its weights.  fp16's
 * range ends at 65504: an intermediate above it is stored as +-inf and
 * tp_get_device_status() reports TP_ERR_RANGE. */
typedef struct {
  const void* ptr; /* device pointer to element (0, 0) of the shard */
  int64_t ld;      /* row stride in elements */
  int32_t dtype;   /* TP_BF16 or TP_FP16 */
  int32_t reserved;
} tp_shard;

typedef void* tp_stream_t; /* cudaStream_t */

/* ------------------------------------------------------------------ FFN block
 * [TP-CR] steps 1-3:  out = sum_{i<t} act(X W1_i + b1_i) W2_i + b2 + residual.
 *
 *  X        [M, h], dtype, ld = h (contiguous).
 *  W1[i]    [h, f/t] view, i < t (column shard i of W1 [h, f]); same dtype as X.
 *  b1       array of t pointers to [f/t] vectors, or NULL (no bias).
 *  W2[i]    [f/t, h] view (row shard i of W2 [f, h]); TP_BF16 or TP_FP16
 *           (act(Z) is stored in the same type).
 *  b2       [h] or NULL; added once, after the sum over shards.
 *  residual [M, h] or NULL; added after the sum (may alias X).
 *  out      [M, h], contiguous; must not alias X, residual or the weights.
 *  dtype    TP_BF16 (tensor cores) or TP_FP32 (exact fp32 FFMA, no TF32).
 *  mode     see tp_reduce_mode (ignored for TP_FP32, which always uses partials).
 *  ws       device workspace of at least tp_ffn_workspace_bytes(...) bytes,
 *           256-byte aligned.  Holds act(Z) [M, f] (and, in TP_REDUCE_PARTIALS
 *           mode, the partials and one arrival counter per 32x128 output region
 *           for the in-GEMM reduction, which the call zeroes on the stream
 *           first).  Its contents on entry are ignored.
 * Limits: 1 <= t <= TP_MAX_SHARDS, f % t == 0, M >= 1.
 */
TP_API size_t tp_ffn_workspace_bytes(int64_t M, int64_t h, int64_t f, int t, tp_dtype dtype, tp_reduce_mode mode);

TP_API tp_status tp_ffn_forward(const void* X, int64_t M, int64_t h, int64_t f, int t, const tp_shard* W1,
                         const void* const* b1, const tp_shard* W2, const void* b2, const void* residual,
                         void* out, tp_dtype dtype, tp_reduce_mode mode, void* ws, size_t ws_bytes,
                         tp_stream_t stream);

/* Same block with a chosen nonlinearity ([TP-CR], the paragraph on where the
 * nonlinearity fits: "GeLU (or ReLU)"). */
TP_API tp_status tp_ffn_forward_act(const void* X, int64_t M, int64_t h, int64_t f, int t, const tp_shard* W1,
                             const void* const* b1, const tp_shard* W2, const void* b2, const void* residual,
                             void* out, tp_dtype dtype, tp_reduce_mode mode, tp_activation act, void* ws,
                             size_t ws_bytes, tp_stream_t stream);

/* FFN block for callers that cannot allocate device memory (no counterpart on
 * the page: it exists for callers that run inside a host framework owning the
 * whole device memory pool, or in loops where a cudaMalloc and its possible
 * device synchronisation are not allowed).  Same math as tp_ffn_forward with
 * GeLU, bf16 X/W1/W2 and the fused reduction, but act(Z) goes to a static
 * 16 MiB device array inside the library instead of a workspace:
 * M * f <= 8,388,608, else TP_ERR_UNSUPPORTED with the sizes in tp_last_error().
 * The caller still passes every input and the output.  It calls no cudaMalloc
 * or cudaFree.  Every call on a device shares that array, so calls that overlap
 * on the GPU (e.g. on two streams) race; nothing in it needs to start at zero.
 * The first call on each device looks up the array's device address: make it
 * before any stream capture.  Later calls on a stream that is not capturing
 * look it up again (a device reset may move it); capturing calls reuse the
 * last address.  Each GPU that loads the library keeps the 16 MiB until the
 * process exits. */
TP_API tp_status tp_ffn_forward_noalloc(const void* X, int64_t M, int64_t h, int64_t f, int t, const tp_shard* W1,
                                        const void* const* b1, const tp_shard* W2, const void* b2,
                                        const void* residual, void* out, tp_stream_t stream);

/* ------------------------------------------------------------------ FFN block, backward pass
 * Gradients of the FFN block for the upstream gradient dY = dL/d(out).  [TP-CR]
 * gives the forward pass and its one all-reduce per two-layer block; the
 * backward pass is the chain rule back through steps 3, 2 and 1, read with the
 * page's column/row pairing: dY is the same for every shard (it is the
 * gradient of the all-reduce's output), so the row layer's input gradient
 * dA_i = dY W2_i^T is local to shard i, and the column layer's input gradient
 * dX = sum_i dZ_i W1_i^T is a sum over shards, the backward pass's one
 * reduction (taken here in one accumulator over the shards' K-slices).
 *
 *   Z_i = X W1_i + b1_i,  A_i = act(Z_i)       (recomputed from X: nothing is
 *                                               kept from the forward call)
 *   dW2_i = A_i^T dY,     db2 = column sums of dY
 *   dZ_i = (dY W2_i^T) * act'(Z_i)
 *   dW1_i = X^T dZ_i,     db1_i = column sums of dZ_i
 *   dX = sum_i dZ_i W1_i^T (+ dX_add)
 *
 *  X, W1, b1, W2  as in tp_ffn_forward, bf16 only (TP_BF16 shards).
 *  dY       [M, h] bf16, contiguous.
 *  dX_add   [M, h] bf16 or NULL: added to dX (pass dY when the forward's
 *           residual was X: the residual path's gradient is dY itself).
 *  dX       [M, h] bf16 out, contiguous; must not alias X, dY or dX_add.
 *  dW1      [h, f] fp32 out, contiguous: shard i's gradient is the column
 *           block [i*f/t, (i+1)*f/t).  Overwritten, not accumulated.
 *  db1      [f] fp32 out or NULL.   dW2  [f, h] fp32 out, contiguous: shard
 *           i's gradient is the row block [i*f/t, (i+1)*f/t).  db2 [h] fp32
 *           out or NULL.
 *  act      the forward's nonlinearity (GeLU'(z) = Phi(z) + z phi(z); ReLU'
 *           is 1 for z > 0, else 0).
 *  ws       tp_ffn_backward_workspace_bytes(...) bytes, 256-byte aligned:
 *           act(Z) (bf16), act'(Z) (fp16, in [-0.17, 1.13] for GeLU) and dZ
 *           (bf16), each [M, f].
 * The sums over rows (dW, db) and over shards (dX) are taken in a fixed
 * order: results are bitwise reproducible on devices with the same SM count.
 * M == 0 zeroes dW1, dW2, db1, db2.  Limits as tp_ffn_forward's bf16 path.
 */
TP_API size_t tp_ffn_backward_workspace_bytes(int64_t M, int64_t h, int64_t f, int t);
TP_API tp_status tp_ffn_backward(const void* X, int64_t M, int64_t h, int64_t f, int t, const tp_shard* W1,
                                 const void* const* b1, const tp_shard* W2, const void* dY, const void* dX_add,
                                 void* dX, float* dW1, float* db1, float* dW2, float* db2, tp_activation act,
                                 void* ws, size_t ws_bytes, tp_stream_t stream);

/* ------------------------------------------------------------------ parallel linears
 * Column-parallel linear alone ([TP-CR] step 1), bf16 or fp16 (W's dtype):
 *   out[:, i*n/t : (i+1)*n/t] = act(X W_i + b_i)   for i < t,
 *   X [M, k] contiguous, W[i] [k, n/t] views, b NULL or t pointers to [n/t] bf16,
 *   out [M, n] contiguous.  X and out have W's dtype.
 *   act: -1 = identity, else tp_activation. */
TP_API tp_status tp_column_linear_forward(const void* X, int64_t M, int64_t k, int64_t n, int t, const tp_shard* W,
                                   const void* const* b, int act, void* out, tp_stream_t stream);

/* Row-parallel linear with the reduction ([TP-CR] steps 2-3), bf16:
 *   out = sum_{i<t} A[:, i*k/t : (i+1)*k/t] W_i + bias + residual,
 *   A [M, k] contiguous (the column layer's output), W[i] [k/t, n] views,
 *   bias [n] or NULL, residual [M, n] or NULL, out [M, n] bf16.
 *   ws: tp_row_linear_workspace_bytes(...) bytes (0 in TP_REDUCE_FUSED mode). */
TP_API size_t tp_row_linear_workspace_bytes(int64_t M, int64_t n, int t, tp_reduce_mode mode);
TP_API tp_status tp_row_linear_forward(const void* A, int64_t M, int64_t k, int64_t n, int t, const tp_shard* W,
                                const void* bias, const void* residual, void* out, tp_reduce_mode mode, void* ws,
                                size_t ws_bytes, tp_stream_t stream);

/* ------------------------------------------------------------------ attention sub-layer
 * [TP-CR], paragraphs on multi-head attention and head independence: the QKV
 * projection is column-parallel by head group, each group attends over its
 * own heads, the output projection is row-parallel and its partial sums are
 * reduced:
 *   out = sum_{i<t} O_i Wo_i + bo + residual,
 *   O_i = concat over heads g of group i of softmax(Q_g K_g^T / sqrt(d) + mask) V_g.
 *
 *  X        [B*S, h] bf16 contiguous (row r = b*S + s).
 *  Wqkv[i]  [h, 3*Hg*d] bf16 view, Hg = heads/t: columns [Q heads | K heads | V heads]
 *           of group i, head g of the group at columns g*d .. g*d+d-1 of each block.
 *           Q, K, V, the softmax weights P and the tensor-core operands of
 *           Q K^T and P V are fp16 (the scores' sensitivity to rounding of Q and
 *           K grows with their magnitude); accumulation is fp32.
 *  bqkv     NULL or t pointers to [3*Hg*d] bf16.
 *  Wo[i]    [Hg*d, h] view (rows of the output projection for group i's heads),
 *           TP_BF16 or TP_FP16 (the attention output O is stored in that type).
 *  bo       [h] or NULL.  residual [B*S, h] or NULL.  out [B*S, h] bf16.
 *  causal   1: key j is visible to query i iff j <= i (same sequence); 0: all keys.
 * Limits: d == 128, heads % t == 0, S >= 1.
 */
TP_API size_t tp_attn_workspace_bytes(int B, int S, int h, int heads, int d, int t, tp_reduce_mode mode);
TP_API tp_status tp_attn_forward(const void* X, int B, int S, int h, int heads, int d, int t, const tp_shard* Wqkv,
                          const void* const* bqkv, const tp_shard* Wo, const void* bo, const void* residual,
                          int causal, void* out, tp_reduce_mode mode, void* ws, size_t ws_bytes,
                          tp_stream_t stream);

/* ------------------------------------------------------------------ attention sub-layer, backward pass
 * Gradients of tp_attn_forward's output for the upstream gradient dY, by the
 * chain rule read with [TP-CR]'s column/row pairing (paragraphs on multi-head
 * attention and head independence): the output projection is row-parallel, so
 * its input gradient dO_i = dY Wo_i^T is local to head group i; each head's
 * attention gradients depend on that head only; the QKV projection is
 * column-parallel, so its input gradient dX = sum_i dQKV_i Wqkv_i^T is the
 * backward pass's one sum over groups (taken in one accumulator).
 *
 *   Q, K, V = X Wqkv_i (+ bqkv_i), O = attention(Q, K, V)   (recomputed from X,
 *                                      with each softmax row's log-sum-exp)
 *   dWo_i = O_i^T dY,   dbo = column sums of dY,   dO_i = dY Wo_i^T
 *   per head: P = softmax rows, dV = P^T dO, dP = dO V^T,
 *             dS = P * (dP - rowsum(dO * O)), dQ = dS K / sqrt(d), dK = dS^T Q / sqrt(d)
 *   dWqkv_i = X^T dQKV_i,   dbqkv_i = column sums of dQKV_i   (dQKV_i = [dQ | dK | dV] of group i)
 *   dX = sum_i dQKV_i Wqkv_i^T (+ dX_add)
 *
 *  X, Wqkv, bqkv, Wo, causal  as in tp_attn_forward, bf16 only (TP_BF16 shards).
 *  dY       [B*S, h] bf16, contiguous.
 *  dX_add   [B*S, h] bf16 or NULL, added to dX (pass dY when the forward's
 *           residual was X).
 *  dX       [B*S, h] bf16 out; must not alias X, dY or dX_add.
 *  dWqkv    [h, 3*heads*d] fp32 out, contiguous: group i's gradient is the column
 *           block [i*3*Hg*d, (i+1)*3*Hg*d) in Wqkv[i]'s [Q | K | V] order.
 *  dbqkv    [3*heads*d] fp32 out or NULL, same column order.
 *  dWo      [heads*d, h] fp32 out, contiguous: group i's rows [i*Hg*d, (i+1)*Hg*d).
 *  dbo      [h] fp32 out or NULL.
 *  ws       tp_attn_backward_workspace_bytes(...) bytes, 256-byte aligned: Q, K, V,
 *           O (fp16 / bf16), dO (fp16), dQKV (bf16), the rows' log-sum-exp and
 *           rowsum(dO * O) (fp32).
 * The attention gradients' tensor-core operands (P, dS, dO, Q, K, V) are fp16
 * with fp32 accumulation; a P or dS value above 65504 sets TP_ERR_RANGE.  The
 * sums over rows, key blocks, query blocks and groups run in a fixed order:
 * results are bitwise reproducible on devices with the same SM count.  B*S == 0
 * zeroes dWqkv, dbqkv, dWo, dbo.  Limits: d == 128, heads % t == 0, S <= 65535*128
 * (else TP_ERR_UNSUPPORTED).
 */
TP_API size_t tp_attn_backward_workspace_bytes(int B, int S, int h, int heads, int d, int t);
TP_API tp_status tp_attn_backward(const void* X, int B, int S, int h, int heads, int d, int t,
                                  const tp_shard* Wqkv, const void* const* bqkv, const tp_shard* Wo,
                                  const void* dY, const void* dX_add, int causal, void* dX, float* dWqkv,
                                  float* dbqkv, float* dWo, float* dbo, void* ws, size_t ws_bytes,
                                  tp_stream_t stream);

/* ------------------------------------------------------------------ pre-LN layer
 * [TP-CR], the paragraph on two reductions per layer, in pre-LN order:
 *   h1  = X + Attn(LN1(X))            (h1 kept in fp32 inside the workspace)
 *   out = h1 + FFN(LN2(h1))           (bf16)
 * LayerNorm runs replicated over the full row ([TP-CR], feature reductions).
 * Weights as in tp_attn_forward and tp_ffn_forward, except that every weight
 * may be TP_BF16 or TP_FP16: LN1's output takes Wqkv's type, O takes Wo's, LN2's
 * output takes W1's and act(Z) takes W2's.  ln*_g / ln*_b are [h] bf16.
 */
TP_API size_t tp_layer_workspace_bytes(int B, int S, int h, int heads, int d, int64_t f, int t, tp_reduce_mode mode);
TP_API tp_status tp_layer_forward(const void* X, int B, int S, int h, int heads, int d, int64_t f, int t,
                           const void* ln1_g, const void* ln1_b, const tp_shard* Wqkv, const void* const* bqkv,
                           const tp_shard* Wo, const void* bo, const void* ln2_g, const void* ln2_b,
                           const tp_shard* W1, const void* const* b1, const tp_shard* W2, const void* b2, float eps,
                           int causal, void* out, tp_reduce_mode mode, void* ws, size_t ws_bytes,
                           tp_stream_t stream);

/* ------------------------------------------------------------------ building blocks
 * LayerNorm over rows: y = (x - mean) / sqrt(var + eps) * gamma + beta, var the
 * biased variance.  x [M, h] bf16 or fp32 (in_dtype); gamma, beta [h] bf16 or
 * NULL (1 and 0); y [M, h] in out_dtype (TP_BF16 or TP_FP16).  h % 8 == 0. */
TP_API tp_status tp_layernorm_forward(const void* x, tp_dtype in_dtype, const void* gamma, const void* beta, int64_t M,
                               int64_t h, float eps, void* y, tp_dtype out_dtype, tp_stream_t stream);

/* The element-wise nonlinearity of step 1 alone ([TP-CR], the paragraph on
 * where the nonlinearity fits), exactly as the column layer's epilogue applies
 * it: y[i] = act(x[i]) for fp32 x, y of n elements (may alias).  GeLU is the
 * exact z*Phi(z) with erfc from the published approximation of Numerical Recipes
 * (fractional error < 1.2e-7); in fp32 within 4e-7 absolute of the exact value. */
TP_API tp_status tp_activation_forward(const float* x, float* y, int64_t n, tp_activation act, tp_stream_t stream);

/* Step 3 alone: out = sum_{i<t} P[i] + bias + residual in fixed order i = 0..t-1.
 * P [t, M, h] fp32 contiguous; bias [h] and residual [M, h] in `dtype` or NULL;
 * out [M, h] in `dtype`.  h % 4 == 0. */
TP_API tp_status tp_reduce_partials(const float* P, int t, int64_t M, int64_t h, const void* bias, const void* residual,
                             tp_dtype dtype, void* out, tp_stream_t stream);

/* ------------------------------------------------------------------ status, limits, tracing */
/* Synchronise `stream`, then read and clear the device status word of the
 * current device.  TP_ERR_TIMEOUT if a device wait ran out since the last call;
 * else TP_ERR_RANGE if a value that a kernel stored in an fp16 intermediate
 * (act(Z) of an fp16 W2, Q/K/V, O of an fp16 Wo, a LayerNorm output of an fp16
 * weight) had a magnitude above 65504, the largest fp16 number: such a value is
 * stored as +-inf, and tp_last_error() names the intermediate.  The check costs
 * one max per stored value and never stops a kernel.  bf16 intermediates have
 * fp32's range and are not checked.  TP_ERR_CUDA if the synchronisation itself
 * failed.  The status word's address is looked up once per device; resetting a
 * device (cudaDeviceReset) that the library has used is not supported. */
TP_API tp_status tp_get_device_status(tp_stream_t stream);

/* Time limit of every device-side wait, in nanoseconds (default 2e9). */
TP_API void tp_set_wait_limit_ns(uint64_t ns);

/* Launch a one-CTA kernel that waits on a barrier nothing ever completes, with
 * the given limit.  It must return and leave TP_ERR_TIMEOUT in the status word. */
TP_API tp_status tp_selftest_bounded_wait(uint64_t limit_ns, tp_stream_t stream);

/* Optional launch trace of the calling thread: while enabled, each kernel the
 * library launches is bracketed by two CUDA events on its stream (at most
 * `capacity` launches are kept).  After synchronising, tp_trace_get returns the
 * kernel name and its event-timed duration in ms. */
TP_API tp_status tp_trace_enable(int capacity);
TP_API void tp_trace_disable(void);
TP_API int tp_trace_count(void);
TP_API tp_status tp_trace_get(int i, const char** name, float* ms);

TP_API const char* tp_status_string(tp_status s);
TP_API const char* tp_last_error(void);
TP_API int tp_version(void);

#ifdef __cplusplus
}
#endif
#endif /* TPBLOCK_H */
