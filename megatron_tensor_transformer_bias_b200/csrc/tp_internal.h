// Internal launch interface between the C-ABI layer (tp_api.cu) and the kernels.
// Host-only types; nothing here is part of the public ABI.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>
#include <cstddef>

#include "../../include/tpblock.h"

namespace tpb {

// Device status word.  Low byte: the code of the first failure (DEV_TIMEOUT), next
// byte: where that wait gave up.  Bits 16..19: a value that an epilogue was about to
// store in fp16 exceeded the largest fp16 number (65504), one bit per producing site;
// these are OR-ed in and do not stop the kernel.
enum : uint32_t { DEV_OK = 0, DEV_TIMEOUT = 5 };
enum : uint32_t {
  DEV_RANGE_COLUMN = 1u << 16,   // column layer output (act(Z) or a column linear), fp16
  DEV_RANGE_QKV = 1u << 17,      // Q, K, V of the attention projection (always fp16)
  DEV_RANGE_ATTN_O = 1u << 18,   // attention output O, fp16
  DEV_RANGE_LAYERNORM = 1u << 19,  // LayerNorm output, fp16
  DEV_RANGE_ATTN_GRAD = 1u << 20,  // attention backward: P^T, dS (fp16 tensor-memory operands)
  DEV_RANGE_MASK = 0x1Fu << 16
};
constexpr float FP16_MAX = 65504.0f;
enum : uint32_t {
  WAIT_SITE_PRODUCER = 1, WAIT_SITE_MMA_FULL = 2, WAIT_SITE_MMA_ACC = 3,
  WAIT_SITE_EPILOGUE = 4, WAIT_SITE_SELFTEST = 5, WAIT_SITE_ATTN = 6
};

// GEMM tile shape of the tcgen05 kernel (one CTA per SM, persistent).
constexpr int GEMM_BM = 128;
constexpr int GEMM_BN = 256;
constexpr int GEMM_BK = 64;

enum GemmEpilogue : int {
  EPI_ACT = 0,         // out[:, g*ncol + n] = act(acc + bias_g[n])            (column-parallel layer)
  EPI_PARTIAL_F32 = 1, // P[g][m, n] = acc as fp32                              (row layer, partials)
  EPI_BIAS_RESID = 2,  // out[m, n] = acc + bias[n] + resid[m, n]              (row layer, fused reduce)
  EPI_QKV = 3,         // scatter acc (+ bias_g) to Q/K/V [B, H, S, d] fp16     (QKV column layer)
  EPI_ACT_GRAD = 4,    // z = acc + bias_g: out = act(z) (16-bit), out2 = act'(z) (fp16)  (backward recompute)
  EPI_MUL_GRAD = 5,    // out[:, g*ncol + n] = acc * grad_mul[:, g*ncol + n] (fp16 factor)  (backward dZ)
};

// Element type of an epilogue output.
enum OutType : int { OUT_BF16 = 0, OUT_F32 = 1, OUT_F16 = 2 };

enum Activation : int { ACT_NONE = 0, ACT_GELU = 1, ACT_RELU = 2 };

struct __align__(64) GemmArgs {
  // Output of the TMA-store epilogues: 16-bit [rows, cols], box {32, 32}; or, for
  // EPI_PARTIAL_F32, fp32 (cols, rows, group), box {16, 32, 1}.  64B swizzle.
  CUtensorMap tmOut;
  // EPI_ACT_GRAD: act'(z) output (fp16); partials mode with the in-GEMM reduction: the bf16
  // output [M, N].  Box {32, 32}, 64B swizzle.
  CUtensorMap tmOut2;
  // A [M, Ktot] K-major: box {64 K, 128 M}; or (a_mn) the matrix [Ktot, M] with M
  // contiguous: a make_tmap_mn map (box {64 M, 64 K, 2 blocks}).  128B swizzle.
  CUtensorMap tmA;
  // B_g [Kg, N] N-major: a make_tmap_mn map (box {64 N, 64 K, 2 blocks}); or (b_kmajor) the
  // matrix [N, Kg] with K contiguous: box {64 K, 128 N}.  128B swizzle.
  CUtensorMap tmB[TP_MAX_SHARDS];
  int M, N, Kg, G;
  int concat;                           // 1: one tile sums all G K-slices in order g = 0..G-1
  int a_k_per_group;                    // column offset of group g's K-slice in A (elements)
  int a_m_per_group;                    // a_mn: M offset of group g's rows in A's map (elements)
  int a_mn;                             // A is M-major (the transpose of a row-major [K, M] matrix)
  int b_kmajor;                         // B is K-major (the transpose of a row-major [N, K] matrix)
  int epi, act;
  int ab_f16;                           // A and B operands are fp16 (else bf16)
  void* out;
  int64_t ld_out;                       // elements
  int64_t out_col_per_group;            // EPI_ACT_BF16: column offset of group g in out
  int64_t out_group_stride;             // EPI_PARTIAL_F32: elements between partials
  int out_type;                         // OutType of EPI_ACT / EPI_BIAS_RESID
  int tma_store;                        // 1: 16-bit EPI_ACT / EPI_BIAS_RESID output leaves through tmOut
  const void* bias_g[TP_MAX_SHARDS];    // bf16 [N] per group, or null
  const void* bias;                     // bf16 [N] or null (EPI_BIAS_RESID)
  const void* resid;                    // [M, N] or null
  int64_t ld_resid;
  int resid_fp32;
  // EPI_MUL_GRAD: fp16 factor [M, ld_grad] read at the output's column
  const void* grad_mul;
  int64_t ld_grad;
  // EPI_QKV scatter: column c of group g -> part c / (Hg*d), head g*Hg + (c % (Hg*d)) / d
  void* q; void* k; void* v;
  int S, H, Hg, d;
  // EPI_PARTIAL_F32 with the reduction in the epilogue (red_out != null): one arrival
  // counter per 32-row x 128-column region of the output, zero on entry.  The epilogue
  // warp whose arrival completes a region's G partials sums them in order g = 0..G-1,
  // adds bias and resid and writes red_out [M, N] (fp32 if red_out_f32, else bf16).
  uint32_t* counters;
  void* red_out;
  int red_out_f32;
  uint32_t* status;
  uint64_t wait_limit_ns;
};

// Arrival counters of the in-epilogue reduction: one per 32-row x 128-column region.
inline size_t partial_counter_count(int64_t M, int64_t N) { return static_cast<size_t>((M + 31) / 32) * ((N + 127) / 128); }

struct AttnArgs {
  CUtensorMap tmQ;   // Q [B*H][S][d] fp16, box {64, 128, 1}, 128B swizzle
  CUtensorMap tmK;   // K [B*H][S][d] fp16, box {64, 64, 1}
  CUtensorMap tmV;   // V [B*H][S][d] fp16, box {64, 64, 1}
  void* O;           // O [B*S, H*d] (head-major columns), bf16 or fp16
  int o_f16;
  int B, S, H, d, causal;
  int head0;         // first head handled (head-group offset)
  float scale_log2;  // log2(e) / sqrt(d)
  // Optional: per-row log2-sum-exp of the scaled scores, lse[(b*H + head) * lse_ld + s]
  // (rows s < S only), so that exp2(s * scale_log2 - lse) is the softmax row.
  float* lse;
  int lse_ld;
  uint32_t* status;
  uint64_t wait_limit_ns;
};

// Attention backward (tp_attention_bwd.cu).  Q, K, V [B*H][S][d] fp16; dO [B*S, H*d] fp16
// as a 4-D map (d, H, S, B).  Maps of the resident 128-row tiles (box rows 128): tmQ, tmdO
// (the dQ kernel), tmK, tmV (the dK/dV kernel); of the streamed 64-row sub-blocks (box rows
// 64): tmQs, tmdOs (dK/dV), tmKs, tmVs (dQ).  lse and Dv [B*H][S_pad] fp32 (S_pad = S
// rounded up to 128); dqkv [B*S, ld_dqkv] bf16, head group g's columns [g*3*Hg*d, ...) =
// [dQ heads | dK heads | dV heads].
struct AttnBwdArgs {
  CUtensorMap tmQ, tmK, tmV, tmdO;
  CUtensorMap tmQs, tmKs, tmVs, tmdOs;
  CUtensorMap tmOut;   // dqkv seen as (3*H*d, S, B) bf16, box {64, 128, 1}: the gradient blocks' TMA stores
  float* lse;
  float* Dv;
  uint16_t* dqkv;
  int64_t ld_dqkv;
  int B, S, H, Hg, head0, causal, S_pad;
  float scale_log2;  // log2(e) / sqrt(d)
  float scale;       // 1 / sqrt(d)
  uint32_t* status;
  uint64_t wait_limit_ns;
};

// Per-device runtime facts.
int sm_count();
uint32_t* device_status_ptr();
uint64_t wait_limit_ns();

// Tensor-map construction (driver entry point fetched through the runtime).
// 2-byte element tensor maps (bf16 or fp16), 128-byte swizzle, zero fill out of bounds.
tp_status make_tmap_2d(CUtensorMap* map, const void* base, int f16, uint64_t inner, uint64_t outer,
                       uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer);
// Map of an MN-major operand ([k_rows, mn_cols] row-major, MN contiguous, mn_cols % 64 == 0):
// 3-D view (64, k_rows, mn_cols / 64), box {64, 64, 2}: one load brings two 64-wide MN
// blocks of 64 K rows, 8 KB apart in shared memory.  128-byte swizzle, zero fill.
tp_status make_tmap_mn(CUtensorMap* map, const void* base, int f16, uint64_t mn_cols, uint64_t k_rows,
                       uint64_t row_stride_bytes);
// Output map of the epilogue stores: box {32, 32} of a 2-byte type, 64-byte swizzle.
tp_status make_tmap_out(CUtensorMap* map, void* base, int f16, uint64_t cols, uint64_t rows,
                        uint64_t row_stride_bytes);

// Kernel launchers.  All are asynchronous on `stream` and validate nothing:
// the C-ABI layer has checked every argument before calling them.
tp_status launch_gemm(const GemmArgs& a, cudaStream_t stream, const char* name);
tp_status launch_attention(const AttnArgs& a, cudaStream_t stream);
// Rows of the K and V tensor-map boxes: the key-block size of the attention kernel in use.
int attention_kv_rows();
// D = rowsum(dO * O) (and the padding rows of D / lse), then dK, dV and dQ into a.dqkv.
tp_status launch_attention_backward(const AttnBwdArgs& a, const uint16_t* dO, const uint16_t* O, int o_f16,
                                    cudaStream_t stream);
tp_status launch_reduce_partials(const float* P, int t, int64_t M, int64_t h, const void* bias, int bias_fp32,
                                 const void* resid, int resid_fp32, void* out, int out_fp32,
                                 cudaStream_t stream);
tp_status launch_layernorm(const void* x, int in_fp32, const void* g, const void* b, int64_t M, int64_t h,
                           float eps, void* y, int out_f16, cudaStream_t stream);
tp_status launch_ffn_fp32(const float* X, int64_t M, int64_t h, int64_t f, int t, const tp_shard* W1,
                          const void* const* b1, const tp_shard* W2, const float* b2, const float* resid,
                          float* out, int act, float* Z, float* P, cudaStream_t stream);
tp_status launch_selftest_wait(uint64_t limit_ns, cudaStream_t stream);
// out[c] = sum_r x[r, c] (bf16 x [M, ld], fp32 out [n]) in a fixed order, one pass, no scratch.
tp_status launch_colsum(const void* x, int64_t M, int64_t n, int64_t ld, float* out, cudaStream_t stream);
tp_status launch_act(const float* x, float* y, int64_t n, int act, cudaStream_t stream);

// Record `msg` as the calling thread's tp_last_error() and return `s`.
tp_status set_error(tp_status s, const char* msg);
// Whether launches carry the programmatic-dependent-launch attribute (TPB_PDL=0: no).
bool pdl_enabled();
// Launch `kern` on `stream` with programmatic dependent launch (the kernel waits for
// its predecessor with griddepcontrol.wait before touching global memory) and an
// optional cluster size.
template <typename... KArgs, typename... Args>
tp_status launch_ex(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream, int cluster_x,
                    Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  int n = 0;
  if (cluster_x > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  if (pdl_enabled()) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = n;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, static_cast<Args&&>(args)...);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(TP_ERR_CUDA, cudaGetErrorString(e));
  return TP_OK;
}


// Launch tracing (tp_trace_*): brackets each kernel launch with events.
void trace_before(cudaStream_t stream, const char* name);
void trace_after(cudaStream_t stream, const char* name);

}  // namespace tpb
