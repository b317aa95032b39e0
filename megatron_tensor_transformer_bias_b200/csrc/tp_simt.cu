// HBM-bound and small kernels of the block:
//  * reduce_partials: step 3 of "Tensor Parallelism > Combining Column and Row
//    Parallelism" on one device -- out = sum_i P_i + bias + residual, shards
//    summed in the fixed order 0..t-1, 128-bit loads, grid-stride over the SMs;
//  * layernorm: the replicated LayerNorm over the full row (the page's paragraph
//    on feature reductions: mean and variance need every feature), one CTA per
//    row, row cached in shared memory, warp-shuffle reductions;
//  * the exact-fp32 FFN (FFMA, no TF32) used for fp32 inputs;
//  * column sums in a fixed order (the bias gradients of the backward pass);
//  * the bounded-wait self-test kernel.
#include "tp_internal.h"
#include "tp_ptx.cuh"

namespace tpb {

#define TP_TRY_LAUNCH(expr)            \
  do {                                 \
    tp_status _s = (expr);             \
    if (_s != TP_OK) return _s;        \
  } while (0)

namespace {

// ---------------------------------------------------------------- reduce
template <bool F32>
__device__ __forceinline__ float4 load4(const void* p, int64_t e) {
  if (F32) return __ldg(reinterpret_cast<const float4*>(static_cast<const float*>(p) + e));
  const uint2 u = __ldg(reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(p) + e));
  return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u), __uint_as_float(u.y << 16),
                     __uint_as_float(u.y & 0xFFFF0000u));
}

template <bool OUT_F32, bool RESID_F32, bool BIAS_F32>
__global__ void __launch_bounds__(256) reduce_partials_kernel(const float* __restrict__ P, int t, int64_t MH,
                                                              const void* __restrict__ bias, int64_t h,
                                                              const void* __restrict__ resid,
                                                              void* __restrict__ out) {
  const int64_t nvec = MH / 4;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  pdl_wait();
  for (int64_t v = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; v < nvec; v += stride) {
    const int64_t e = v * 4;
    // fixed shard order 0..t-1
    float4 acc = __ldcs(reinterpret_cast<const float4*>(P) + v);
    for (int i = 1; i < t; ++i) {
      const float4 p = __ldcs(reinterpret_cast<const float4*>(P + static_cast<int64_t>(i) * MH) + v);
      acc.x += p.x; acc.y += p.y; acc.z += p.z; acc.w += p.w;
    }
    if (bias) {
      const float4 b = load4<BIAS_F32>(bias, e % h);
      acc.x += b.x; acc.y += b.y; acc.z += b.z; acc.w += b.w;
    }
    if (resid) {
      const float4 r = load4<RESID_F32>(resid, e);
      acc.x += r.x; acc.y += r.y; acc.z += r.z; acc.w += r.w;
    }
    if (OUT_F32) {
      *reinterpret_cast<float4*>(static_cast<float*>(out) + e) = acc;
    } else {
      uint2 o;
      o.x = pack_bf16x2(acc.x, acc.y);
      o.y = pack_bf16x2(acc.z, acc.w);
      *reinterpret_cast<uint2*>(static_cast<uint16_t*>(out) + e) = o;
    }
  }
  pdl_launch_dependents();
}

// ---------------------------------------------------------------- layernorm
constexpr int LN_THREADS = 256;

// 8 consecutive bf16 values (16-byte aligned) as floats
__device__ __forceinline__ void load_bf16x8(const uint16_t* p, float (&f)[8]) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    f[2 * j] = __uint_as_float(w[j] << 16);
    f[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x / 32, l = threadIdx.x % 32;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < LN_THREADS / 32; ++i) s += red[i];
  return s;
}

template <bool IN_F32, bool OUT_F16>
__global__ void __launch_bounds__(LN_THREADS) layernorm_kernel(const void* __restrict__ x,
                                                               const uint16_t* __restrict__ g,
                                                               const uint16_t* __restrict__ b, int64_t h,
                                                               float eps, uint16_t* __restrict__ y,
                                                               uint32_t* status) {
  extern __shared__ float row[];
  __shared__ float red[LN_THREADS / 32];
  const int64_t r = blockIdx.x;
  const int64_t n8 = h / 8;
  float s = 0.f;
  pdl_wait();
  for (int64_t v = threadIdx.x; v < n8; v += LN_THREADS) {
    float f[8];
    if (IN_F32) {
      const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(x) + r * h) + 2 * v;
      const float4 a = __ldcs(p), c = __ldcs(p + 1);
      f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = c.x; f[5] = c.y; f[6] = c.z; f[7] = c.w;
    } else {
      const uint4 u = __ldcs(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(x) + r * h) + v);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        f[2 * j] = __uint_as_float(w[j] << 16);
        f[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
      }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      row[v * 8 + j] = f[j];
      s += f[j];
    }
  }
  const float mean = block_sum(s, red) / static_cast<float>(h);
  float q = 0.f;
  for (int64_t i = threadIdx.x; i < h; i += LN_THREADS) {
    const float d = row[i] - mean;
    q += d * d;
  }
  const float var = block_sum(q, red) / static_cast<float>(h);
  const float rstd = rsqrtf(var + eps);
  for (int64_t v = threadIdx.x; v < n8; v += LN_THREADS) {
    float o[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int64_t c = v * 8 + j;
      const float gg = g ? bf16_bits_to_float(g[c]) : 1.f;
      const float bb = b ? bf16_bits_to_float(b[c]) : 0.f;
      o[j] = (row[c] - mean) * rstd * gg + bb;
    }
    uint4 u;
    if (OUT_F16) {
      float m = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(o[j]));
      note_f16_range(status, m, DEV_RANGE_LAYERNORM);
      u.x = pack_f16x2(o[0], o[1]);
      u.y = pack_f16x2(o[2], o[3]);
      u.z = pack_f16x2(o[4], o[5]);
      u.w = pack_f16x2(o[6], o[7]);
    } else {
      u.x = pack_bf16x2(o[0], o[1]);
      u.y = pack_bf16x2(o[2], o[3]);
      u.z = pack_bf16x2(o[4], o[5]);
      u.w = pack_bf16x2(o[6], o[7]);
    }
    reinterpret_cast<uint4*>(y + r * h)[v] = u;
  }
  pdl_launch_dependents();
}

// ---------------------------------------------------------------- exact fp32 FFN
constexpr int SG = 16;

struct F32ShardPtrs {
  const float* B[TP_MAX_SHARDS];
  int64_t ldb[TP_MAX_SHARDS];
  const float* bias[TP_MAX_SHARDS];
};

// C_z[M, N] = act(A_z[M, K] B_z[K, N] + bias_z) for shard z = blockIdx.z.
// A_z = A + z * a_col_step (columns), C_z = C + z * c_col_step (columns) + z * c_mat_step.
__global__ void __launch_bounds__(SG * SG) f32_gemm_kernel(const float* __restrict__ A, int64_t lda,
                                                           int64_t a_col_step, F32ShardPtrs sp, float* C,
                                                           int64_t ldc, int64_t c_col_step, int64_t c_mat_step,
                                                           int M, int N, int K, int act) {
  __shared__ float As[SG][SG + 1];
  __shared__ float Bs[SG][SG + 1];
  const int z = blockIdx.z;
  const float* Az = A + z * a_col_step;
  const float* Bz = sp.B[z];
  const int64_t ldb = sp.ldb[z];
  const int row = blockIdx.y * SG + threadIdx.y;
  const int col = blockIdx.x * SG + threadIdx.x;
  float acc = 0.f;
  for (int k0 = 0; k0 < K; k0 += SG) {
    const int ka = k0 + threadIdx.x, kb = k0 + threadIdx.y;
    As[threadIdx.y][threadIdx.x] = (row < M && ka < K) ? Az[static_cast<int64_t>(row) * lda + ka] : 0.f;
    Bs[threadIdx.y][threadIdx.x] = (kb < K && col < N) ? Bz[static_cast<int64_t>(kb) * ldb + col] : 0.f;
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < SG; ++kk) acc = fmaf(As[threadIdx.y][kk], Bs[kk][threadIdx.x], acc);
    __syncthreads();
  }
  if (row < M && col < N) {
    if (sp.bias[z]) acc += sp.bias[z][col];
    acc = act_apply(acc, act);
    C[z * c_mat_step + z * c_col_step + static_cast<int64_t>(row) * ldc + col] = acc;
  }
}

// ---------------------------------------------------------------- element-wise nonlinearity
__global__ void __launch_bounds__(256) act_kernel(const float* __restrict__ x, float* __restrict__ y, int64_t n,
                                                  int act) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    y[i] = act_apply(x[i], act);
}

// ---------------------------------------------------------------- column sums
// out[c] = sum over rows of x[r, c] for a bf16 x [M, ld], in a fixed order: pass 1 gives
// each 128-row chunk's sum per column (warp w of a CTA adds the chunk's rows w, w + 8, ...
// in turn, then the 8 warps' sums are added in the order 0..7); pass 2 adds the chunks'
// sums in the order 0, 1, ...  Each thread of pass 1 owns 8 adjacent columns (one
// 16-byte load per row), so a warp reads 512 contiguous bytes of a row.
// Column sums of a bf16 [M, n] matrix (row stride ld) in one launch: a cluster of 8 CTAs owns
// 128 columns, CTA q of it the rows [q R, (q + 1) R) with R = ceil(M / 8); in a CTA, row slot
// k = 2 w + (lane / 16) of warp w reads rows k, k + 16, ... of its range (256 contiguous
// bytes per row, 8 columns per lane) and sums them in increasing order; the 16 slots' sums
// add up in order 0..15, and CTA 0 of the cluster adds the 8 CTAs' sums in order 0..7 through
// distributed shared memory.  Fixed order throughout: the result does not depend on timing.
constexpr int CS_COLS = 128;    // 16 lanes x 8 columns
constexpr int CS_SLOTS = 16;    // rows read at once by a CTA: 8 warps x 2
constexpr int CS_SPLIT = 8;     // CTAs (row ranges) per cluster
__global__ void __launch_bounds__(256) colsum_kernel(const uint16_t* __restrict__ x, int64_t M, int64_t n,
                                                     int64_t ld, float* __restrict__ out) {
  __shared__ float red[CS_SLOTS][CS_COLS];
  __shared__ float psum[CS_COLS];
  const int slot = threadIdx.x / 16, l16 = threadIdx.x % 16;
  const uint32_t q = cluster_ctarank();
  const int64_t cb = blockIdx.x / CS_SPLIT;
  const int64_t c0 = cb * CS_COLS + l16 * 8;
  const int64_t rows = (M + CS_SPLIT - 1) / CS_SPLIT;
  const int64_t r_lo = static_cast<int64_t>(q) * rows;
  const int64_t r_hi = r_lo + rows < M ? r_lo + rows : M;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  pdl_wait();
  if (c0 < n) {
    // eight rows' loads in flight per thread (32 KB per CTA), then their adds in row order
    int64_t r = r_lo + slot;
    for (; r + 7 * CS_SLOTS < r_hi; r += 8 * CS_SLOTS) {
      uint4 u[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) u[k] = __ldg(reinterpret_cast<const uint4*>(x + (r + k * CS_SLOTS) * ld + c0));
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint32_t w[4] = {u[k].x, u[k].y, u[k].z, u[k].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc[2 * j] += __uint_as_float(w[j] << 16);
          acc[2 * j + 1] += __uint_as_float(w[j] & 0xFFFF0000u);
        }
      }
    }
    for (; r < r_hi; r += CS_SLOTS) {
      float f[8];
      load_bf16x8(x + r * ld + c0, f);
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[j] += f[j];
    }
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) red[slot][l16 * 8 + j] = acc[j];
  __syncthreads();
  if (threadIdx.x < CS_COLS) {
    float v = red[0][threadIdx.x];
#pragma unroll
    for (int i = 1; i < CS_SLOTS; ++i) v += red[i][threadIdx.x];
    psum[threadIdx.x] = v;
  }
  cluster_sync_all();   // every CTA's psum is written and visible to the cluster
  if (q == 0 && threadIdx.x < CS_COLS) {
    const int64_t c = cb * CS_COLS + threadIdx.x;
    if (c < n) {
      float v = psum[threadIdx.x];
      const uint32_t own = smem_u32(&psum[threadIdx.x]);
#pragma unroll
      for (uint32_t k = 1; k < CS_SPLIT; ++k) {
        float pk;
        asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(pk) : "r"(mapa_shared(own, k)) : "memory");
        v += pk;
      }
      out[c] = v;
    }
  }
  cluster_sync_all();   // the other CTAs' shared memory stays until CTA 0 has read it
  pdl_launch_dependents();
}

// ---------------------------------------------------------------- self-test
__global__ void selftest_wait_kernel(uint64_t limit_ns, uint32_t* status) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // Nothing ever arrives on `bar`: the wait must run out and report it.
    mbar_wait_bounded(&bar, 0, limit_ns, status, WAIT_SITE_SELFTEST);
  }
  __syncthreads();
}

}  // namespace

tp_status launch_reduce_partials(const float* P, int t, int64_t M, int64_t h, const void* bias, int bias_fp32,
                                 const void* resid, int resid_fp32, void* out, int out_fp32, cudaStream_t stream) {
  const int64_t nvec = M * h / 4;
  if (nvec == 0) return TP_OK;
  int64_t blocks = (nvec + 255) / 256;
  const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
  if (blocks > cap) blocks = cap;
  const int g = static_cast<int>(blocks);
  const int key = (out_fp32 ? 4 : 0) | (resid_fp32 ? 2 : 0) | (bias_fp32 ? 1 : 0);
  trace_before(stream, "reduce_partials");
  tp_status st = TP_OK;
  switch (key) {
#define TP_REDUCE_CASE(K, O, R, B)                                                                              \
    case K:                                                                                                    \
      st = launch_ex(reduce_partials_kernel<O, R, B>, dim3(g), dim3(256), 0, stream, 1, P, t, M * h, bias, h, \
                     resid, out);                                                                              \
      break;
    TP_REDUCE_CASE(0, false, false, false)
    TP_REDUCE_CASE(1, false, false, true)
    TP_REDUCE_CASE(2, false, true, false)
    TP_REDUCE_CASE(3, false, true, true)
    TP_REDUCE_CASE(4, true, false, false)
    TP_REDUCE_CASE(5, true, false, true)
    TP_REDUCE_CASE(6, true, true, false)
    TP_REDUCE_CASE(7, true, true, true)
#undef TP_REDUCE_CASE
  }
  if (st != TP_OK) return st;
  trace_after(stream, "reduce_partials");
  return TP_OK;
}

// Register-resident LayerNorm for h <= 2048 * NCH: one 256-thread CTA per row, thread i
// holds the 8-element chunks i, i + 256, ... (NCH of them) in registers.  Every load of
// the row is issued before the first reduction, the mean and the variance are taken in
// two exact passes over the registers, and gamma / beta are read 8 at a time.
template <bool IN_F32, bool OUT_F16, int NCH>
__global__ void __launch_bounds__(LN_THREADS) layernorm_reg_kernel(const void* __restrict__ x,
                                                                   const uint16_t* __restrict__ g,
                                                                   const uint16_t* __restrict__ b, int64_t h,
                                                                   float eps, uint16_t* __restrict__ y,
                                                                   uint32_t* status) {
  __shared__ float red[LN_THREADS / 32];
  const int64_t r = blockIdx.x;
  const int n8 = static_cast<int>(h / 8);
  float f[NCH][8];
  pdl_wait();
#pragma unroll
  for (int k = 0; k < NCH; ++k) {
    const int v = threadIdx.x + k * LN_THREADS;
    if (v < n8) {
      if (IN_F32) {
        const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(x) + r * h) + 2 * v;
        const float4 a = __ldcs(p), c = __ldcs(p + 1);
        f[k][0] = a.x; f[k][1] = a.y; f[k][2] = a.z; f[k][3] = a.w;
        f[k][4] = c.x; f[k][5] = c.y; f[k][6] = c.z; f[k][7] = c.w;
      } else {
        const uint4 u = __ldcs(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(x) + r * h) + v);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          f[k][2 * j] = __uint_as_float(w[j] << 16);
          f[k][2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
        }
      }
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) f[k][j] = 0.f;
    }
  }
  float s = 0.f;
#pragma unroll
  for (int k = 0; k < NCH; ++k)
#pragma unroll
    for (int j = 0; j < 8; ++j) s += f[k][j];
  const float mean = block_sum(s, red) / static_cast<float>(h);
  float q = 0.f;
#pragma unroll
  for (int k = 0; k < NCH; ++k) {
    if (threadIdx.x + k * LN_THREADS < n8) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float d = f[k][j] - mean;
        q += d * d;
      }
    }
  }
  const float var = block_sum(q, red) / static_cast<float>(h);
  const float rstd = rsqrtf(var + eps);
#pragma unroll
  for (int k = 0; k < NCH; ++k) {
    const int v = threadIdx.x + k * LN_THREADS;
    if (v >= n8) continue;
    float gg[8], bb[8];
    if (g) {
      load_bf16x8(g + 8 * static_cast<int64_t>(v), gg);
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) gg[j] = 1.f;
    }
    if (b) {
      load_bf16x8(b + 8 * static_cast<int64_t>(v), bb);
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) bb[j] = 0.f;
    }
    float o[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) o[j] = (f[k][j] - mean) * rstd * gg[j] + bb[j];
    uint4 u;
    if (OUT_F16) {
      float m = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(o[j]));
      note_f16_range(status, m, DEV_RANGE_LAYERNORM);
      u.x = pack_f16x2(o[0], o[1]); u.y = pack_f16x2(o[2], o[3]);
      u.z = pack_f16x2(o[4], o[5]); u.w = pack_f16x2(o[6], o[7]);
    } else {
      u.x = pack_bf16x2(o[0], o[1]); u.y = pack_bf16x2(o[2], o[3]);
      u.z = pack_bf16x2(o[4], o[5]); u.w = pack_bf16x2(o[6], o[7]);
    }
    reinterpret_cast<uint4*>(y + r * h)[v] = u;
  }
  pdl_launch_dependents();
}

template <int NCH>
static tp_status launch_layernorm_reg(const void* x, int in_fp32, const void* g, const void* b, int64_t M, int64_t h,
                                      float eps, void* y, int out_f16, cudaStream_t stream) {
  const int key = (in_fp32 ? 1 : 0) | (out_f16 ? 2 : 0);
  void (*kern)(const void*, const uint16_t*, const uint16_t*, int64_t, float, uint16_t*, uint32_t*) =
      key == 0   ? layernorm_reg_kernel<false, false, NCH>
      : key == 1 ? layernorm_reg_kernel<true, false, NCH>
      : key == 2 ? layernorm_reg_kernel<false, true, NCH>
                 : layernorm_reg_kernel<true, true, NCH>;
  trace_before(stream, "layernorm");
  const tp_status st = launch_ex(kern, dim3(static_cast<unsigned>(M)), dim3(LN_THREADS), 0, stream, 1, x,
                                 static_cast<const uint16_t*>(g), static_cast<const uint16_t*>(b), h, eps,
                                 static_cast<uint16_t*>(y), device_status_ptr());
  if (st != TP_OK) return st;
  trace_after(stream, "layernorm");
  return TP_OK;
}

tp_status launch_layernorm(const void* x, int in_fp32, const void* g, const void* b, int64_t M, int64_t h,
                           float eps, void* y, int out_f16, cudaStream_t stream) {
  if (M > 0 && h <= 8 * LN_THREADS * 4) {
    if (h <= 8 * LN_THREADS) return launch_layernorm_reg<1>(x, in_fp32, g, b, M, h, eps, y, out_f16, stream);
    if (h <= 8 * LN_THREADS * 2) return launch_layernorm_reg<2>(x, in_fp32, g, b, M, h, eps, y, out_f16, stream);
    return launch_layernorm_reg<4>(x, in_fp32, g, b, M, h, eps, y, out_f16, stream);
  }
  if (M == 0) return TP_OK;
  const size_t smem = static_cast<size_t>(h) * sizeof(float);
  const int key = (in_fp32 ? 1 : 0) | (out_f16 ? 2 : 0);
  void (*kern)(const void*, const uint16_t*, const uint16_t*, int64_t, float, uint16_t*, uint32_t*) =
      key == 0 ? layernorm_kernel<false, false>
               : key == 1 ? layernorm_kernel<true, false> : key == 2 ? layernorm_kernel<false, true>
                                                                     : layernorm_kernel<true, true>;
  static int attr_set[64][4] = {{0}};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return TP_ERR_CUDA;
  if (smem > 48 * 1024 && dev < 64 && !attr_set[dev][key]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024) != cudaSuccess)
      return TP_ERR_CUDA;
    attr_set[dev][key] = 1;
  }
  trace_before(stream, "layernorm");
  const tp_status st = launch_ex(kern, dim3(static_cast<unsigned>(M)), dim3(LN_THREADS), smem, stream, 1, x,
                                 static_cast<const uint16_t*>(g), static_cast<const uint16_t*>(b), h, eps,
                                 static_cast<uint16_t*>(y), device_status_ptr());
  if (st != TP_OK) return st;
  trace_after(stream, "layernorm");
  return TP_OK;
}

tp_status launch_ffn_fp32(const float* X, int64_t M, int64_t h, int64_t f, int t, const tp_shard* W1,
                          const void* const* b1, const tp_shard* W2, const float* b2, const float* resid,
                          float* out, int act, float* Z, float* P, cudaStream_t stream) {
  const int64_t fs = f / t;
  F32ShardPtrs s1{}, s2{};
  for (int i = 0; i < t; ++i) {
    s1.B[i] = static_cast<const float*>(W1[i].ptr);
    s1.ldb[i] = W1[i].ld;
    s1.bias[i] = b1 ? static_cast<const float*>(b1[i]) : nullptr;
    s2.B[i] = static_cast<const float*>(W2[i].ptr);
    s2.ldb[i] = W2[i].ld;
    s2.bias[i] = nullptr;
  }
  // Step 1: Z[:, i*fs:(i+1)*fs] = act(X W1_i + b1_i)
  dim3 blk(SG, SG);
  dim3 g1(static_cast<unsigned>((fs + SG - 1) / SG), static_cast<unsigned>((M + SG - 1) / SG), t);
  trace_before(stream, "f32_col_gemm");
  f32_gemm_kernel<<<g1, blk, 0, stream>>>(X, h, 0, s1, Z, f, fs, 0, static_cast<int>(M), static_cast<int>(fs),
                                          static_cast<int>(h), act);
  if (cudaGetLastError() != cudaSuccess) return TP_ERR_CUDA;
  trace_after(stream, "f32_col_gemm");
  // Step 2: P[i] = Z_i W2_i
  dim3 g2(static_cast<unsigned>((h + SG - 1) / SG), static_cast<unsigned>((M + SG - 1) / SG), t);
  trace_before(stream, "f32_row_gemm");
  f32_gemm_kernel<<<g2, blk, 0, stream>>>(Z, f, fs, s2, P, h, 0, M * h, static_cast<int>(M), static_cast<int>(h),
                                          static_cast<int>(fs), ACT_NONE);
  if (cudaGetLastError() != cudaSuccess) return TP_ERR_CUDA;
  trace_after(stream, "f32_row_gemm");
  // Step 3: out = sum_i P[i] + b2 + residual
  return launch_reduce_partials(P, t, M, h, b2, 1, resid, 1, out, 1, stream);
}

tp_status launch_act(const float* x, float* y, int64_t n, int act, cudaStream_t stream) {
  if (n == 0) return TP_OK;
  int64_t blocks = (n + 255) / 256;
  const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
  if (blocks > cap) blocks = cap;
  trace_before(stream, "activation");
  act_kernel<<<static_cast<int>(blocks), 256, 0, stream>>>(x, y, n, act);
  if (cudaGetLastError() != cudaSuccess) return TP_ERR_CUDA;
  trace_after(stream, "activation");
  return TP_OK;
}

tp_status launch_colsum(const void* x, int64_t M, int64_t n, int64_t ld, float* out, cudaStream_t stream) {
  if (n == 0) return TP_OK;
  if (M == 0) {
    const cudaError_t e = cudaMemsetAsync(out, 0, static_cast<size_t>(n) * sizeof(float), stream);
    return e == cudaSuccess ? TP_OK : set_error(TP_ERR_CUDA, cudaGetErrorString(e));
  }
  trace_before(stream, "colsum");
  TP_TRY_LAUNCH(launch_ex(colsum_kernel, dim3(static_cast<unsigned>((n + CS_COLS - 1) / CS_COLS * CS_SPLIT)),
                          dim3(256), 0, stream, CS_SPLIT, static_cast<const uint16_t*>(x), M, n, ld, out));
  trace_after(stream, "colsum");
  return TP_OK;
}

tp_status launch_selftest_wait(uint64_t limit_ns, cudaStream_t stream) {
  trace_before(stream, "selftest_wait");
  selftest_wait_kernel<<<1, 32, 0, stream>>>(limit_ns, device_status_ptr());
  if (cudaGetLastError() != cudaSuccess) return TP_ERR_CUDA;
  trace_after(stream, "selftest_wait");
  return TP_OK;
}

}  // namespace tpb
