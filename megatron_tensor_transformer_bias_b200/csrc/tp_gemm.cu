// Persistent warp-specialised tcgen05 GEMM for the column- and row-parallel linears.
//
//   C_g[M, N] = A[:, g*a_k_per_group : +Kg] (M x Kg, K-major) * B_g (Kg x N, N-major)
//
// Column-parallel layer ("Tensor Parallelism > Combining Column and Row
// Parallelism", step 1): one tile per (shard g, m-block, n-block); the
// epilogue adds the shard's bias and applies the element-wise nonlinearity
// straight from TMEM (no communication is needed, the nonlinearity is local).
// Row-parallel layer (steps 2-3): either one tile per (m-block, n-block) whose
// K loop walks the K-slices of all shards into the same TMEM accumulator (the
// reduction happens in the accumulator) with a bias + residual epilogue, or one
// tile per (shard, m, n) writing fp32 partials.
//
// Two kernels share the roles below: tp_gemm_pair_kernel (the default; a cluster
// of two CTAs computes a 256x256 tile, or a 256x512 one, with cta_group::2 MMAs) and
// tp_gemm_kernel (one CTA, 128x256 tiles).  Roles per CTA (320 threads, one CTA per SM):
//   warp 0      TMA producer: this CTA's operand tiles, one 64-wide K step per stage
//   warp 1      TMEM allocation; issues tcgen05.mma (16-deep K per instruction): in the
//               pair kernel the whole warp runs the loop and one lane is elected per
//               instruction, in the one-CTA kernel lane 0 issues
//   warps 2..9  epilogue: tcgen05.ld TMEM -> registers -> bias/act/residual -> global
//               (16-bit outputs through swizzled shared-memory staging and TMA stores)
// A shared-memory ring (6 stages of 32 KB for 256x256 pair tiles, 4 of 48 KB for 256x512,
// 4 for one CTA) feeds the MMA; with 256-column tiles two TMEM accumulators let the
// epilogue of one tile overlap the main loop of the next (a 256x512 tile's accumulator
// fills all 512 columns).
#include <cstdlib>

#include "tp_internal.h"
#include "tp_ptx.cuh"

namespace tpb {

namespace {

constexpr int BM = GEMM_BM, BN = GEMM_BN, BK = GEMM_BK;
constexpr int STAGES = 4;
constexpr int A_STAGE_BYTES = BM * BK * 2;          // 16 KB
constexpr int B_BLOCK_BYTES = 64 * BK * 2;          // 8 KB: 64 N-columns x 64 K-rows
constexpr int B_STAGE_BYTES = BN * BK * 2;          // 32 KB
constexpr int STAGE_BYTES = A_STAGE_BYTES + B_STAGE_BYTES;
constexpr int NUM_ACC = 2;
constexpr int TMEM_COLS = NUM_ACC * BN;             // 512
constexpr int EPI_WARPS = 8;                        // two per TMEM sub-partition, each owns half the columns
constexpr int THREADS = 64 + 32 * EPI_WARPS;        // warp 0 TMA, warp 1 MMA, warps 2..9 epilogue
constexpr int STAGING_BYTES = EPI_WARPS * 2 * 2048;   // two 32x32 16-bit buffers per epilogue warp
constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + STAGING_BYTES + 256;

// Operand layouts a kernel instantiation is compiled for (template parameter OPL).
constexpr int OPL_A_MN = 1;      // A M-major (the backward's weight gradients)
constexpr int OPL_B_KMAJOR = 2;  // B K-major (the backward's input gradients)

struct TileCoord {
  int g, m_blk, n_blk;
};

// Tile order: m fastest, then n, then the group -- so the pairs working at the same time
// share the group's B tiles through L2.
__device__ __forceinline__ TileCoord tile_coord(const GemmArgs& a, int tile, int m_tiles, int n_tiles) {
  TileCoord c;
  c.m_blk = tile % m_tiles;
  const int rest = tile / m_tiles;
  c.n_blk = rest % n_tiles;
  c.g = a.concat ? 0 : rest / n_tiles;
  return c;
}

__device__ __forceinline__ void load_bf16x32(const void* p, float (&v)[32]) {
  const uint4* q = reinterpret_cast<const uint4*>(p);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint4 u = __ldg(q + i);
    uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[i * 8 + j * 2] = __uint_as_float(w[j] << 16);
      v[i * 8 + j * 2 + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
    }
  }
}

__device__ __forceinline__ void load_f32x32(const void* p, float (&v)[32]) {
  const float4* q = reinterpret_cast<const float4*>(p);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float4 u = __ldg(q + i);
    v[i * 4] = u.x; v[i * 4 + 1] = u.y; v[i * 4 + 2] = u.z; v[i * 4 + 3] = u.w;
  }
}

__device__ __forceinline__ void store_bf16x32(void* p, const float (&v)[32]) {
  uint4* q = reinterpret_cast<uint4*>(p);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint4 u;
    u.x = pack_bf16x2(v[i * 8 + 0], v[i * 8 + 1]);
    u.y = pack_bf16x2(v[i * 8 + 2], v[i * 8 + 3]);
    u.z = pack_bf16x2(v[i * 8 + 4], v[i * 8 + 5]);
    u.w = pack_bf16x2(v[i * 8 + 6], v[i * 8 + 7]);
    q[i] = u;
  }
}

__device__ __forceinline__ void store_f16x32(void* p, const float (&v)[32]) {
  uint4* q = reinterpret_cast<uint4*>(p);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint4 u;
    u.x = pack_f16x2(v[i * 8 + 0], v[i * 8 + 1]);
    u.y = pack_f16x2(v[i * 8 + 2], v[i * 8 + 3]);
    u.z = pack_f16x2(v[i * 8 + 4], v[i * 8 + 5]);
    u.w = pack_f16x2(v[i * 8 + 6], v[i * 8 + 7]);
    q[i] = u;
  }
}

__device__ __forceinline__ void store_f32x32(void* p, const float (&v)[32]) {
  float4* q = reinterpret_cast<float4*>(p);
#pragma unroll
  for (int i = 0; i < 8; ++i) q[i] = make_float4(v[i * 4], v[i * 4 + 1], v[i * 4 + 2], v[i * 4 + 3]);
}

__device__ __forceinline__ void store_x32(void* base, int64_t idx, int out_type, const float (&v)[32]) {
  if (out_type == OUT_F32)
    store_f32x32(static_cast<float*>(base) + idx, v);
  else if (out_type == OUT_F16)
    store_f16x32(static_cast<uint16_t*>(base) + idx, v);
  else
    store_bf16x32(static_cast<uint16_t*>(base) + idx, v);
}

// Bias / nonlinearity / residual of one 32-column chunk for the epilogues whose
// 16-bit output leaves through a TMA store (EPI_ACT, EPI_BIAS_RESID).  Rows at or
// beyond M still run (their values are clipped by the store) but read no residual.
template <int EPI>
__device__ __forceinline__ void epilogue_math(const GemmArgs& a, const TileCoord& tc, int row, int n, float (&v)[32]) {
  const void* bias = EPI == EPI_ACT ? a.bias_g[tc.g] : a.bias;
  if (bias) {
    float b[32];
    load_bf16x32(static_cast<const uint16_t*>(bias) + n, b);
    add32(v, b);
  }
  if (EPI == EPI_ACT) {
    if (a.act == ACT_GELU) {
#pragma unroll
      for (int j = 0; j < 32; j += 2) gelu_exact2(v[j], v[j + 1]);
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = act_apply(v[j], a.act);
    }
  } else if (a.resid && row < a.M) {
    float r[32];
    if (a.resid_fp32)
      load_f32x32(static_cast<const float*>(a.resid) + static_cast<int64_t>(row) * a.ld_resid + n, r);
    else
      load_bf16x32(static_cast<const uint16_t*>(a.resid) + static_cast<int64_t>(row) * a.ld_resid + n, r);
    add32(v, r);
  }
}

// Each epilogue warp owns two 2 KB staging buffers for 32 rows x 32 16-bit columns,
// laid out like the 64-byte-swizzled TMA box: lane r's 16-byte piece j goes to
// position j ^ ((r >> 1) & 3) of its 64-byte row (no bank conflicts).  Lane 0
// stores the chunk at (x, y0) and recycles a buffer once the store issued two
// chunks earlier has read it.
// Stage 16 32-bit words per lane (a 32-row x 64-byte box) and store the box with TMA:
// 2-D at (x, y0), or 3-D at (x, y0, z) when z >= 0.
__device__ __forceinline__ void stage_words_and_store(const GemmArgs& a, const CUtensorMap* map,
                                                      uint8_t* warp_staging, int& count, int lane,
                                                      const uint32_t (&pk)[16], int x, int y0, int z) {
  uint8_t* buf = warp_staging + (count & 1) * 2048;
  if (count >= 2) {
    if (lane == 0) bulk_wait_group_read<1>();
    __syncwarp();
  }
  const int sw = (lane >> 1) & 3;
#pragma unroll
  for (int j = 0; j < 4; ++j)
    *reinterpret_cast<uint4*>(buf + lane * 64 + ((j ^ sw) << 4)) =
        make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0 && y0 < a.M) {
    if (z < 0)
      tma_store_2d(map, buf, x, y0);
    else
      tma_store_3d(map, buf, x, y0, z);
    bulk_commit_group();
  }
  ++count;
}

__device__ __forceinline__ void stage_and_store(const GemmArgs& a, const CUtensorMap* map, int out_type,
                                                uint8_t* warp_staging, int& count, int lane, const float (&v)[32],
                                                int x, int y0) {
  uint32_t pk[16];
  if (out_type == OUT_F16) {
    note_f16_range(a.status, absmax32(v), DEV_RANGE_COLUMN);
#pragma unroll
    for (int i = 0; i < 16; ++i) pk[i] = pack_f16x2(v[2 * i], v[2 * i + 1]);
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
  }
  stage_words_and_store(a, map, warp_staging, count, lane, pk, x, y0, -1);
}

__device__ __forceinline__ void load_f16x32(const void* p, float (&v)[32]) {
  const uint4* q = reinterpret_cast<const uint4*>(p);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 u = __ldg(q + i);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[j]));
      v[i * 8 + j * 2] = f.x;
      v[i * 8 + j * 2 + 1] = f.y;
    }
  }
}

// One 32-column chunk of an epilogue whose 16-bit output leaves through TMA stores.
// `x` is the chunk's first output column, `y0` the first row of the warp's 32 rows.
template <int EPI>
__device__ __forceinline__ void epilogue_tma_chunk(const GemmArgs& a, const TileCoord& tc, int row, int n,
                                                   float (&v)[32], uint8_t* warp_staging, int& count, int lane,
                                                   int x, int y0) {
  if (EPI == EPI_ACT_GRAD) {
    // the backward's recomputation of the column layer: act(z) and act'(z), z = acc + b
    if (a.bias_g[tc.g]) {
      float b[32];
      load_bf16x32(static_cast<const uint16_t*>(a.bias_g[tc.g]) + n, b);
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] += b[j];
    }
    float gr[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = act_and_grad(v[j], a.act, gr[j]);
    stage_and_store(a, &a.tmOut, a.out_type, warp_staging, count, lane, v, x, y0);
    stage_and_store(a, &a.tmOut2, OUT_F16, warp_staging, count, lane, gr, x, y0);
    return;
  }
  if (EPI == EPI_PARTIAL_F32) {
    // fp32 output through a 3-D map (column, row, group): two 16-column boxes per chunk
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      uint32_t pk[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) pk[i] = __float_as_uint(v[half * 16 + i]);
      stage_words_and_store(a, &a.tmOut, warp_staging, count, lane, pk, n + half * 16, y0, tc.g);
    }
    return;
  }
  if (EPI == EPI_MUL_GRAD) {
    // dZ = dA * act'(Z): the factor sits at the output's own position
    if (row < a.M) {
      float gm[32];
      load_f16x32(static_cast<const uint16_t*>(a.grad_mul) + static_cast<int64_t>(row) * a.ld_grad + x, gm);
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] *= gm[j];
    }
    stage_and_store(a, &a.tmOut, a.out_type, warp_staging, count, lane, v, x, y0);
    return;
  }
  epilogue_math<EPI>(a, tc, row, n, v);
  stage_and_store(a, &a.tmOut, a.out_type, warp_staging, count, lane, v, x, y0);
}

__device__ __forceinline__ void load_f32x32_cg(const float* p, float (&v)[32]) {
  const float4* q = reinterpret_cast<const float4*>(p);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 u = __ldcg(q + i);
    v[i * 4] = u.x; v[i * 4 + 1] = u.y; v[i * 4 + 2] = u.z; v[i * 4 + 3] = u.w;
  }
}

// Step 3 inside the row GEMM (partials mode, a.red_out set).  Tiles run in the order
// m, n, group, so in every CTA pair's sequence all tiles of groups 0..G-2 come before any
// tile of group G-1.  A warp of a group g < G-1 tile stores its 32-row x 128-column region
// of the fp32 partial P_g (TMA stores) and counts it on the region's arrival counter.  The warp of the
// group G-1 tile that covers the same region waits (bounded) until the G-1 earlier
// partials are counted -- they were stored before their pairs started any group G-1
// tile, so the wait always ends -- and then sums P_0 .. P_{G-2} from memory and its own
// P_{G-1} straight from the accumulator, in the order 0..G-1, adds bias and residual and
// writes the output.  P_{G-1} is never stored.  The sums are those of a separate pass
// over the stored partials: same order, same bits.

// Arrival counter of the region (32 rows from row0, the 128 columns of col_region).
__device__ __forceinline__ int region_counter(const GemmArgs& a, int row0, int col_region) {
  return (row0 / 32) * ((a.N + 127) / 128) + col_region;
}

// Publish this warp's region of a partial.  Its lane 0 issued the region's TMA stores: it
// waits for them to complete, orders them before its generic accesses, and fences before the
// atomic that counts the region.
__device__ __forceinline__ void partial_signal(const GemmArgs& a, int ctr, int lane) {
  __syncwarp();
  if (lane == 0) {
    bulk_wait_group_all();
    fence_proxy_async_global();
    __threadfence();
    atomicAdd(&a.counters[ctr], 1u);
  }
  __syncwarp();
}

// Wait until the region's G-1 earlier partials are counted; fenced so that the warp's
// later loads see them.  false: the wait ran out (recorded in the status word).
__device__ __forceinline__ bool partial_wait(const GemmArgs& a, int ctr, int lane) {
  int ok = 1;
  if (lane == 0) {
    const volatile uint32_t* c = a.counters + ctr;
    const uint32_t want = static_cast<uint32_t>(a.G - 1);
    if (*c < want) {
      const uint64_t t0 = globaltimer_ns();
      while (*c < want) {
        if (globaltimer_ns() - t0 > a.wait_limit_ns) {
          record_status(a.status, DEV_TIMEOUT, WAIT_SITE_EPILOGUE);
          ok = 0;
          break;
        }
      }
    }
    __threadfence();
  }
  ok = __shfl_sync(0xffffffffu, ok, 0);
  __syncwarp();
  __threadfence();
  return ok != 0;
}

// One 32-column chunk of a group G-1 tile: out = ((P_0 + P_1) + ...) + P_{G-1} + bias + resid,
// taken 8 columns at a time (the result replaces v) to keep the registers in check.  The
// partials were written earlier in this launch: they are read with plain (L1-allocating)
// loads, never through the read-only path, and no line of them was in this SM's L1 before.
__device__ __forceinline__ void reduce_chunk(const GemmArgs& a, int row, int n, float (&v)[32], bool ok,
                                             uint8_t* warp_staging, int& count, int lane) {
  if (row < a.M && ok) {
    const float* p = static_cast<const float*>(a.out) + static_cast<int64_t>(row) * a.ld_out + n;
#pragma unroll
    for (int qt = 0; qt < 4; ++qt) {
      float4 acc[2];
      // 8 columns at a time: the loads of partials 0..G-2 (up to four at a time) are all
      // issued before the adds, which then run in the order 0, 1, 2, ...
      for (int g0 = 0; g0 < a.G - 1; g0 += 4) {
        float4 w[4][2];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if (g0 + u < a.G - 1) {
            const float4* q =
                reinterpret_cast<const float4*>(p + static_cast<int64_t>(g0 + u) * a.out_group_stride + qt * 8);
            w[u][0] = q[0];
            w[u][1] = q[1];
          }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if (g0 + u < a.G - 1) {
#pragma unroll
            for (int i = 0; i < 2; ++i) {
              if (g0 + u == 0) {
                acc[i] = w[u][i];
              } else {
                acc[i].x += w[u][i].x; acc[i].y += w[u][i].y; acc[i].z += w[u][i].z; acc[i].w += w[u][i].w;
              }
            }
          }
        }
      }
      // then the last partial, straight from the accumulator
      if (a.G > 1) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          float* d = &v[qt * 8 + i * 4];
          d[0] = acc[i].x + d[0]; d[1] = acc[i].y + d[1]; d[2] = acc[i].z + d[2]; d[3] = acc[i].w + d[3];
        }
      }
    }
    if (a.bias) {
      float b[32];
      load_bf16x32(static_cast<const uint16_t*>(a.bias) + n, b);
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] += b[j];
    }
    if (a.resid) {
      float r[32];
      if (a.resid_fp32)
        load_f32x32(static_cast<const float*>(a.resid) + static_cast<int64_t>(row) * a.ld_resid + n, r);
      else
        load_bf16x32(static_cast<const uint16_t*>(a.resid) + static_cast<int64_t>(row) * a.ld_resid + n, r);
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] += r[j];
    }
  }
  if (a.red_out_f32) {
    if (row < a.M) store_f32x32(static_cast<float*>(a.red_out) + static_cast<int64_t>(row) * a.N + n, v);
  } else {
    stage_and_store(a, &a.tmOut2, OUT_BF16, warp_staging, count, lane, v, n, row - lane);
  }
}

// One 32-column chunk of one accumulator row: apply the epilogue and store.
template <int EPI>
__device__ __forceinline__ void epilogue_chunk(const GemmArgs& a, const TileCoord& tc, int row, int n,
                                               float (&v)[32]) {
  switch (EPI) {
    case EPI_ACT: {
      if (a.bias_g[tc.g]) {
        float b[32];
        load_bf16x32(static_cast<const uint16_t*>(a.bias_g[tc.g]) + n, b);
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] += b[j];
      }
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = act_apply(v[j], a.act);
      if (a.out_type == OUT_F16) note_f16_range(a.status, absmax32(v), DEV_RANGE_COLUMN);
      store_x32(a.out, static_cast<int64_t>(row) * a.ld_out + static_cast<int64_t>(tc.g) * a.out_col_per_group + n,
                a.out_type, v);
      break;
    }
    case EPI_PARTIAL_F32: {
      float* o = static_cast<float*>(a.out) + static_cast<int64_t>(tc.g) * a.out_group_stride +
                 static_cast<int64_t>(row) * a.ld_out + n;
      store_f32x32(o, v);
      break;
    }
    case EPI_BIAS_RESID: {
      if (a.bias) {
        float b[32];
        load_bf16x32(static_cast<const uint16_t*>(a.bias) + n, b);
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] += b[j];
      }
      if (a.resid) {
        float r[32];
        if (a.resid_fp32)
          load_f32x32(static_cast<const float*>(a.resid) + static_cast<int64_t>(row) * a.ld_resid + n, r);
        else
          load_bf16x32(static_cast<const uint16_t*>(a.resid) + static_cast<int64_t>(row) * a.ld_resid + n, r);
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] += r[j];
      }
      store_x32(a.out, static_cast<int64_t>(row) * a.ld_out + n, a.out_type, v);
      break;
    }
    case EPI_QKV: {
      if (a.bias_g[tc.g]) {
        float b[32];
        load_bf16x32(static_cast<const uint16_t*>(a.bias_g[tc.g]) + n, b);
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] += b[j];
      }
      const int per = a.Hg * a.d;
      const int part = n / per;
      const int within = n - part * per;
      const int head = tc.g * a.Hg + within / a.d;
      const int dd = within % a.d;
      const int b = row / a.S;
      const int s = row - b * a.S;
      void* base = part == 0 ? a.q : (part == 1 ? a.k : a.v);
      uint16_t* o = static_cast<uint16_t*>(base) +
                    ((static_cast<int64_t>(b) * a.H + head) * a.S + s) * a.d + dd;
      note_f16_range(a.status, absmax32(v), DEV_RANGE_QKV);
      store_f16x32(o, v);
      break;
    }
    default:
      break;
  }
}

template <int EPI, int OPL>
__global__ void __launch_bounds__(THREADS, 1) tp_gemm_kernel(const __grid_constant__ GemmArgs a) {
  constexpr bool A_MN = (OPL & OPL_A_MN) != 0;
  constexpr bool B_KM = (OPL & OPL_B_KMAJOR) != 0;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment for the 128-byte-swizzled tiles.
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_STAGE_BYTES;
  uint8_t* staging = smem + STAGES * STAGE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(staging + STAGING_BYTES);
  uint64_t* full_bar = bars;                       // [STAGES]
  uint64_t* empty_bar = bars + STAGES;             // [STAGES]
  uint64_t* acc_full = bars + 2 * STAGES;          // [NUM_ACC]
  uint64_t* acc_empty = bars + 2 * STAGES + NUM_ACC;  // [NUM_ACC]
  uint64_t* drain_bar = bars + 2 * STAGES + 2 * NUM_ACC;
  uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(drain_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_base_slot + 1);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  const int m_tiles = (a.M + BM - 1) / BM;
  const int n_tiles = (a.N + BN - 1) / BN;
  const int num_tiles = m_tiles * n_tiles * (a.concat ? 1 : a.G);
  const int kb_per_group = (a.Kg + BK - 1) / BK;   // a ragged last K step reads zero fill
  const int k_iters = a.concat ? kb_per_group * a.G : kb_per_group;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int s = 0; s < NUM_ACC; ++s) {
      mbar_init(&acc_full[s], 1);
      mbar_init(&acc_empty[s], EPI_WARPS);  // one arrival per epilogue warp
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(tmem_base_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_base_slot;
  // Dependents may start once every CTA of this grid is resident (see the pair kernel).
  pdl_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&a.tmA);
      for (int g = 0; g < a.G; ++g) tma_prefetch_desc(&a.tmB[g]);
      if (a.tma_store) tma_prefetch_desc(&a.tmOut);
      // both operands are re-read by several CTAs at about the same time: default L2 policy
      const uint64_t pol_a = l2_policy_evict_normal();
      const uint64_t pol_b = pol_a;
      pdl_wait();  // the previous kernel's outputs (our operands) are complete
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const TileCoord tc = tile_coord(a, tile, m_tiles, n_tiles);
        const int m0 = tc.m_blk * BM;
        const int n0 = tc.n_blk * BN;
        for (int it = 0; it < k_iters; ++it) {
          if (*abort_flag) { ok = false; break; }
          if (!mbar_wait_bounded(&empty_bar[stage], phase ^ 1u, a.wait_limit_ns, a.status, WAIT_SITE_PRODUCER)) {
            *abort_flag = 1; ok = false; break;
          }
          const int g = a.concat ? it / kb_per_group : tc.g;
          const int kb = a.concat ? it - g * kb_per_group : it;
          mbar_arrive_expect_tx(&full_bar[stage], STAGE_BYTES);
          uint8_t* a_dst = sA + stage * A_STAGE_BYTES;
          const int ka = g * a.a_k_per_group + kb * BK;
          if (!A_MN) {
            tma_load_2d_hint(a_dst, &a.tmA, &full_bar[stage], ka, m0, pol_a);
          } else {  // two 64-wide M blocks of 64 K rows
            tma_load_3d_hint(a_dst, &a.tmA, &full_bar[stage], 0, ka, (g * a.a_m_per_group + m0) / 64, pol_a);
          }
          uint8_t* b_dst = sB + stage * B_STAGE_BYTES;
          if (!B_KM) {  // four 64-wide N blocks of 64 K rows, two per load
            tma_load_3d_hint(b_dst, &a.tmB[g], &full_bar[stage], 0, kb * BK, n0 / 64, pol_b);
            tma_load_3d_hint(b_dst + 2 * B_BLOCK_BYTES, &a.tmB[g], &full_bar[stage], 0, kb * BK, n0 / 64 + 2, pol_b);
          } else {  // two 128-row N blocks of 64 K each
            tma_load_2d_hint(b_dst, &a.tmB[g], &full_bar[stage], kb * BK, n0, pol_b);
            tma_load_2d_hint(b_dst + BN / 2 * 128, &a.tmB[g], &full_bar[stage], kb * BK, n0 + BN / 2, pol_b);
          }
          ++issued;
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      // Wait for our own copies still in flight (the last min(issued, STAGES) stages).
      const int pending = issued < STAGES ? issued : STAGES;
      int s = stage;
      uint32_t ph = phase;
      for (int i = 0; i < pending; ++i) {
        if (--s < 0) { s = STAGES - 1; ph ^= 1u; }
        mbar_wait_bounded(&full_bar[s], ph, a.wait_limit_ns, a.status, WAIT_SITE_PRODUCER);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      const uint32_t idesc = a.ab_f16 ? idesc_f16_f32(BM, BN, A_MN, !B_KM)
                                      : idesc_bf16_f32(BM, BN, A_MN, !B_KM);
      const uint32_t sA_addr = smem_u32(sA);
      const uint32_t sB_addr = smem_u32(sB);
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        if (!mbar_wait_bounded(&acc_empty[acc], acc_phase ^ 1u, a.wait_limit_ns, a.status, WAIT_SITE_MMA_ACC)) {
          *abort_flag = 1; ok = false; break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int it = 0; it < k_iters; ++it) {
          if (*abort_flag) { ok = false; break; }
          if (!mbar_wait_bounded(&full_bar[stage], phase, a.wait_limit_ns, a.status, WAIT_SITE_MMA_FULL)) {
            *abort_flag = 1; ok = false; break;
          }
          tc_fence_after();
          const uint32_t a_base = sA_addr + stage * A_STAGE_BYTES;
          const uint32_t b_base = sB_addr + stage * B_STAGE_BYTES;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            // K-major operand: advance 16 elements (32 bytes) inside the swizzle atom;
            // MN-major operand: advance 16 K-rows (2048 bytes), 64-wide MN blocks 8 KB apart.
            const uint64_t adesc = A_MN ? smem_desc_sw128(a_base + k * 16 * 128, B_BLOCK_BYTES, 1024)
                                          : smem_desc_sw128(a_base + k * 32, 16, 1024);
            const uint64_t bdesc = B_KM ? smem_desc_sw128(b_base + k * 32, 16, 1024)
                                              : smem_desc_sw128(b_base + k * 16 * 128, B_BLOCK_BYTES, 1024);
            mma_bf16_ss(d_tmem, adesc, bdesc, idesc, (it > 0 || k > 0) ? 1u : 0u);
          }
          mma_commit(&empty_bar[stage]);  // frees the smem stage once these MMAs finish
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        mma_commit(&acc_full[acc]);       // accumulator ready for the epilogue
        if (++acc == NUM_ACC) { acc = 0; acc_phase ^= 1u; }
      }
      // Drain: wait until every MMA issued by this thread has completed.
      mma_commit(drain_bar);
      mbar_wait_bounded(drain_bar, 0, a.wait_limit_ns, a.status, WAIT_SITE_MMA_ACC);
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..5)
    const int sub = warp & 3;               // TMEM sub-partition this warp may access
    const int row_in_tile = sub * 32 + lane;
    const int col_half = (warp - 2) / 4;    // columns [col_half*BN/2, +BN/2) of each tile
    int acc = 0;
    uint32_t acc_phase = 0;
    const bool tma_out = a.tma_store && (EPI == EPI_ACT || EPI == EPI_BIAS_RESID || EPI == EPI_ACT_GRAD ||
                                         EPI == EPI_MUL_GRAD || EPI == EPI_PARTIAL_F32);
    uint8_t* warp_staging = staging + (warp - 2) * 4096;
    int store_count = 0;
    pdl_wait();  // bias / residual inputs and our outputs: after the previous kernel completes
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      if (*abort_flag) break;
      // the decision is made warp-uniform: tcgen05.ld below is a warp-collective instruction
      const bool ready = __all_sync(0xffffffffu,
                                    mbar_wait_bounded(&acc_full[acc], acc_phase, a.wait_limit_ns, a.status,
                                                      WAIT_SITE_EPILOGUE));
      if (!ready) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const TileCoord tc = tile_coord(a, tile, m_tiles, n_tiles);
      const int row = tc.m_blk * BM + row_in_tile;
      const int n0 = tc.n_blk * BN;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(sub * 32) << 16) + static_cast<uint32_t>(acc * BN);
      // columns [c_begin*32, c_end*32) of the tile, clipped to N (a multiple of 32);
      // the TMEM load of chunk c+1 is issued before chunk c is processed
      const int c_begin = col_half * (BN / 64);
      int c_end = (col_half + 1) * (BN / 64);
      if (n0 + c_end * 32 > a.N) c_end = (a.N - n0) / 32;
      // partials mode with the reduction here: this warp's region and its role in it
      const int row0 = tc.m_blk * BM + sub * 32;
      const bool in_region = EPI == EPI_PARTIAL_F32 && a.red_out && row0 < a.M && c_begin < c_end;
      const int ctr = in_region ? region_counter(a, row0, n0 / 128 + col_half) : 0;
      const bool red_tile = EPI == EPI_PARTIAL_F32 && a.red_out && tc.g == a.G - 1;
      bool red_ok = true;
      if (red_tile && in_region) {
        red_ok = partial_wait(a, ctr, lane);
        if (!red_ok) *abort_flag = 1;
      }
      if (c_begin < c_end && red_tile) {
        // last shard's tile: one chunk at a time (the registers go to the partials' loads)
        for (int c = c_begin; c < c_end; ++c) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(t_row + c * 32, r);
          tmem_ld_wait();
          float v[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
          reduce_chunk(a, row, n0 + c * 32, v, red_ok, warp_staging, store_count, lane);
        }
      } else if (c_begin < c_end) {
        uint32_t r[2][32];
        tmem_ld_32x32b_x32(t_row + c_begin * 32, r[0]);
#pragma unroll
        for (int c = c_begin; c < c_begin + BN / 64; ++c) {
          if (c >= c_end) break;
          tmem_ld_wait();
          const int cur = (c - c_begin) & 1;
          if (c + 1 < c_end) tmem_ld_32x32b_x32(t_row + (c + 1) * 32, r[cur ^ 1]);
          float v[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[cur][j]);
          if (tma_out) {
            const int x = (EPI == EPI_BIAS_RESID ? 0 : tc.g * static_cast<int>(a.out_col_per_group)) + n0 + c * 32;
            epilogue_tma_chunk<EPI>(a, tc, row, n0 + c * 32, v, warp_staging, store_count, lane, x, row - lane);
          } else if (row < a.M) {
            epilogue_chunk<EPI>(a, tc, row, n0 + c * 32, v);
          }
        }
        tmem_ld_wait();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);
      if (++acc == NUM_ACC) { acc = 0; acc_phase ^= 1u; }
      if (in_region && !red_tile) partial_signal(a, ctr, lane);
    }
    if (lane == 0) bulk_wait_group_all();  // our output stores are complete before exit
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ============================================================================ CTA-pair variant
// Same roles and epilogues; a cluster of two CTAs computes a 256x256 tile with
// tcgen05.mma.cta_group::2 (M=256, N=256, K=16) issued by the leader (rank 0).
// Each CTA loads only its own operand halves -- A rows [rank*128, +128) and B
// columns [rank*128, +128) of the tile -- so each SM streams 32 KB per 64-wide K
// step instead of 48 KB.  Both CTAs' TMA loads count their bytes on the leader's
// full barrier; the leader's commits arrive on both CTAs' empty / accumulator
// barriers; both CTAs' epilogues arrive on the leader's accumulator-empty barrier.
// No load is multicast.
//
// A wide variant (PBN = 512: 256 x 512 tiles): each 64-wide K step feeds two N=256 MMAs
// from one A tile, so an SM streams 48 KB per 1024 tensor cycles instead of 32 KB per 512
// (a quarter fewer operand bytes for the same work).  Its one accumulator fills all 512
// TMEM columns, so each round's epilogue is exposed instead of overlapping the next tile's
// main loop; the launcher picks it only where that costs little (launch_gemm_pair).
constexpr int P_ROWS = 2 * BM;                      // 256 rows per pair
constexpr int P_A_BYTES = BM * BK * 2;              // 16 KB per CTA

template <int PBN>
struct PairCfg {
  static_assert(PBN == 256 || PBN == 512, "pair tile width");
  static constexpr int NH = PBN / 256;                      // N=256 MMAs per 16-deep K step
  static constexpr int B_BYTES = (PBN / 2) * BK * 2;        // this CTA's B columns: 16 or 32 KB
  static constexpr int STAGE_BYTES = P_A_BYTES + B_BYTES;
  static constexpr int STAGES = PBN == 256 ? 6 : 4;
  static constexpr int NUM_ACC = TMEM_COLS / PBN;           // 2 or 1
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + STAGING_BYTES + 256;
};
static_assert(PairCfg<256>::SMEM_BYTES == PairCfg<512>::SMEM_BYTES, "both widths share the smem attribute");
constexpr int P_SMEM_BYTES = PairCfg<256>::SMEM_BYTES;

template <int EPI, int OPL, int PBN>
__global__ void __launch_bounds__(THREADS, 1) tp_gemm_pair_kernel(const __grid_constant__ GemmArgs a) {
  using C = PairCfg<PBN>;
  constexpr bool A_MN = (OPL & OPL_A_MN) != 0;
  constexpr bool B_KM = (OPL & OPL_B_KMAJOR) != 0;
  // the in-epilogue partials reduction counts 128-column regions of 256-wide tiles
  static_assert(PBN == 256 || EPI != EPI_PARTIAL_F32, "wide tiles: no partials epilogue");
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::STAGES * P_A_BYTES;
  uint8_t* staging = smem + C::STAGES * C::STAGE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(staging + STAGING_BYTES);
  uint64_t* full_bar = bars;                                    // [STAGES], used in the leader
  uint64_t* empty_bar = bars + C::STAGES;                       // [STAGES], both CTAs
  uint64_t* acc_full = bars + 2 * C::STAGES;                    // [NUM_ACC], both CTAs
  uint64_t* acc_empty = bars + 2 * C::STAGES + C::NUM_ACC;      // [NUM_ACC], used in the leader
  uint64_t* drain_bar = bars + 2 * C::STAGES + 2 * C::NUM_ACC;
  uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(drain_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_base_slot + 1);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int cid = static_cast<int>(blockIdx.x >> 1);
  const int nclusters = static_cast<int>(gridDim.x >> 1);

  const int m_tiles = (a.M + P_ROWS - 1) / P_ROWS;
  const int n_tiles = (a.N + PBN - 1) / PBN;
  const int num_tiles = m_tiles * n_tiles * (a.concat ? 1 : a.G);
  const int kb_per_group = (a.Kg + BK - 1) / BK;   // a ragged last K step reads zero fill
  const int k_iters = a.concat ? kb_per_group * a.G : kb_per_group;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int s = 0; s < C::NUM_ACC; ++s) {
      mbar_init(&acc_full[s], 1);
      mbar_init(&acc_empty[s], 2 * EPI_WARPS);  // one arrival per epilogue warp of each CTA
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_base_slot, TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // barriers of both CTAs initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem_base = *tmem_base_slot;
  // The next kernel may be scheduled onto SMs this grid leaves idle in its tail.  It starts
  // only once every CTA of this grid has issued this, i.e. is resident, so it cannot take
  // an SM this grid still needs; its own wait keeps it from our outputs until we finish.
  pdl_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      tma_prefetch_desc(&a.tmA);
      for (int g = 0; g < a.G; ++g) tma_prefetch_desc(&a.tmB[g]);
      if (a.tma_store) tma_prefetch_desc(&a.tmOut);
      // both operands are re-read by several CTAs at about the same time: default L2 policy
      const uint64_t pol_a = l2_policy_evict_normal();
      const uint64_t pol_b = pol_a;
      const uint32_t full0_leader = mapa_shared(smem_u32(&full_bar[0]), 0);
      // Before waiting for the previous kernel: pull the first stages of this CTA's first
      // tile into L2 (prefetch only; the loads into shared memory come after the wait).
      if (cid < num_tiles) {
        const TileCoord tc = tile_coord(a, cid, m_tiles, n_tiles);
        const int m0 = tc.m_blk * P_ROWS + static_cast<int>(rank) * BM;
        const int n0 = tc.n_blk * PBN + static_cast<int>(rank) * 128;
        const bool rev = a.concat != 0;
        const int pre = k_iters < C::STAGES ? k_iters : C::STAGES;
        for (int it = 0; it < pre; ++it) {
          const int kidx = rev ? k_iters - 1 - it : it;
          const int g = a.concat ? kidx / kb_per_group : tc.g;
          const int kb = a.concat ? kidx - g * kb_per_group : kidx;
          const int ka = g * a.a_k_per_group + kb * BK;
          if (!A_MN) tma_prefetch_l2_2d(&a.tmA, ka, m0);
          else tma_prefetch_l2_3d(&a.tmA, 0, ka, (g * a.a_m_per_group + m0) / 64);
#pragma unroll
          for (int h = 0; h < C::NH; ++h) {
            if (!B_KM) tma_prefetch_l2_3d(&a.tmB[g], 0, kb * BK, (n0 + h * 256) / 64);
            else tma_prefetch_l2_2d(&a.tmB[g], kb * BK, n0 + h * 256);
          }
        }
      }
      pdl_wait();  // the previous kernel's outputs (our operands) are complete
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      for (int tile = cid; tile < num_tiles && ok; tile += nclusters) {
        const TileCoord tc = tile_coord(a, tile, m_tiles, n_tiles);
        const int m0 = tc.m_blk * P_ROWS + static_cast<int>(rank) * BM;
        // this CTA's B columns: [n0 + h*256, +128) for each N=256 half h of the tile
        const int n0 = tc.n_blk * PBN + static_cast<int>(rank) * 128;
        // Row layer: the K loop runs backwards in even rounds of tiles and forwards in odd
        // ones, so each round starts on the K-slices of A that are still in L2 -- the end
        // of K for the first round (the producing layer wrote it last), the start for the
        // second (the first round read it last), and so on.  The order is fixed per tile.
        const bool rev = a.concat && (((tile - cid) / nclusters) & 1) == 0;
        for (int it = 0; it < k_iters; ++it) {
          if (*abort_flag) { ok = false; break; }
          if (!mbar_wait_bounded(&empty_bar[stage], phase ^ 1u, a.wait_limit_ns, a.status, WAIT_SITE_PRODUCER)) {
            *abort_flag = 1; ok = false; break;
          }
          const int kidx = rev ? k_iters - 1 - it : it;
          const int g = a.concat ? kidx / kb_per_group : tc.g;
          const int kb = a.concat ? kidx - g * kb_per_group : kidx;
          const uint32_t fb = full0_leader + static_cast<uint32_t>(stage) * 8u;
          if (leader) mbar_arrive_expect_tx(&full_bar[stage], 2 * C::STAGE_BYTES);
          uint8_t* a_dst = sA + stage * P_A_BYTES;
          const int ka = g * a.a_k_per_group + kb * BK;
          if (!A_MN) {
            tma_load_2d_pair(a_dst, &a.tmA, fb, ka, m0, pol_a);
          } else {  // two 64-wide M blocks of 64 K rows, one load
            tma_load_3d_pair(a_dst, &a.tmA, fb, 0, ka, (g * a.a_m_per_group + m0) / 64, pol_a);
          }
          uint8_t* b_dst = sB + stage * C::B_BYTES;
#pragma unroll
          for (int h = 0; h < C::NH; ++h) {
            if (!B_KM) {  // this CTA's two 64-wide N blocks of 64 K rows, one load
              tma_load_3d_pair(b_dst + h * 16384, &a.tmB[g], fb, 0, kb * BK, (n0 + h * 256) / 64, pol_b);
            } else {  // this CTA's 128 N rows, 64 K each
              tma_load_2d_pair(b_dst + h * 16384, &a.tmB[g], fb, kb * BK, n0 + h * 256, pol_b);
            }
          }
          ++issued;
          if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      // Our copies are in flight until the leader's MMAs have consumed their stage:
      // wait for the consumption of the last min(issued, STAGES) stages.
      const int pending = issued < C::STAGES ? issued : C::STAGES;
      int s = stage;
      uint32_t ph = phase;
      for (int i = 0; i < pending; ++i) {
        if (--s < 0) { s = C::STAGES - 1; ph ^= 1u; }
        mbar_wait_bounded(&empty_bar[s], ph, a.wait_limit_ns, a.status, WAIT_SITE_PRODUCER);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader only)
    // The whole warp runs the loop (its values stay warp-uniform); one elected lane issues.
    if (leader) {
      const uint32_t idesc = a.ab_f16 ? idesc_f16_f32(P_ROWS, 256, A_MN, !B_KM)
                                      : idesc_bf16_f32(P_ROWS, 256, A_MN, !B_KM);
      const uint32_t sA_addr = smem_u32(sA);
      const uint32_t sB_addr = smem_u32(sB);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = cid; tile < num_tiles && ok; tile += nclusters) {
        if (!warp_wait_bounded(&acc_empty[acc], acc_phase ^ 1u, a.wait_limit_ns, a.status, WAIT_SITE_MMA_ACC)) {
          *abort_flag = 1; ok = false; break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * PBN);
        for (int it = 0; it < k_iters; ++it) {
          if (__any_sync(0xffffffffu, *abort_flag != 0)) { ok = false; break; }
          if (!warp_wait_bounded(&full_bar[stage], phase, a.wait_limit_ns, a.status, WAIT_SITE_MMA_FULL)) {
            *abort_flag = 1; ok = false; break;
          }
          tc_fence_after();
          const uint32_t a_base = sA_addr + stage * P_A_BYTES;
          const uint32_t b_base = sB_addr + stage * C::B_BYTES;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t adesc = A_MN ? smem_desc_sw128(a_base + k * 16 * 128, B_BLOCK_BYTES, 1024)
                                          : smem_desc_sw128(a_base + k * 32, 16, 1024);
#pragma unroll
            for (int h = 0; h < C::NH; ++h) {
              const uint32_t bh = b_base + static_cast<uint32_t>(h) * 16384u;
              const uint64_t bdesc = B_KM ? smem_desc_sw128(bh + k * 32, 16, 1024)
                                          : smem_desc_sw128(bh + k * 16 * 128, B_BLOCK_BYTES, 1024);
              mma_pair_ss_elect(d_tmem + static_cast<uint32_t>(h * 256), adesc, bdesc, idesc, (it > 0 || k > 0) ? 1u : 0u);
            }
          }
          mma_commit_pair_mask_elect(&empty_bar[stage], 0x3);  // frees this stage in both CTAs
          if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        mma_commit_pair_mask_elect(&acc_full[acc], 0x3);       // accumulator ready in both CTAs
        if (++acc == C::NUM_ACC) { acc = 0; acc_phase ^= 1u; }
      }
      mma_commit_pair_local_elect(drain_bar);
      warp_wait_bounded(drain_bar, 0, a.wait_limit_ns, a.status, WAIT_SITE_MMA_ACC);
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..5 of both CTAs)
    const int sub = warp & 3;
    const int row_in_tile = static_cast<int>(rank) * BM + sub * 32 + lane;
    const int col_half = (warp - 2) / 4;    // columns [col_half*PBN/2, +PBN/2) of each tile
    const uint32_t acc_empty0_leader = mapa_shared(smem_u32(&acc_empty[0]), 0);
    pdl_wait();  // bias / residual inputs and our outputs: after the previous kernel completes
    int acc = 0;
    uint32_t acc_phase = 0;
    const bool tma_out = a.tma_store && (EPI == EPI_ACT || EPI == EPI_BIAS_RESID || EPI == EPI_ACT_GRAD ||
                                         EPI == EPI_MUL_GRAD || EPI == EPI_PARTIAL_F32);
    uint8_t* warp_staging = staging + (warp - 2) * 4096;
    int store_count = 0;
    for (int tile = cid; tile < num_tiles; tile += nclusters) {
      if (*abort_flag) break;
      const bool ready = __all_sync(0xffffffffu,
                                    mbar_wait_bounded(&acc_full[acc], acc_phase, a.wait_limit_ns, a.status,
                                                      WAIT_SITE_EPILOGUE));
      if (!ready) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const TileCoord tc = tile_coord(a, tile, m_tiles, n_tiles);
      const int row = tc.m_blk * P_ROWS + row_in_tile;
      const int n0 = tc.n_blk * PBN;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(sub * 32) << 16) + static_cast<uint32_t>(acc * PBN);
      // columns [c_begin*32, c_end*32) of the tile, clipped to N (a multiple of 32);
      // the TMEM load of chunk c+1 is issued before chunk c is processed
      const int c_begin = col_half * (PBN / 64);
      int c_end = (col_half + 1) * (PBN / 64);
      if (n0 + c_end * 32 > a.N) c_end = (a.N - n0) / 32;
      // partials mode with the reduction here: this warp's region and its role in it
      const int row0 = tc.m_blk * P_ROWS + static_cast<int>(rank) * BM + sub * 32;
      const bool in_region = EPI == EPI_PARTIAL_F32 && a.red_out && row0 < a.M && c_begin < c_end;
      const int ctr = in_region ? region_counter(a, row0, n0 / 128 + col_half) : 0;
      const bool red_tile = EPI == EPI_PARTIAL_F32 && a.red_out && tc.g == a.G - 1;
      bool red_ok = true;
      if (red_tile && in_region) {
        red_ok = partial_wait(a, ctr, lane);
        if (!red_ok) *abort_flag = 1;
      }
      if (c_begin < c_end && red_tile) {
        // last shard's tile: one chunk at a time (the registers go to the partials' loads)
        for (int c = c_begin; c < c_end; ++c) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(t_row + c * 32, r);
          tmem_ld_wait();
          float v[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
          reduce_chunk(a, row, n0 + c * 32, v, red_ok, warp_staging, store_count, lane);
        }
      } else if (c_begin < c_end) {
        uint32_t r[2][32];
        tmem_ld_32x32b_x32(t_row + c_begin * 32, r[0]);
#pragma unroll
        for (int c = c_begin; c < c_begin + PBN / 64; ++c) {
          if (c >= c_end) break;
          tmem_ld_wait();
          const int cur = (c - c_begin) & 1;
          if (c + 1 < c_end) tmem_ld_32x32b_x32(t_row + (c + 1) * 32, r[cur ^ 1]);
          float v[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[cur][j]);
          if (tma_out) {
            const int x = (EPI == EPI_BIAS_RESID ? 0 : tc.g * static_cast<int>(a.out_col_per_group)) + n0 + c * 32;
            epilogue_tma_chunk<EPI>(a, tc, row, n0 + c * 32, v, warp_staging, store_count, lane, x, row - lane);
          } else if (row < a.M) {
            epilogue_chunk<EPI>(a, tc, row, n0 + c * 32, v);
          }
        }
        tmem_ld_wait();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty0_leader + static_cast<uint32_t>(acc) * 8u);
      if (++acc == C::NUM_ACC) { acc = 0; acc_phase ^= 1u; }
      if (in_region && !red_tile) partial_signal(a, ctr, lane);
    }
    if (lane == 0) bulk_wait_group_all();  // our output stores are complete before exit
  }

  __syncwarp();
  tc_fence_before();
  cluster_sync_all();  // the leader's MMAs and the remote arrives are done in both CTAs
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

}  // namespace

// CTA pairs are the default; TPB_GEMM_PAIRS=0 selects the one-CTA kernel.
static bool gemm_use_pairs() {
  static int v = -1;
  if (v < 0) {
    const char* e = getenv("TPB_GEMM_PAIRS");
    v = (e && e[0] == '0') ? 0 : 1;
  }
  return v == 1;
}

// 256 x 512 pair tiles (TPB_GEMM_WIDE=0 turns them off) for the grids they bring down to
// one round of tiles.
static bool gemm_use_wide() {
  static int v = -1;
  if (v < 0) {
    const char* e = getenv("TPB_GEMM_WIDE");
    v = (e && e[0] == '0') ? 0 : 1;
  }
  return v == 1;
}

typedef void (*GemmKernel)(GemmArgs);

// Kernel variants: the one-CTA kernel, CTA pairs on 256 x 256 tiles, CTA pairs on 256 x 512.
enum { VAR_SINGLE = 0, VAR_PAIR = 1, VAR_PAIR_WIDE = 2, NUM_VAR = 3 };

// The kernel instantiation for an epilogue kind and operand layout: each instantiation holds
// only its own epilogue and operand addressing, so neither the register budget nor the
// MMA-issuing warp pays for the paths it does not take.  The combinations the
// library launches: forward layers (K-major A, N-major B) with every forward epilogue; the
// backward's dZ (K-major B, fp16 factor), weight gradients (M-major A, fp32 out) and dX
// (K-major B, sum over shards).
static GemmKernel gemm_kernel_for(int epi, int opl, int var) {
  // wide tiles: the row layer's bias + residual epilogue (forward, and the backward's dX)
  if (var == VAR_PAIR_WIDE) {
    if (epi == EPI_BIAS_RESID && opl == 0) return tp_gemm_pair_kernel<EPI_BIAS_RESID, 0, 512>;
    if (epi == EPI_BIAS_RESID && opl == OPL_B_KMAJOR) return tp_gemm_pair_kernel<EPI_BIAS_RESID, OPL_B_KMAJOR, 512>;
    return nullptr;
  }
  const bool pair = var == VAR_PAIR;
#define TP_GEMM_PICK(E, O) \
  if (epi == E && opl == O) return pair ? tp_gemm_pair_kernel<E, O, 256> : tp_gemm_kernel<E, O>;
  TP_GEMM_PICK(EPI_ACT, 0)
  TP_GEMM_PICK(EPI_PARTIAL_F32, 0)
  TP_GEMM_PICK(EPI_BIAS_RESID, 0)
  TP_GEMM_PICK(EPI_QKV, 0)
  TP_GEMM_PICK(EPI_ACT_GRAD, 0)
  TP_GEMM_PICK(EPI_MUL_GRAD, OPL_B_KMAJOR)
  TP_GEMM_PICK(EPI_PARTIAL_F32, OPL_A_MN)
  TP_GEMM_PICK(EPI_BIAS_RESID, OPL_B_KMAJOR)
  TP_GEMM_PICK(EPI_ACT, OPL_B_KMAJOR)
#undef TP_GEMM_PICK
  return nullptr;
}

static int operand_layout(const GemmArgs& a) { return (a.a_mn ? OPL_A_MN : 0) | (a.b_kmajor ? OPL_B_KMAJOR : 0); }

constexpr int NUM_EPI = 6;
static int g_pair_clusters[64] = {0};
static bool g_attr_set[64][NUM_VAR][NUM_EPI][4] = {};

// Allow the kernel's dynamic shared memory (once per device and instantiation).
static tp_status set_smem_attr(int dev, int epi, int opl, int var) {
  const bool known = dev >= 0 && dev < 64 && epi >= 0 && epi < NUM_EPI && opl >= 0 && opl < 4;
  if (known && g_attr_set[dev][var][epi][opl]) return TP_OK;
  GemmKernel k = gemm_kernel_for(epi, opl, var);
  if (!k) return set_error(TP_ERR_CUDA, "no GEMM instantiation for this epilogue and operand layout");
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           var == VAR_SINGLE ? SMEM_BYTES : P_SMEM_BYTES) != cudaSuccess)
    return set_error(TP_ERR_CUDA, "cudaFuncSetAttribute (shared memory) failed");
  if (known) g_attr_set[dev][var][epi][opl] = true;
  return TP_OK;
}

// Largest number of co-resident CTA pairs for the pair kernel on this device (every
// instantiation has the same block size and shared memory).
static int pair_clusters(int dev) {
  if (dev < 0 || dev >= 64) return 0;
  if (g_pair_clusters[dev]) return g_pair_clusters[dev];
  if (set_smem_attr(dev, EPI_ACT, 0, VAR_PAIR) != TP_OK) return -1;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(2 * (sm_count() / 2), 1, 1);
  cfg.blockDim = dim3(THREADS, 1, 1);
  cfg.dynamicSmemBytes = P_SMEM_BYTES;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, gemm_kernel_for(EPI_ACT, 0, VAR_PAIR), &cfg) != cudaSuccess || n <= 0) return -1;
  g_pair_clusters[dev] = n;
  return n;
}

static tp_status launch_gemm_pair(const GemmArgs& a, cudaStream_t stream, const char* name, int dev) {
  const int nclusters_max = pair_clusters(dev);
  if (nclusters_max <= 0) return TP_ERR_CUDA;
  const int opl = operand_layout(a);
  const int m_tiles = (a.M + P_ROWS - 1) / P_ROWS;
  const long long tiles256 = 1LL * m_tiles * ((a.N + 255) / 256) * (a.concat ? 1 : a.G);
  const long long tiles512 = 1LL * m_tiles * ((a.N + 511) / 512) * (a.concat ? 1 : a.G);
  // A wide tile is twice the tensor work of a 256 x 256 one, with a quarter fewer operand
  // bytes per SM, but its one accumulator leaves each round's epilogue exposed.  So: wide
  // where that takes no more rounds of tensor work (2 * rounds512 <= rounds256) and either
  // one round suffices or the K loop is long enough (>= 128 steps of 64) for the exposed
  // epilogue to be a few percent of a round.
  const long long rounds256 = (tiles256 + nclusters_max - 1) / nclusters_max;
  const long long rounds512 = (tiles512 + nclusters_max - 1) / nclusters_max;
  const long long k_steps = 1LL * ((a.Kg + BK - 1) / BK) * (a.concat ? a.G : 1);
  const bool wide = gemm_use_wide() && gemm_kernel_for(a.epi, opl, VAR_PAIR_WIDE) != nullptr &&
                    2 * rounds512 <= rounds256 && (rounds512 == 1 || k_steps >= 128);
  const int var = wide ? VAR_PAIR_WIDE : VAR_PAIR;
  const tp_status sa = set_smem_attr(dev, a.epi, opl, var);
  if (sa != TP_OK) return sa;
  const long long tiles = wide ? tiles512 : tiles256;
  if (tiles <= 0) return TP_OK;
  const int nclusters = static_cast<int>(tiles < nclusters_max ? tiles : nclusters_max);
  trace_before(stream, name);
  const tp_status st = launch_ex(gemm_kernel_for(a.epi, opl, var), dim3(2 * nclusters), dim3(THREADS), P_SMEM_BYTES,
                                 stream, 2, a);
  if (st != TP_OK) return st;
  trace_after(stream, name);
  return TP_OK;
}

tp_status launch_gemm(const GemmArgs& a, cudaStream_t stream, const char* name) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return TP_ERR_CUDA;
  if (gemm_use_pairs()) return launch_gemm_pair(a, stream, name, dev);
  const int opl = operand_layout(a);
  const tp_status sa = set_smem_attr(dev, a.epi, opl, VAR_SINGLE);
  if (sa != TP_OK) return sa;
  const int m_tiles = (a.M + BM - 1) / BM;
  const int n_tiles = (a.N + BN - 1) / BN;
  const long long tiles = 1LL * m_tiles * n_tiles * (a.concat ? 1 : a.G);
  if (tiles <= 0) return TP_OK;
  const int grid = static_cast<int>(tiles < sm_count() ? tiles : sm_count());
  trace_before(stream, name);
  const tp_status st = launch_ex(gemm_kernel_for(a.epi, opl, VAR_SINGLE), dim3(grid), dim3(THREADS), SMEM_BYTES, stream, 1, a);
  if (st != TP_OK) return st;
  trace_after(stream, name);
  return TP_OK;
}

}  // namespace tpb
