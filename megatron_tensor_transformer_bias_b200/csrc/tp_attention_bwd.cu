// Backward pass of per-head attention on tcgen05 tensor cores.
//
// "Tensor Parallelism > Combining Column and Row Parallelism", paragraphs on
// multi-head attention and head independence: the gradients of each head depend
// on that head's Q, K, V and output gradient only, so every head group's shard
// runs on its own; all heads run in one launch.
//
// For one head, with s = Q K^T (raw), P = exp2(s * log2(e)/sqrt(d) - LSE2) the
// softmax rows (LSE2 = the row's log2-sum-exp of the scaled scores, written by the
// forward kernel) and D = rowsum(dO * O):
//     dV = P^T dO,  dP = dO V^T,  dS = P * (dP - D),
//     dQ = dS K / sqrt(d),  dK = dS^T Q / sqrt(d).
// rowsum(P * dP) = rowsum(dO * O) because O = P V, so D is the softmax Jacobian's
// row correction.  Two kernels, each one resident 128-row block per CTA and no
// atomics (the sums run in one TMEM accumulator, in sub-block order):
//  * tp_attn_bwd_dkdv_kernel: one CTA per (128 keys, head, batch).  It keeps K_j and
//    V_j in shared memory and streams the 64-query sub-blocks that see them:
//    S^T = K_j Q_n^T and dP^T = V_j dO_n^T into TMEM; the compute warps (one key row
//    per thread) form P^T and dS^T in fp16 over them; then dV += P^T dO_n and
//    dK += dS^T Q_n read those from TMEM.
//  * tp_attn_bwd_dq_kernel: one CTA per (128 queries, head, batch).  It keeps Q_i
//    and dO_i and streams the 64-key sub-blocks the queries see: S = Q_i K_n^T and
//    dP = dO_i V_n^T; dS (one query row per thread); dQ += dS K_n.
// The score tiles are double-buffered in TMEM: the tensor core computes sub-block
// n+1's S and dP while the compute warps work on sub-block n, and the gradient MMAs
// of n run right after its compute.
// Each recomputes S (the forward's scores) instead of storing them.  Q, K, V are
// [B*H][S][d] fp16 (the forward's workspace), dO is [B*S, H*d] fp16 (read through a
// 4-D tensor map), LSE2 and D are [B*H][S_pad] fp32 with S_pad a multiple of 128 and
// the rows past S set to (+inf, 0), so those queries weigh nothing.  dQ, dK, dV are
// written as bf16 into the packed gradient of the QKV projection, [B*S, 3*H*d], head
// group g's columns being [dQ heads | dK heads | dV heads] like its weight shard.
#include <cstdio>

#include "tp_internal.h"
#include "tp_ptx.cuh"

namespace tpb {

namespace {

constexpr int BR = 128;                      // resident rows per CTA (keys or queries)
constexpr int BS = 64;                       // streamed rows per sub-block
constexpr int D = 128;                       // head dim
constexpr int HALF_R = BR * 64 * 2;          // [128 rows x 64 d] fp16, 128-byte swizzle: 16 KB
constexpr int TILE_R = 2 * HALF_R;           // 32 KB
constexpr int HALF_S = BS * 64 * 2;          // [64 rows x 64 d]: 8 KB
constexpr int TILE_S = 2 * HALF_S;           // 16 KB
constexpr int NST_KV = 3;                    // shared-memory stages of streamed sub-blocks (dK/dV)
constexpr int NST_Q = 4;                     // (dQ)
constexpr int STAGING = 2 * HALF_R;          // a 128 x 128 bf16 gradient block on its way out (TMA store)
constexpr int THREADS = 224;                 // warp 0 TMA, warps 1 and 2 MMA, warps 3..6 compute
constexpr int ISSUERS = 2;                   // MMA-issuing warps (an MMA costs its issuer ~50-100 cycles)
constexpr int COMPUTE_THREADS = 128;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t IDESC_SS = idesc_f16_f32(BR, BS, 0, 0);   // resident x streamed^T, both K-major
constexpr uint32_t IDESC_TS = idesc_f16_f32(BR, D, 0, 1);    // A from TMEM, B N-major (N = d)

// dK/dV: stage = Q_n, dO_n, LSE2 and D of 64 queries (padded to 1 KB)
constexpr int VEC_BYTES = BS * 4;
constexpr int STAGE_KV = ((2 * TILE_S + 2 * VEC_BYTES + 1023) / 1024) * 1024;
constexpr int DKDV_SMEM = 1024 + 2 * TILE_R + NST_KV * STAGE_KV + STAGING + 256;
// dQ: stage = K_n, V_n of 64 keys
constexpr int STAGE_Q = 2 * TILE_S;
constexpr int DQ_SMEM = 1024 + 2 * TILE_R + NST_Q * STAGE_Q + STAGING + 256;
// TMEM: score buffer b at b*128 (64 columns), its dP at b*128 + 64; accumulators at 256 (and 384)
constexpr uint32_t T_ACC0 = 256, T_ACC1 = 384;

// D[tmem] (+)= A[tmem] * B[smem desc], issued by the lane elect.sync picks (whole warp converged).
__device__ __forceinline__ void mma_ts_elect(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void load_3d(void* dst, const void* tmap, uint64_t* bar, int32_t x, int32_t y, int32_t z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::
          "r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

__device__ __forceinline__ void load_4d(void* dst, const void* tmap, uint64_t* bar, int32_t x, int32_t y, int32_t z,
                                        int32_t w) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6}], "
      "[%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z), "r"(w)
      : "memory");
}

// Plain bulk copy global -> shared (16-byte aligned, size a multiple of 16).
__device__ __forceinline__ void load_bulk(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// K-major tile (two 64-d halves of `half` bytes each), K step kk of 16 along d.
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t base, int kk, uint32_t half) {
  return smem_desc_sw128(base + (kk >> 2) * half + (kk & 3) * 32, 16, 1024);
}
// A streamed [64 rows x 128 d] tile read N-major (N = d), K step kk of 16 rows.
__device__ __forceinline__ uint64_t nmajor_desc(uint32_t base, int kk) {
  return smem_desc_sw128(base + kk * 16 * 128, HALF_S, 1024);
}

// D[128 x 64] = A[resident 128 x d] * B[streamed 64 x d]^T, both K-major in shared memory.
// Issued by an issuing warp (all lanes converged; one elected lane issues).
__device__ __forceinline__ void mma_ss_tile(uint32_t d_tmem, uint32_t a_base, uint32_t b_base) {
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk)
    mma_bf16_ss_elect(d_tmem, kmajor_desc(a_base, kk, HALF_R), kmajor_desc(b_base, kk, HALF_S), IDESC_SS,
                kk > 0 ? 1u : 0u);
}

// D[128 x d] (+)= A[tmem, 128 x 64 fp16] * B[streamed 64 x d, read N-major].  Issued by an
// issuing warp (all lanes converged; one elected lane issues).
__device__ __forceinline__ void mma_ts_tile(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_base, bool accumulate) {
#pragma unroll
  for (int kk = 0; kk < BS / 16; ++kk)
    mma_ts_elect(d_tmem, a_tmem + static_cast<uint32_t>(kk * 8), nmajor_desc(b_base, kk), IDESC_TS,
           (accumulate || kk > 0) ? 1u : 0u);
}

// Write a 128 x 128 gradient block (this thread's row r of it in v, times `scale`) as bf16:
// the rows go into a 128-byte-swizzled staging tile (two 64-column halves), and one thread
// sends the halves with TMA stores to columns x0 and x0 + 64 of rows y0.. of sequence z
// (the tensor map clips rows at S).  `blk` counts the blocks this CTA has stored.  stg_free
// completes once the previous block's stores have read the tile, stg_full once every row is
// in it; both waits are bounded.
__device__ __forceinline__ void store_block(const AttnBwdArgs& a, uint8_t* staging, uint64_t* stg_full,
                                            uint64_t* stg_free, int blk, int r, const uint32_t (&v)[4][32],
                                            float scale, int x0, int y0, int z, bool st_leader) {
  if (st_leader) {
    bulk_wait_group_read<0>();
    mbar_arrive(stg_free);
  }
  mbar_wait_bounded(stg_free, blk & 1, a.wait_limit_ns, a.status, WAIT_SITE_ATTN);
#pragma unroll
  for (int half = 0; half < 2; ++half) {
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {      // 16-byte chunk: 8 columns
      const int c = half * 2 + ch / 4;    // 32-column group of v
      const int i0 = (ch % 4) * 8;
      uint4 w;
      w.x = pack_bf16x2(__uint_as_float(v[c][i0 + 0]) * scale, __uint_as_float(v[c][i0 + 1]) * scale);
      w.y = pack_bf16x2(__uint_as_float(v[c][i0 + 2]) * scale, __uint_as_float(v[c][i0 + 3]) * scale);
      w.z = pack_bf16x2(__uint_as_float(v[c][i0 + 4]) * scale, __uint_as_float(v[c][i0 + 5]) * scale);
      w.w = pack_bf16x2(__uint_as_float(v[c][i0 + 6]) * scale, __uint_as_float(v[c][i0 + 7]) * scale);
      *reinterpret_cast<uint4*>(staging + half * HALF_R + r * 128 + ((ch ^ (r & 7)) * 16)) = w;
    }
  }
  fence_proxy_async_smem();
  mbar_arrive(stg_full);
  if (st_leader && mbar_wait_bounded(stg_full, blk & 1, a.wait_limit_ns, a.status, WAIT_SITE_ATTN)) {
    tma_store_3d(&a.tmOut, staging, x0, y0, z);
    tma_store_3d(&a.tmOut, staging + HALF_R, x0 + 64, y0, z);
    bulk_commit_group();
  }
}

// ------------------------------------------------------------------------ work items
// Both gradient kernels are persistent: one CTA per SM walks a list of 128-row blocks (key
// blocks for dK/dV, query blocks for dQ) of every (head, batch), numbered longest first under
// the causal mask; CTA c of G takes, in round r, item r*G + c (even r) or r*G + G-1-c (odd r).
// Barrier phases run on across items (a running count of items and one of streamed
// sub-blocks), so the next item's resident tiles load as soon as the current item's last score
// product has read them, and its first score products run while the compute warps still
// write the current item's gradients out.
struct BwdItem {
  int blk;          // key block (dK/dV) or query block (dQ)
  int head, b, bh;
  int sb0;          // first streamed sub-block
  int N;            // streamed sub-blocks
};

__device__ __forceinline__ bool bwd_item(const AttnBwdArgs& a, int r, bool kv, BwdItem& it) {
  const int nh = a.H - a.head0;
  const int per = nh * a.B;
  const int nb = (a.S + BR - 1) / BR;
  const int G = static_cast<int>(gridDim.x);
  const int c = static_cast<int>(blockIdx.x);
  const int idx = r * G + ((r & 1) ? G - 1 - c : c);
  if (idx >= nb * per) return false;
  const int ord = idx / per;            // 0: the longest blocks
  const int rem = idx - ord * per;
  it.head = a.head0 + rem % nh;
  it.b = rem / nh;
  it.bh = it.b * a.H + it.head;
  const int nsb_all = (a.S + BS - 1) / BS;
  if (kv) {
    it.blk = ord;                       // key block 0 is seen by every query
    it.sb0 = a.causal ? it.blk * BR / BS : 0;
    it.N = nsb_all - it.sb0;
  } else {
    it.blk = nb - 1 - ord;              // the last query block sees every key
    it.sb0 = 0;
    it.N = a.causal ? min(nsb_all, (it.blk * BR + BR - 1) / BS + 1) : nsb_all;
  }
  return true;
}

__device__ __forceinline__ int bwd_rounds(const AttnBwdArgs& a) {
  const int items = ((a.S + BR - 1) / BR) * (a.H - a.head0) * a.B;
  return (items + static_cast<int>(gridDim.x) - 1) / static_cast<int>(gridDim.x);
}

struct BwdBars {
  uint64_t *res_full, *res_empty, *st_full, *st_empty, *s_full, *p_full, *acc_full, *acc_empty, *drain;
  uint64_t *stg_full, *stg_free;
};

// Carve the barriers (and the TMEM slot) out of the shared memory after the stages.
template <int NSTG>
__device__ __forceinline__ BwdBars bwd_bars(uint8_t* base, uint32_t** tmem_slot, volatile int** abort_flag) {
  uint64_t* bars = reinterpret_cast<uint64_t*>(base);
  BwdBars z;
  z.res_full = bars;
  z.res_empty = bars + 1;
  z.st_full = bars + 2;                 // [NSTG]
  z.st_empty = bars + 2 + NSTG;          // [NSTG]
  z.s_full = bars + 2 + 2 * NSTG;        // [2] per score buffer
  z.p_full = bars + 4 + 2 * NSTG;        // [2] per score buffer, 128 arrivals
  z.acc_full = bars + 6 + 2 * NSTG;
  z.acc_empty = bars + 7 + 2 * NSTG;     // 128 arrivals
  z.drain = bars + 8 + 2 * NSTG;
  z.stg_full = bars + 9 + 2 * NSTG;     // 128 arrivals: a gradient block's rows are staged
  z.stg_free = bars + 10 + 2 * NSTG;    // the staging tile has been read by the last stores
  *tmem_slot = reinterpret_cast<uint32_t*>(bars + 11 + 2 * NSTG);
  *abort_flag = reinterpret_cast<volatile int*>(*tmem_slot + 1);
  return z;
}

template <int NSTG>
__device__ __forceinline__ void bwd_bars_init(const BwdBars& z, int ts_issuers) {
  mbar_init(z.res_full, 1);
  mbar_init(z.res_empty, ISSUERS);
  for (int i = 0; i < NSTG; ++i) {
    mbar_init(&z.st_full[i], 1);
    mbar_init(&z.st_empty[i], ISSUERS);
  }
  for (int i = 0; i < 2; ++i) {
    mbar_init(&z.s_full[i], ISSUERS);
    mbar_init(&z.p_full[i], COMPUTE_THREADS);
  }
  mbar_init(z.acc_full, ts_issuers);
  mbar_init(z.acc_empty, COMPUTE_THREADS);
  mbar_init(z.drain, ISSUERS);
  mbar_init(z.stg_full, COMPUTE_THREADS);
  mbar_init(z.stg_free, 1);
}

__device__ __forceinline__ bool bwait(uint64_t* bar, uint32_t parity, const AttnBwdArgs& a) {
  return mbar_wait_bounded(bar, parity, a.wait_limit_ns, a.status, WAIT_SITE_ATTN);
}
// The same wait taken by a whole issuing warp (one verdict for all lanes).
__device__ __forceinline__ bool bwait_warp(uint64_t* bar, uint32_t parity, const AttnBwdArgs& a) {
  return warp_wait_bounded(bar, parity, a.wait_limit_ns, a.status, WAIT_SITE_ATTN);
}

// One MMA-issuing warp's work on one item (all 32 lanes run it; one elected lane issues).
// Each kernel has two such warps with disjoint products: a single issuer issues an MMA every
// ~50-100 cycles whatever its size, below the tensor pipe's rate on these 64-wide tiles.  `issue_ss(n, g)` is this thread's score product of the
// item's sub-block n (running sub-block g, into score buffer g & 1), `issue_ts(n, g)` its
// gradient product (when `has_ts`), issued once the compute warps have written P and dS of
// g.  A score product into a buffer waits until the compute warps are done with the buffer's
// previous sub-block; every product reads or writes only this thread's own columns of a
// buffer, so tensor-pipe order within the thread is the only other order needed.  Stage g is
// released by each thread once its last reader of the stage completes (st_empty counts both
// threads); res_empty after the item's last score product (the resident tiles are free);
// acc_full after its last gradient product.  The first gradient product of an item
// overwrites the accumulator, so it waits until the compute warps have read out the previous
// item's (acc_empty).
template <int NSTG, typename SS, typename TS>
__device__ __forceinline__ bool issue_item(int N, int g0, int item, const BwdBars& z, const AttnBwdArgs& a,
                                           bool has_ts, SS issue_ss, TS issue_ts) {
  auto score = [&](int n) -> bool {
    const int g = g0 + n;
    if (g >= 2 && !bwait_warp(&z.p_full[g & 1], ((g - 2) >> 1) & 1, a)) return false;
    if (!bwait_warp(&z.st_full[g % NSTG], (g / NSTG) & 1, a)) return false;
    tc_fence_after();
    issue_ss(n, g);
    mma_commit_elect(&z.s_full[g & 1]);
    if (!has_ts) mma_commit_elect(&z.st_empty[g % NSTG]);
    if (n == N - 1) mma_commit_elect(z.res_empty);
    return true;
  };
  for (int n = 0; n < N && n < 2; ++n)
    if (!score(n)) return false;
  for (int n = 0; n < N; ++n) {
    const int g = g0 + n;
    if (has_ts) {
      if (!bwait_warp(&z.p_full[g & 1], (g >> 1) & 1, a)) return false;
      if (n == 0 && item > 0 && !bwait_warp(z.acc_empty, (item - 1) & 1, a)) return false;
      tc_fence_after();
      issue_ts(n, g);
      mma_commit_elect(&z.st_empty[g % NSTG]);
    }
    if (n + 2 < N && !score(n + 2)) return false;
  }
  if (has_ts) mma_commit_elect(z.acc_full);
  return true;
}

// ------------------------------------------------------------------------------ D
// D[bh][s] = sum_e dO[b*S+s][h*d+e] * O[b*S+s][h*d+e]: 16 threads per (row, head), 8 columns
// (16 bytes) each; the padding rows s in [S, S_pad) of D and LSE2 set to (0, +inf).
__global__ void __launch_bounds__(256) tp_attn_bwd_rowdot_kernel(const uint16_t* __restrict__ dO,
                                                                 const uint16_t* __restrict__ O, int o_f16,
                                                                 float* __restrict__ Dv, float* __restrict__ lse,
                                                                 int B, int S, int H, int S_pad) {
  pdl_wait();
  const int64_t item = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) / 16;
  const int sub = threadIdx.x % 16;
  const int64_t total = static_cast<int64_t>(B) * H * S_pad;
  float acc = 0.f;
  int s = 0;
  if (item < total) {
    s = static_cast<int>(item % S_pad);
    const int64_t bh = item / S_pad;
    const int h = static_cast<int>(bh % H);
    const int b = static_cast<int>(bh / H);
    if (s < S) {
      const int64_t off = (static_cast<int64_t>(b) * S + s) * (static_cast<int64_t>(H) * D) + h * D + sub * 8;
      const uint4 g = *reinterpret_cast<const uint4*>(dO + off);
      const uint4 o = *reinterpret_cast<const uint4*>(O + off);
      const uint32_t gw[4] = {g.x, g.y, g.z, g.w}, ow[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 gf = __half22float2(*reinterpret_cast<const __half2*>(&gw[k]));
        float o0, o1;
        if (o_f16) {
          const float2 of = __half22float2(*reinterpret_cast<const __half2*>(&ow[k]));
          o0 = of.x;
          o1 = of.y;
        } else {
          o0 = __uint_as_float(ow[k] << 16);
          o1 = __uint_as_float(ow[k] & 0xFFFF0000u);
        }
        acc = fmaf(gf.x, o0, acc);
        acc = fmaf(gf.y, o1, acc);
      }
    }
  }
#pragma unroll
  for (int m = 8; m > 0; m >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
  if (item < total && sub == 0) {
    Dv[item] = s < S ? acc : 0.f;
    if (s >= S) lse[item] = INFINITY;
  }
  pdl_launch_dependents();
}

// --------------------------------------------------------------------------- dK, dV
__global__ void __launch_bounds__(THREADS, 1) tp_attn_bwd_dkdv_kernel(const __grid_constant__ AttnBwdArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* sK = smem;
  uint8_t* sV = sK + TILE_R;
  uint8_t* sStage = sV + TILE_R;             // [NST_KV] x {Q_n, dO_n, LSE2[64], D[64]}
  uint8_t* sStaging = sStage + NST_KV * STAGE_KV;
  uint32_t* tmem_slot;
  volatile int* abort_flag;
  const BwdBars z = bwd_bars<NST_KV>(sStage + NST_KV * STAGE_KV + STAGING, &tmem_slot, &abort_flag);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int rounds = bwd_rounds(a);

  if (threadIdx.x == 0) {
    bwd_bars_init<NST_KV>(z, ISSUERS);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&a.tmK);
      tma_prefetch_desc(&a.tmV);
      tma_prefetch_desc(&a.tmQs);
      tma_prefetch_desc(&a.tmdOs);
      tma_prefetch_desc(&a.tmOut);
      int item = 0, g = 0;
      bool ok = true;
      for (int r = 0; r < rounds && ok; ++r) {
        BwdItem it;
        if (!bwd_item(a, r, true, it)) continue;
        const int k0 = it.blk * BR;
        // the resident K_j, V_j: after the previous item's last score product has read them
        if (item > 0 && !bwait(z.res_empty, (item - 1) & 1, a)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(z.res_full, 2 * TILE_R);
        load_3d(sK, &a.tmK, z.res_full, 0, k0, it.bh);
        load_3d(sK + HALF_R, &a.tmK, z.res_full, 64, k0, it.bh);
        load_3d(sV, &a.tmV, z.res_full, 0, k0, it.bh);
        load_3d(sV + HALF_R, &a.tmV, z.res_full, 64, k0, it.bh);
        for (int n = 0; n < it.N; ++n, ++g) {
          if (*abort_flag || !bwait(&z.st_empty[g % NST_KV], ((g / NST_KV) & 1) ^ 1u, a)) {
            ok = false;
            break;
          }
          const int q0 = (it.sb0 + n) * BS;
          uint8_t* stage = sStage + (g % NST_KV) * STAGE_KV;
          uint64_t* bar = &z.st_full[g % NST_KV];
          mbar_arrive_expect_tx(bar, 2 * TILE_S + 2 * VEC_BYTES);
          load_3d(stage, &a.tmQs, bar, 0, q0, it.bh);
          load_3d(stage + HALF_S, &a.tmQs, bar, 64, q0, it.bh);
          load_4d(stage + TILE_S, &a.tmdOs, bar, 0, it.head, q0, it.b);
          load_4d(stage + TILE_S + HALF_S, &a.tmdOs, bar, 64, it.head, q0, it.b);
          load_bulk(stage + 2 * TILE_S, a.lse + static_cast<int64_t>(it.bh) * a.S_pad + q0, VEC_BYTES, bar);
          load_bulk(stage + 2 * TILE_S + VEC_BYTES, a.Dv + static_cast<int64_t>(it.bh) * a.S_pad + q0, VEC_BYTES, bar);
        }
        ++item;
      }
      if (!ok) *abort_flag = 1;
      // our copies in flight complete before the CTA can exit
      if (item > 0) bwait(z.res_full, (item - 1) & 1, a);
      for (int j = g - NST_KV > 0 ? g - NST_KV : 0; j < g; ++j) bwait(&z.st_full[j % NST_KV], (j / NST_KV) & 1, a);
    }
  } else if (warp <= ISSUERS) {
    // issuer 0: S^T = K Q_n^T and dV += P^T dO_n (buffer columns 0..63);
    // issuer 1: dP^T = V dO_n^T and dK += dS^T Q_n (buffer columns 64..127)
    // (the whole warp runs the loop; one elected lane issues)
    {
      const uint32_t col = static_cast<uint32_t>((warp - 1) * 64);
      const uint32_t resA = smem_u32(warp == 1 ? sK : sV);
      const uint32_t ss_off = warp == 1 ? 0u : static_cast<uint32_t>(TILE_S);    // Q_n or dO_n
      const uint32_t ts_off = warp == 1 ? static_cast<uint32_t>(TILE_S) : 0u;    // dO_n or Q_n
      const uint32_t acc = tmem_base + (warp == 1 ? T_ACC0 : T_ACC1);
      int item = 0, g0 = 0;
      bool ok = true;
      for (int r = 0; r < rounds && ok; ++r) {
        BwdItem it;
        if (!bwd_item(a, r, true, it)) continue;
        ok = bwait_warp(z.res_full, item & 1, a);
        if (ok) {
          tc_fence_after();
          ok = issue_item<NST_KV>(
              it.N, g0, item, z, a, true,
              [&](int, int g) {
                const uint32_t st = smem_u32(sStage + (g % NST_KV) * STAGE_KV);
                const uint32_t buf = tmem_base + static_cast<uint32_t>((g & 1) * 128) + col;
                mma_ss_tile(buf, resA, st + ss_off);
              },
              [&](int n, int g) {
                const uint32_t st = smem_u32(sStage + (g % NST_KV) * STAGE_KV);
                const uint32_t buf = tmem_base + static_cast<uint32_t>((g & 1) * 128) + col;
                mma_ts_tile(acc, buf, st + ts_off, n > 0);
              });
        }
        g0 += it.N;
        ++item;
      }
      if (!ok) *abort_flag = 1;
      mma_commit_elect(z.drain);
      bwait_warp(z.drain, 0, a);
    }
  } else {
    // one key row per thread
    const bool st_leader = warp == ISSUERS + 1 && lane == 0;
    int blk = 0;                            // gradient blocks stored
    const int quad = warp & 3;
    const int r_in = quad * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const float sl2 = a.scale_log2;
    int item = 0, g = 0;
    bool ok = true;
    for (int rr = 0; rr < rounds && ok; ++rr) {
      BwdItem it;
      if (!bwd_item(a, rr, true, it)) continue;
      const int k0 = it.blk * BR;
      const int k = k0 + r_in;
      for (int n = 0; n < it.N; ++n, ++g) {
        const int bsel = g & 1;
        if (!__all_sync(0xffffffffu, bwait(&z.s_full[bsel], (g >> 1) & 1, a))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int q0 = (it.sb0 + n) * BS;
        const float* vec = reinterpret_cast<const float*>(sStage + (g % NST_KV) * STAGE_KV + 2 * TILE_S);
        const bool diag = a.causal && q0 < k0 + BR;     // sub-blocks with keys after some queries
        const uint32_t buf = tmem_base + lane_off + static_cast<uint32_t>(bsel * 128);
        uint32_t sv[2][32], gv[2][32];
        tmem_ld_32x32b_x32(buf, sv[0]);
        tmem_ld_32x32b_x32(buf + 32, sv[1]);
        tmem_ld_32x32b_x32(buf + 64, gv[0]);
        tmem_ld_32x32b_x32(buf + 96, gv[1]);
        tmem_ld_wait();
        uint32_t pk[32], dk[32];
        float gmax = 0.f;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float pr[2], ds[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int j = c * 32 + 2 * i + e;   // query within the sub-block
              float pv = ex2f(__uint_as_float(sv[c][2 * i + e]) * sl2 - vec[j]);
              if (diag && k > q0 + j) pv = 0.f;
              pr[e] = pv;
              ds[e] = pv * (__uint_as_float(gv[c][2 * i + e]) - vec[BS + j]);
              gmax = fmaxf(gmax, fabsf(ds[e]));
            }
            pk[c * 16 + i] = pack_f16x2(pr[0], pr[1]);
            dk[c * 16 + i] = pack_f16x2(ds[0], ds[1]);
          }
        }
        tmem_st_32x32b_x32(buf, pk);          // P^T over the scores' first 32 columns
        tmem_st_32x32b_x32(buf + 64, dk);     // dS^T over dP^T's first 32 columns
        note_f16_range(a.status, gmax, DEV_RANGE_ATTN_GRAD);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&z.p_full[bsel]);
      }
      if (!ok || !__all_sync(0xffffffffu, bwait(z.acc_full, item & 1, a))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t v[4][32];
      const int g_ = it.head / a.Hg, hl = it.head % a.Hg;
      const int x = g_ * 3 * a.Hg * D + hl * D;
      // dV (no scale), then dK (times 1/sqrt(d)); the accumulators are released once both
      // are in registers
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld_32x32b_x32(tmem_base + lane_off + T_ACC0 + c * 32, v[c]);
      tmem_ld_wait();
      store_block(a, sStaging, z.stg_full, z.stg_free, blk++, r_in, v, 1.f, x + 2 * a.Hg * D, k0, it.b, st_leader);
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld_32x32b_x32(tmem_base + lane_off + T_ACC1 + c * 32, v[c]);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(z.acc_empty);
      store_block(a, sStaging, z.stg_full, z.stg_free, blk++, r_in, v, a.scale, x + a.Hg * D, k0, it.b, st_leader);
      ++item;
    }
    if (!ok) *abort_flag = 1;
    if (st_leader) bulk_wait_group_all();   // our output stores are complete before exit
  }

  pdl_launch_dependents();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ------------------------------------------------------------------------------- dQ
__global__ void __launch_bounds__(THREADS, 1) tp_attn_bwd_dq_kernel(const __grid_constant__ AttnBwdArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* sQ = smem;
  uint8_t* sdO = sQ + TILE_R;
  uint8_t* sStage = sdO + TILE_R;            // [NST_Q] x {K_n, V_n}
  uint8_t* sStaging = sStage + NST_Q * STAGE_Q;
  uint32_t* tmem_slot;
  volatile int* abort_flag;
  const BwdBars z = bwd_bars<NST_Q>(sStage + NST_Q * STAGE_Q + STAGING, &tmem_slot, &abort_flag);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int rounds = bwd_rounds(a);

  if (threadIdx.x == 0) {
    bwd_bars_init<NST_Q>(z, 1);      // the dQ product comes from issuer 0 alone
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&a.tmQ);
      tma_prefetch_desc(&a.tmdO);
      tma_prefetch_desc(&a.tmKs);
      tma_prefetch_desc(&a.tmVs);
      tma_prefetch_desc(&a.tmOut);
      int item = 0, g = 0;
      bool ok = true;
      for (int r = 0; r < rounds && ok; ++r) {
        BwdItem it;
        if (!bwd_item(a, r, false, it)) continue;
        const int q0 = it.blk * BR;
        if (item > 0 && !bwait(z.res_empty, (item - 1) & 1, a)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(z.res_full, 2 * TILE_R);
        load_3d(sQ, &a.tmQ, z.res_full, 0, q0, it.bh);
        load_3d(sQ + HALF_R, &a.tmQ, z.res_full, 64, q0, it.bh);
        load_4d(sdO, &a.tmdO, z.res_full, 0, it.head, q0, it.b);
        load_4d(sdO + HALF_R, &a.tmdO, z.res_full, 64, it.head, q0, it.b);
        for (int n = 0; n < it.N; ++n, ++g) {
          if (*abort_flag || !bwait(&z.st_empty[g % NST_Q], ((g / NST_Q) & 1) ^ 1u, a)) {
            ok = false;
            break;
          }
          const int k0 = (it.sb0 + n) * BS;
          uint8_t* stage = sStage + (g % NST_Q) * STAGE_Q;
          uint64_t* bar = &z.st_full[g % NST_Q];
          mbar_arrive_expect_tx(bar, 2 * TILE_S);
          load_3d(stage, &a.tmKs, bar, 0, k0, it.bh);
          load_3d(stage + HALF_S, &a.tmKs, bar, 64, k0, it.bh);
          load_3d(stage + TILE_S, &a.tmVs, bar, 0, k0, it.bh);
          load_3d(stage + TILE_S + HALF_S, &a.tmVs, bar, 64, k0, it.bh);
        }
        ++item;
      }
      if (!ok) *abort_flag = 1;
      if (item > 0) bwait(z.res_full, (item - 1) & 1, a);
      for (int j = g - NST_Q > 0 ? g - NST_Q : 0; j < g; ++j) bwait(&z.st_full[j % NST_Q], (j / NST_Q) & 1, a);
    }
  } else if (warp <= ISSUERS) {
    // issuer 0: S = Q K_n^T and dQ += dS K_n (buffer columns 0..63); issuer 1: dP = dO V_n^T
    // (the whole warp runs the loop; one elected lane issues)
    {
      const uint32_t col = static_cast<uint32_t>((warp - 1) * 64);
      const uint32_t resA = smem_u32(warp == 1 ? sQ : sdO);
      const uint32_t ss_off = warp == 1 ? 0u : static_cast<uint32_t>(TILE_S);    // K_n or V_n
      int item = 0, g0 = 0;
      bool ok = true;
      for (int r = 0; r < rounds && ok; ++r) {
        BwdItem it;
        if (!bwd_item(a, r, false, it)) continue;
        ok = bwait_warp(z.res_full, item & 1, a);
        if (ok) {
          tc_fence_after();
          ok = issue_item<NST_Q>(
              it.N, g0, item, z, a, warp == 1,
              [&](int, int g) {
                const uint32_t st = smem_u32(sStage + (g % NST_Q) * STAGE_Q);
                const uint32_t buf = tmem_base + static_cast<uint32_t>((g & 1) * 128) + col;
                mma_ss_tile(buf, resA, st + ss_off);
              },
              [&](int n, int g) {
                const uint32_t st = smem_u32(sStage + (g % NST_Q) * STAGE_Q);
                const uint32_t buf = tmem_base + static_cast<uint32_t>((g & 1) * 128);
                mma_ts_tile(tmem_base + T_ACC0, buf, st, n > 0);
              });
        }
        g0 += it.N;
        ++item;
      }
      if (!ok) *abort_flag = 1;
      mma_commit_elect(z.drain);
      bwait_warp(z.drain, 0, a);
    }
  } else {
    // one query row per thread
    const bool st_leader = warp == ISSUERS + 1 && lane == 0;
    int blk = 0;                            // gradient blocks stored
    const int quad = warp & 3;
    const int r_in = quad * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const float sl2 = a.scale_log2;
    int item = 0, g = 0;
    bool ok = true;
    for (int rr = 0; rr < rounds && ok; ++rr) {
      BwdItem it;
      if (!bwd_item(a, rr, false, it)) continue;
      const int q0 = it.blk * BR;
      const int q = q0 + r_in;
      const float lse2 = a.lse[static_cast<int64_t>(it.bh) * a.S_pad + q];   // +inf past the sequence
      const float drow = a.Dv[static_cast<int64_t>(it.bh) * a.S_pad + q];
      for (int n = 0; n < it.N; ++n, ++g) {
        const int bsel = g & 1;
        if (!__all_sync(0xffffffffu, bwait(&z.s_full[bsel], (g >> 1) & 1, a))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int k0 = (it.sb0 + n) * BS;
        // keys k0 + j with j <= lim are seen by this row (causal, and inside the sequence)
        const int lim = min(a.causal ? q - k0 : BS - 1, a.S - 1 - k0);
        const bool whole = k0 + BS <= a.S && (!a.causal || k0 + BS - 1 <= q0);
        const uint32_t buf = tmem_base + lane_off + static_cast<uint32_t>(bsel * 128);
        uint32_t sv[2][32], gv[2][32];
        tmem_ld_32x32b_x32(buf, sv[0]);
        tmem_ld_32x32b_x32(buf + 32, sv[1]);
        tmem_ld_32x32b_x32(buf + 64, gv[0]);
        tmem_ld_32x32b_x32(buf + 96, gv[1]);
        tmem_ld_wait();
        uint32_t dk[32];
        float gmax = 0.f;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float ds[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int j = c * 32 + 2 * i + e;
              float pv = ex2f(__uint_as_float(sv[c][2 * i + e]) * sl2 - lse2);
              if (!whole && j > lim) pv = 0.f;
              ds[e] = pv * (__uint_as_float(gv[c][2 * i + e]) - drow);
              gmax = fmaxf(gmax, fabsf(ds[e]));
            }
            dk[c * 16 + i] = pack_f16x2(ds[0], ds[1]);
          }
        }
        tmem_st_32x32b_x32(buf, dk);          // dS over the scores' first 32 columns
        note_f16_range(a.status, gmax, DEV_RANGE_ATTN_GRAD);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&z.p_full[bsel]);
      }
      if (!ok || !__all_sync(0xffffffffu, bwait(z.acc_full, item & 1, a))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t v[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld_32x32b_x32(tmem_base + lane_off + T_ACC0 + c * 32, v[c]);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(z.acc_empty);
      const int g_ = it.head / a.Hg, hl = it.head % a.Hg;
      store_block(a, sStaging, z.stg_full, z.stg_free, blk++, r_in, v, a.scale, g_ * 3 * a.Hg * D + hl * D, q0, it.b,
                  st_leader);
      ++item;
    }
    if (!ok) *abort_flag = 1;
    if (st_leader) bulk_wait_group_all();   // our output stores are complete before exit
  }

  pdl_launch_dependents();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace

tp_status launch_attention_backward(const AttnBwdArgs& a, const uint16_t* dO, const uint16_t* O, int o_f16,
                                    cudaStream_t stream) {
  static int attr_set[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return TP_ERR_CUDA;
  if (dev < 64 && !attr_set[dev]) {
    if (cudaFuncSetAttribute(tp_attn_bwd_dkdv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, DKDV_SMEM) !=
            cudaSuccess ||
        cudaFuncSetAttribute(tp_attn_bwd_dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, DQ_SMEM) !=
            cudaSuccess)
      return set_error(TP_ERR_CUDA, "cudaFuncSetAttribute (attention backward shared memory) failed");
    attr_set[dev] = 1;
  }
  const int nh = a.H - a.head0;
  const int nb = (a.S + BR - 1) / BR;
  if (a.S <= 0 || a.B == 0 || nh <= 0) return TP_OK;
  // persistent: one CTA per SM (at most one per 128-row block)
  const long long items = static_cast<long long>(nb) * nh * a.B;
  const unsigned grid = static_cast<unsigned>(items < sm_count() ? items : sm_count());
  {
    const int64_t threads = static_cast<int64_t>(a.B) * a.H * a.S_pad * 16;
    const unsigned blocks = static_cast<unsigned>((threads + 255) / 256);
    trace_before(stream, "attn_bwd_rowdot");
    const tp_status st = launch_ex(tp_attn_bwd_rowdot_kernel, dim3(blocks), dim3(256), 0, stream, 1, dO, O, o_f16,
                                   a.Dv, a.lse, a.B, a.S, a.H, a.S_pad);
    if (st != TP_OK) return st;
    trace_after(stream, "attn_bwd_rowdot");
  }
  {
    trace_before(stream, "attn_bwd_dkdv");
    const tp_status st = launch_ex(tp_attn_bwd_dkdv_kernel, dim3(grid), dim3(THREADS), DKDV_SMEM, stream, 1, a);
    if (st != TP_OK) return st;
    trace_after(stream, "attn_bwd_dkdv");
  }
  {
    trace_before(stream, "attn_bwd_dq");
    const tp_status st = launch_ex(tp_attn_bwd_dq_kernel, dim3(grid), dim3(THREADS), DQ_SMEM, stream, 1, a);
    if (st != TP_OK) return st;
    trace_after(stream, "attn_bwd_dq");
  }
  return TP_OK;
}

}  // namespace tpb
