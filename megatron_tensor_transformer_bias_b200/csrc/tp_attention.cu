// Per-head causal (or full) attention with online softmax on tcgen05 tensor cores.
//
// "Tensor Parallelism > Combining Column and Row Parallelism", paragraphs on
// multi-head attention and head independence: each head attends over the full
// sequence on its own, so a head group's shard runs with no communication.
// All heads of all groups run in one launch; groups differ only in which
// heads they own.
//
// Two kernels compute the same result:
//  * tp_attention_tt_kernel (default): one CTA per SM takes two 128-query tiles that
//    share each 128-key K/V block; the tensor core works on one tile while the other
//    tile's softmax runs (layout and schedule above the kernel).
//  * tp_attention_kernel (TPB_ATTN_ONE_TILE=1): one 128-query tile per CTA, two CTAs
//    per SM, 64-key blocks, the score buffer double-buffered in tensor memory.
// Common to both: S = Q K^T and O += P V on the tensor core with fp32 accumulation in
// TMEM; one query row per softmax thread; P = exp2(s * log2(e)/sqrt(d) - m) in fp16
// written over its score buffer and read by the P V MMA straight from tensor memory.
// The running max m is only moved (and O, l rescaled in place) when a row's max grows
// by more than 2^8, so P stays <= 256 and the final O / l is unchanged; O never
// leaves TMEM until the end.
// Q, K, V are [B*H][S][d] fp16 (d = 128); O is written to [B*S, H*d] (bf16 or
// fp16), the layout the row-parallel output projection reads.  Q, K and P are
// fp16 because the scores' rounding error grows with |Q||K|: bf16 Q and K cost
// up to ~5e-3 relative error at hidden size 8192, fp16 about 8x less.
#include <cstdio>
#include <cstdlib>

#include "tp_internal.h"
#include "tp_ptx.cuh"

namespace tpb {

namespace {

constexpr int BQ = 128;                         // queries per CTA
constexpr int BKV = 64;                         // keys per block
constexpr int D = 128;                          // head dim
constexpr int Q_HALF = BQ * 64 * 2;             // [128 rows x 64 d] fp16 swizzled box: 16 KB
constexpr int Q_BYTES = 2 * Q_HALF;             // 32 KB
constexpr int KV_HALF = BKV * 64 * 2;           // [64 rows x 64 d]: 8 KB
constexpr int KV_BYTES = 2 * KV_HALF;           // 16 KB
constexpr int THREADS = 192;
constexpr int SOFTMAX_THREADS = 128;
constexpr int SMEM_BYTES = 1024 + Q_BYTES + 2 * KV_BYTES /*K*/ + KV_BYTES /*V*/ + 256;
constexpr uint32_t TMEM_COLS = 256;             // S0 [0,64), S1 [64,128), O [128,256); P_j over S_j
constexpr uint32_t O_COL = 128;
constexpr float RESCALE_LOG2 = 8.0f;            // move the running max only when it grows by > 2^8
constexpr uint32_t IDESC_S = idesc_f16_f32(BQ, BKV, 0, 0);   // Q K-major, K K-major (N = keys)
constexpr uint32_t IDESC_PV = idesc_f16_f32(BQ, D, 0, 1);    // P (TMEM, K-major), V N-major (N = d)

// D[tmem] (+)= A[tmem] * B[smem desc]: fp16 A read from tensor memory, lane = row,
// two 16-bit K elements per 32-bit column (the lower K index in the low half).
__device__ __forceinline__ void mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// mma_f16_ts issued by the lane elect.sync picks (whole warp converged).
__device__ __forceinline__ void mma_f16_ts_elect(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                                 uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d(void* smem_dst, const void* tmap, uint64_t* bar, int32_t x, int32_t y,
                                            int32_t z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::
          "r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// 2^x with the MUFU instruction (relative error ~2^-22; inputs below -126 give +0).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// (d0, d1) = (a0 * b + c, a1 * b + c) as one packed fp32x2 instruction
__device__ __forceinline__ void fma2_bc(float& d0, float& d1, float a0, float a1, float b, float c) {
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %4};\n\tmov.b64 rc, {%5, %5};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b), "f"(c));
}

// (s0, s1) += (a0, a1) as one packed fp32x2 instruction
__device__ __forceinline__ void add2_acc(float& s0, float& s1, float a0, float a1) {
  asm("{\n\t.reg .b64 ra, rs;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rs, {%0, %1};\n\t"
      "add.rn.f32x2 rs, rs, ra;\n\tmov.b64 {%0, %1}, rs;\n\t}"
      : "+f"(s0), "+f"(s1)
      : "f"(a0), "f"(a1));
}

__global__ void __launch_bounds__(THREADS, 2) tp_attention_kernel(const __grid_constant__ AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + Q_BYTES;              // [2] blocks
  uint8_t* sV = sK + 2 * KV_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + KV_BYTES);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;             // [2]
  uint64_t* k_empty = bars + 3;            // [2]
  uint64_t* v_full = bars + 5;
  uint64_t* v_empty = bars + 6;
  uint64_t* s_full = bars + 7;             // [2]
  // [2], by block parity: a softmax warp can finish block j+1 while another is still on
  // block j (P_j no longer waits for P_{j-1} V_{j-1}), so the two blocks' arrivals must
  // not meet on one barrier.  It cannot get two blocks ahead: S_{j+2} is issued only
  // after P_j V_j, which needs every arrival of block j.
  uint64_t* p_full = bars + 9;
  uint64_t* pv_done = bars + 11;
  uint64_t* drain_bar = bars + 12;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 13);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int nqb = (a.S + BQ - 1) / BQ;
  const int qb = nqb - 1 - static_cast<int>(blockIdx.x);  // longest causal rows first
  const int head = a.head0 + static_cast<int>(blockIdx.y);
  const int b = blockIdx.z;
  const int bh = b * a.H + head;
  const int q0 = qb * BQ;
  const int nkv_all = (a.S + BKV - 1) / BKV;
  const int nkv = a.causal ? min(nkv_all, (q0 + BQ - 1) / BKV + 1) : nkv_all;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&s_full[s], 1);
    }
    mbar_init(v_full, 1);
    mbar_init(v_empty, 1);
    mbar_init(&p_full[0], SOFTMAX_THREADS);
    mbar_init(&p_full[1], SOFTMAX_THREADS);
    mbar_init(pv_done, 1);
    mbar_init(drain_bar, 1);
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
  pdl_wait();  // Q, K, V come from the preceding projection kernel

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&a.tmQ);
      tma_prefetch_desc(&a.tmK);
      tma_prefetch_desc(&a.tmV);
      mbar_arrive_expect_tx(q_full, Q_BYTES);
      tma_load_3d(sQ, &a.tmQ, q_full, 0, q0, bh);
      tma_load_3d(sQ + Q_HALF, &a.tmQ, q_full, 64, q0, bh);
      int k_issued = 0, v_issued = 0;
      bool ok = true;
      // K runs up to two blocks ahead of V: K_j and K_{j+1} can be in flight while V_j
      // waits for P_{j-1} V_{j-1} to release the single V buffer.
      for (int j = 0; j <= nkv && ok; ++j) {
        if (*abort_flag) break;
        if (j < nkv) {
          const int ks = j & 1;
          if (!mbar_wait_bounded(&k_empty[ks], ((j >> 1) & 1) ^ 1u, a.wait_limit_ns, a.status, WAIT_SITE_ATTN)) {
            *abort_flag = 1; ok = false; break;
          }
          mbar_arrive_expect_tx(&k_full[ks], KV_BYTES);
          tma_load_3d(sK + ks * KV_BYTES, &a.tmK, &k_full[ks], 0, j * BKV, bh);
          tma_load_3d(sK + ks * KV_BYTES + KV_HALF, &a.tmK, &k_full[ks], 64, j * BKV, bh);
          ++k_issued;
        }
        if (j >= 1) {
          const int jv = j - 1;
          if (!mbar_wait_bounded(v_empty, (jv & 1) ^ 1u, a.wait_limit_ns, a.status, WAIT_SITE_ATTN)) {
            *abort_flag = 1; ok = false; break;
          }
          mbar_arrive_expect_tx(v_full, KV_BYTES);
          tma_load_3d(sV, &a.tmV, v_full, 0, jv * BKV, bh);
          tma_load_3d(sV + KV_HALF, &a.tmV, v_full, 64, jv * BKV, bh);
          ++v_issued;
        }
      }
      // wait for our own copies in flight
      mbar_wait_bounded(q_full, 0, a.wait_limit_ns, a.status, WAIT_SITE_ATTN);
      for (int j = k_issued - 2 > 0 ? k_issued - 2 : 0; j < k_issued; ++j)
        mbar_wait_bounded(&k_full[j & 1], (j >> 1) & 1, a.wait_limit_ns, a.status, WAIT_SITE_ATTN);
      if (v_issued > 0) mbar_wait_bounded(v_full, (v_issued - 1) & 1, a.wait_limit_ns, a.status, WAIT_SITE_ATTN);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t qa = smem_u32(sQ);
      const uint32_t va = smem_u32(sV);
      const uint32_t t_o = tmem_base + O_COL;
      bool ok = mbar_wait_bounded(q_full, 0, a.wait_limit_ns, a.status, WAIT_SITE_ATTN);
      if (!ok) *abort_flag = 1;
      for (int j = 0; j <= nkv && ok; ++j) {
        if (j < nkv) {
          const int ks = j & 1;
          if (!mbar_wait_bounded(&k_full[ks], (j >> 1) & 1, a.wait_limit_ns, a.status, WAIT_SITE_ATTN)) {
            *abort_flag = 1; ok = false; break;
          }
          // score buffer ks held S_{j-2}; the softmax released it with p_full(j-2), which this
          // thread already waited for before issuing P_{j-2} V_{j-2} (waiting again here could
          // see the barrier two phases on and stall)
          tc_fence_after();
          const uint32_t ka = smem_u32(sK + ks * KV_BYTES);
          const uint32_t t_s = tmem_base + static_cast<uint32_t>(ks * BKV);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t qoff = (kk >> 2) * Q_HALF + (kk & 3) * 32;
            const uint32_t koff = (kk >> 2) * KV_HALF + (kk & 3) * 32;
            mma_bf16_ss(t_s, smem_desc_sw128(qa + qoff, 16, 1024), smem_desc_sw128(ka + koff, 16, 1024), IDESC_S,
                        kk > 0 ? 1u : 0u);
          }
          mma_commit(&s_full[ks]);
          mma_commit(&k_empty[ks]);
        }
        if (j >= 1) {
          const int jp = j - 1;
          // P_{jp} written over S_{jp} (and O rescaled) by the softmax, V_{jp} loaded
          if (!mbar_wait_bounded(&p_full[jp & 1], (jp >> 1) & 1, a.wait_limit_ns, a.status, WAIT_SITE_ATTN) ||
              !mbar_wait_bounded(v_full, jp & 1, a.wait_limit_ns, a.status, WAIT_SITE_ATTN)) {
            *abort_flag = 1; ok = false; break;
          }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < BKV / 16; ++kk) {
            const uint32_t a_tmem = tmem_base + static_cast<uint32_t>((jp & 1) * BKV + kk * 8);
            mma_f16_ts(t_o, a_tmem, smem_desc_sw128(va + kk * 16 * 128, KV_HALF, 1024), IDESC_PV,
                       (jp > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(pv_done);
          mma_commit(v_empty);
        }
      }
      mma_commit(drain_bar);
      mbar_wait_bounded(drain_bar, 0, a.wait_limit_ns, a.status, WAIT_SITE_ATTN);
    }
  } else {
    // ------------------------------------------------------------ softmax + output (warps 2..5)
    const int sub = warp & 3;
    const int r = sub * 32 + lane;      // query row within the block
    const int q = q0 + r;
    const uint32_t lane_off = static_cast<uint32_t>(sub * 32) << 16;
    const uint32_t t_o = tmem_base + O_COL + lane_off;
    const float sl2 = a.scale_log2;
    float m_ref = -INFINITY;   // reference max of the scaled scores (log2 units)
    float l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < nkv && ok; ++j) {
      const int ks = j & 1;
      // waits are made warp-uniform: tcgen05.ld/st are warp-collective instructions
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(&s_full[ks], (j >> 1) & 1, a.wait_limit_ns, a.status,
                                                     WAIT_SITE_ATTN))) {
        *abort_flag = 1; ok = false; break;
      }
      tc_fence_after();
      const uint32_t t_s = tmem_base + lane_off + static_cast<uint32_t>(ks * BKV);
      const int k0 = j * BKV;
      uint32_t sr[2][32];
      tmem_ld_32x32b_x32(t_s, sr[0]);
      tmem_ld_32x32b_x32(t_s + 32, sr[1]);
      tmem_ld_wait();
      // Keys k0 + i with i <= lim are visible to this row (causal, and inside the
      // sequence); a block every row sees whole takes the mask-free path.
      const int lim = min(a.causal ? q - k0 : BKV - 1, a.S - 1 - k0);
      const bool whole = k0 + BKV <= a.S && (!a.causal || k0 + BKV - 1 <= q0);
      if (!whole) {
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (c * 32 + i > lim) sr[c][i] = __float_as_uint(-INFINITY);
      }
      // row max of the raw scores, then scaled (the scale is positive)
      float mx;
      {
        float m4[4] = {__uint_as_float(sr[0][0]), __uint_as_float(sr[0][1]), __uint_as_float(sr[1][0]),
                       __uint_as_float(sr[1][1])};
#pragma unroll
        for (int i = 2; i < 32; i += 2) {
          m4[0] = max3f(m4[0], __uint_as_float(sr[0][i]), __uint_as_float(sr[0][i + 1]));
          m4[1] = max3f(m4[1], __uint_as_float(sr[1][i]), __uint_as_float(sr[1][i + 1]));
        }
        mx = max3f(m4[0], m4[1], fmaxf(m4[2], m4[3])) * sl2;
      }
      const bool move = mx > m_ref + RESCALE_LOG2;
      const float m_new = move ? mx : m_ref;
      // O is rescaled only after P_{j-1} V_{j-1} is done (P_j goes over S_j, so nothing
      // else has to wait for it).  P_{j-2} V_{j-2} completed before S_j did, so the
      // barrier is at most one phase behind and the parity wait is exact.
      if (j > 0 && __any_sync(0xffffffffu, move)) {
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(pv_done, (j - 1) & 1, a.wait_limit_ns, a.status,
                                                       WAIT_SITE_ATTN))) {
          *abort_flag = 1; ok = false; break;
        }
        tc_fence_after();
        {
          const float alpha = move ? exp2f(m_ref - m_new) : 1.0f;
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld_32x32b_x32(t_o + c * 32, o);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st_32x32b_x32(t_o + c * 32, o);
          }
          tmem_st_wait();
          l_run *= alpha;
        }
      }
      const float m_use = m_new == -INFINITY ? 0.f : m_new;
      m_ref = m_new;
      // P = exp2(s * scale - m) in fp16, two keys per 32-bit column, stored over the first
      // 32 columns of S_j's buffer; masked scores are -inf and give 0.  The row sum is
      // taken over the fp32 values.
      float ls0 = 0.f, ls1 = 0.f;
      const float neg_m = -m_use;
      uint32_t pk[32];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float x0, x1;
          fma2_bc(x0, x1, __uint_as_float(sr[c][2 * i]), __uint_as_float(sr[c][2 * i + 1]), sl2, neg_m);
          const float e0 = ex2_approx(x0), e1 = ex2_approx(x1);
          add2_acc(ls0, ls1, e0, e1);
          pk[c * 16 + i] = pack_f16x2(e0, e1);
        }
      }
      tmem_st_32x32b_x32(t_s, pk);
      tmem_st_wait();
      const float lsum = ls0 + ls1;
      l_run += lsum;
      // publish P_j (tensor memory) to the tensor core; O is released with it
      tc_fence_before();
      mbar_arrive(&p_full[ks]);
    }
    if (ok && nkv > 0) {
      // all of O is complete when the MMA thread's final commit (after the last P V) lands;
      // pv_done could be two phases behind here, where its parity test is ambiguous
      if (__all_sync(0xffffffffu, mbar_wait_bounded(drain_bar, 0, a.wait_limit_ns, a.status, WAIT_SITE_ATTN))) {
        tc_fence_after();
        const float inv = 1.f / l_run;
        if (a.lse && q < a.S) a.lse[static_cast<int64_t>(bh) * a.lse_ld + q] = m_ref + log2f(l_run);
        uint16_t* dst = static_cast<uint16_t*>(a.O) + (static_cast<int64_t>(b) * a.S + q) * (a.H * D) + head * D;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld_32x32b_x32(t_o + c * 32, o);
          tmem_ld_wait();
          if (q < a.S) {
            if (a.o_f16) {
              float m = 0.f;
#pragma unroll
              for (int i = 0; i < 32; ++i) m = fmaxf(m, fabsf(__uint_as_float(o[i])));
              note_f16_range(a.status, m * inv, DEV_RANGE_ATTN_O);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              uint4 w;
              uint32_t* wp = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float lo = __uint_as_float(o[u * 8 + 2 * e]) * inv;
                const float hi = __uint_as_float(o[u * 8 + 2 * e + 1]) * inv;
                wp[e] = a.o_f16 ? pack_f16x2(lo, hi) : pack_bf16x2(lo, hi);
              }
              reinterpret_cast<uint4*>(dst + c * 32)[u] = w;
            }
          }
        }
      } else {
        *abort_flag = 1;
      }
    }
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


// ---------------------------------------------------------------------------------------
// Two query tiles per CTA, one persistent CTA per SM (the default kernel).
//
// A work item is (two 128-query tiles, head, batch); each CTA loops over its items
// (order and assignment above tt_item).  384 threads, all 512 TMEM columns:
//   warps 0..3   softmax and output of query tile 0, one row per thread
//   warps 4..7   softmax and output of query tile 1
//   warp 8       TMA: Q0 and Q1 per item, then K_j and V_j (two stages each, 128 keys per
//                block) in one running sequence across items
//   warp 9       TMEM allocation; issues every MMA (one lane elected per instruction)
//   warps 10, 11 idle (they only hand their registers to the softmax warps)
// Both tiles share each K/V block.  The MMA warp interleaves the tiles per key block:
//   O0 += P0_{j-1} V_{j-1};  S0_j = Q0 K_j^T;  O1 += P1_{j-1} V_{j-1};  S1_j = Q1 K_j^T
// so the tensor core works on one tile while the other tile's softmax runs.  Each score
// row (128 keys) stays in registers: the softmax warpgroups raise their register limit
// to 200 with setmaxnreg, the control warpgroup lowers its own to 104.
// S_t,j is issued after O_t += P_t,{j-1} V_{j-1} and its commit tracks every earlier MMA
// of the thread, so when S_t,j is ready the accumulator O_t is idle: the softmax of
// tile t rescales O_t in place (rarely, see RESCALE_LOG2) without another barrier.
// P_t,j is written in fp16 over the first 64 columns of S_t,j and read from tensor
// memory by the P V MMA; S_t,{j+1} overwrites it only after that MMA (same thread, in
// order).  Across items: the next item's Q_t load starts once the last S_t MMA of the
// current one has read Q_t (q_empty), and its first P V into O_t waits until the softmax
// warps have read O_t out (o_empty), so one item's output overlaps the next one's
// first score blocks.
namespace tt {

constexpr int BQ = 128;                    // queries per tile (two tiles per CTA)
constexpr int BK = 128;                    // keys per block
constexpr int Q_HALF = BQ * 64 * 2;        // [128 rows x 64 d] fp16, 128-byte swizzle: 16 KB
constexpr int Q_TILE = 2 * Q_HALF;         // 32 KB
constexpr int KV_HALF = BK * 64 * 2;       // 16 KB
constexpr int KV_BLOCK = 2 * KV_HALF;      // 32 KB
constexpr int THREADS = 384;
constexpr int SOFTMAX_THREADS = 128;       // per tile
constexpr int SMEM_BYTES = 1024 + 2 * Q_TILE + 4 * KV_BLOCK + 256;  // Q0 Q1, K x2, V x2, barriers
constexpr uint32_t TMEM_COLS = 512;        // S0 [0,128) S1 [128,256) O0 [256,384) O1 [384,512)
constexpr uint32_t O_COL = 256;
constexpr int SOFTMAX_REGS = 200;          // setmaxnreg targets; 2 * 200 + 104 = 3 * 168
constexpr int CONTROL_REGS = 104;
constexpr int MIN_LAUNCH_REGS = (2 * SOFTMAX_REGS + CONTROL_REGS + 2) / 3;
constexpr uint32_t IDESC_S = idesc_f16_f32(BQ, BK, 0, 0);    // Q K-major, K K-major (N = keys)
constexpr uint32_t IDESC_PV = idesc_f16_f32(BQ, D, 0, 1);    // P (TMEM), V N-major (N = d)

}  // namespace tt

// One work item = (pair of query tiles, head, batch).  Items are numbered longest first
// (pair index descending for causal attention); CTA c of G takes, in round r, item
// r*G + c for even r and r*G + G-1-c for odd r, which keeps the causal work per CTA
// within a few percent of the mean without a shared counter.
struct TtItem {
  int q0, bh, head, b;
  int n[2];   // key blocks of tile 0 and tile 1 (0 for a tile wholly past the sequence end)
  int n_max;
};

__device__ __forceinline__ bool tt_item(const AttnArgs& a, int r, TtItem& it) {
  const int hc = a.H - a.head0;
  const int per_pair = hc * a.B;
  const int npairs = (a.S + 2 * tt::BQ - 1) / (2 * tt::BQ);
  const int G = static_cast<int>(gridDim.x);
  const int c = static_cast<int>(blockIdx.x);
  const int idx = r * G + ((r & 1) ? G - 1 - c : c);
  if (idx >= npairs * per_pair) return false;
  const int pr = npairs - 1 - idx / per_pair;
  const int rem = idx % per_pair;
  it.head = a.head0 + rem % hc;
  it.b = rem / hc;
  it.bh = it.b * a.H + it.head;
  it.q0 = pr * 2 * tt::BQ;
  const int nkv_all = (a.S + tt::BK - 1) / tt::BK;
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int qt = it.q0 + t * tt::BQ;
    it.n[t] = qt >= a.S ? 0 : (a.causal ? min(nkv_all, qt / tt::BK + 1) : nkv_all);
  }
  it.n_max = max(it.n[0], it.n[1]);
  return true;
}

__device__ __forceinline__ int tt_rounds(const AttnArgs& a) {
  const int npairs = (a.S + 2 * tt::BQ - 1) / (2 * tt::BQ);
  const int items = npairs * (a.H - a.head0) * a.B;
  return (items + static_cast<int>(gridDim.x) - 1) / static_cast<int>(gridDim.x);
}

__global__ void __launch_bounds__(tt::THREADS, 1) tp_attention_tt_kernel(const __grid_constant__ AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* sQ = smem;                        // [2] tiles
  uint8_t* sK = sQ + 2 * tt::Q_TILE;         // [2] stages
  uint8_t* sV = sK + 2 * tt::KV_BLOCK;       // [2] stages
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + 2 * tt::KV_BLOCK);
  uint64_t* q_full = bars + 0;               // [2] per tile
  uint64_t* q_empty = bars + 2;              // [2] per tile: last S MMA of the item done
  uint64_t* k_full = bars + 4;               // [2] per stage
  uint64_t* k_empty = bars + 6;
  uint64_t* v_full = bars + 8;
  uint64_t* v_empty = bars + 10;
  uint64_t* s_full = bars + 12;              // [2] per tile
  uint64_t* p_full = bars + 14;              // [2] per tile, 128 arrivals
  uint64_t* o_done = bars + 16;              // [2] per tile: last P V of the item complete
  uint64_t* o_empty = bars + 18;             // [2] per tile, 128 arrivals: O_t read out
  uint64_t* drain_bar = bars + 20;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 21);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int rounds = tt_rounds(a);

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], tt::SOFTMAX_THREADS);
      mbar_init(&o_done[i], 1);
      mbar_init(&o_empty[i], tt::SOFTMAX_THREADS);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, tt::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();               // Q, K, V come from the preceding projection kernel
  pdl_launch_dependents();  // the next kernel still waits for this grid to finish

  if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(tt::CONTROL_REGS));
    if (warp == 8 && lane == 0) {
      // ------------------------------------------------------------ TMA producer
      tma_prefetch_desc(&a.tmQ);
      tma_prefetch_desc(&a.tmK);
      tma_prefetch_desc(&a.tmV);
      uint32_t nq[2] = {0, 0};  // Q tiles loaded so far, per tile slot
      int nk = 0, nv = 0;       // K and V blocks loaded so far (ring index)
      bool ok = true;
      for (int r = 0; r < rounds && ok; ++r) {
        TtItem it;
        if (!tt_item(a, r, it)) continue;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          if (it.n[t] == 0) continue;
          // the slot is free once the previous item's last S_t MMA has read it
          if (!mbar_wait_bounded(&q_empty[t], (nq[t] & 1) ^ 1u, a.wait_limit_ns, a.status, WAIT_SITE_ATTN)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&q_full[t], tt::Q_TILE);
          tma_load_3d(sQ + t * tt::Q_TILE, &a.tmQ, &q_full[t], 0, it.q0 + t * tt::BQ, it.bh);
          tma_load_3d(sQ + t * tt::Q_TILE + tt::Q_HALF, &a.tmQ, &q_full[t], 64, it.q0 + t * tt::BQ, it.bh);
          ++nq[t];
        }
        for (int j = 0; j < it.n_max && ok; ++j) {
          if (*abort_flag) {
            ok = false;
            break;
          }
          const int st = nk & 1;
          if (!mbar_wait_bounded(&k_empty[st], ((nk >> 1) & 1) ^ 1u, a.wait_limit_ns, a.status, WAIT_SITE_ATTN)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&k_full[st], tt::KV_BLOCK);
          tma_load_3d(sK + st * tt::KV_BLOCK, &a.tmK, &k_full[st], 0, j * tt::BK, it.bh);
          tma_load_3d(sK + st * tt::KV_BLOCK + tt::KV_HALF, &a.tmK, &k_full[st], 64, j * tt::BK, it.bh);
          ++nk;
          if (!mbar_wait_bounded(&v_empty[st], ((nv >> 1) & 1) ^ 1u, a.wait_limit_ns, a.status, WAIT_SITE_ATTN)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&v_full[st], tt::KV_BLOCK);
          tma_load_3d(sV + st * tt::KV_BLOCK, &a.tmV, &v_full[st], 0, j * tt::BK, it.bh);
          tma_load_3d(sV + st * tt::KV_BLOCK + tt::KV_HALF, &a.tmV, &v_full[st], 64, j * tt::BK, it.bh);
          ++nv;
        }
      }
      if (!ok) *abort_flag = 1;
      // wait for our own copies in flight before the CTA can exit
#pragma unroll
      for (int t = 0; t < 2; ++t)
        if (nq[t] > 0) mbar_wait_bounded(&q_full[t], (nq[t] - 1) & 1, a.wait_limit_ns, a.status, WAIT_SITE_ATTN);
      for (int j = max(0, nk - 2); j < nk; ++j)
        mbar_wait_bounded(&k_full[j & 1], (j >> 1) & 1, a.wait_limit_ns, a.status, WAIT_SITE_ATTN);
      for (int j = max(0, nv - 2); j < nv; ++j)
        mbar_wait_bounded(&v_full[j & 1], (j >> 1) & 1, a.wait_limit_ns, a.status, WAIT_SITE_ATTN);
    } else if (warp == 9) {
      // ------------------------------------------------------------ MMA issuer
      // The whole warp runs the loop (its values stay warp-uniform); one elected lane issues.
      // Shared-memory descriptors of every operand buffer, built once: an MMA's operand is
      // its buffer's descriptor plus the byte offset / 16 in the start-address field (the
      // field holds address / 16 in 14 bits; no buffer ends above 256 KB, so no carry).
      const uint64_t dq0 = smem_desc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t dq1 = smem_desc_sw128(smem_u32(sQ + tt::Q_TILE), 16, 1024);
      const uint64_t dk0 = smem_desc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t dk1 = smem_desc_sw128(smem_u32(sK + tt::KV_BLOCK), 16, 1024);
      const uint64_t dv0 = smem_desc_sw128(smem_u32(sV), tt::KV_HALF, 1024);
      const uint64_t dv1 = smem_desc_sw128(smem_u32(sV + tt::KV_BLOCK), tt::KV_HALF, 1024);
      uint32_t nq[2] = {0, 0};    // items per tile slot so far (Q loads, o_done / o_empty phases)
      uint32_t blk[2] = {0, 0};   // key blocks per tile slot so far (s_full / p_full phases)
      int gb = 0;                 // K/V ring index of the item's block 0
      bool ok = true;
      for (int r = 0; r < rounds && ok; ++r) {
        TtItem it;
        if (!tt_item(a, r, it)) continue;
        for (int j = 0; j <= it.n_max && ok; ++j) {
          const int gj = gb + j;
          bool v_ready = false, k_ready = false;
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            const uint32_t t_s = tmem_base + static_cast<uint32_t>(t * tt::BQ);
            if (j >= 1 && j <= it.n[t]) {
              // O_t += P_t,{j-1} V_{j-1}; the first one overwrites O_t, which the previous
              // item's epilogue must have read out
              const int jp = j - 1;
              const int gv = gb + jp;
              if (!warp_wait_bounded(&p_full[t], (blk[t] + jp) & 1, a.wait_limit_ns, a.status, WAIT_SITE_ATTN) ||
                  (jp == 0 && nq[t] > 0 &&
                   !warp_wait_bounded(&o_empty[t], (nq[t] - 1) & 1, a.wait_limit_ns, a.status, WAIT_SITE_ATTN)) ||
                  (!v_ready &&
                   !warp_wait_bounded(&v_full[gv & 1], (gv >> 1) & 1, a.wait_limit_ns, a.status, WAIT_SITE_ATTN))) {
                ok = false;
                break;
              }
              v_ready = true;
              tc_fence_after();
              const uint64_t vd = (gv & 1) ? dv1 : dv0;
              const uint32_t t_o = tmem_base + tt::O_COL + static_cast<uint32_t>(t * D);
#pragma unroll
              for (int kk = 0; kk < tt::BK / 16; ++kk)
                mma_f16_ts_elect(t_o, t_s + static_cast<uint32_t>(kk * 8), vd + static_cast<uint64_t>((kk * 16 * 128) >> 4),
                           tt::IDESC_PV, (jp > 0 || kk > 0) ? 1u : 0u);
              if (j == it.n[t]) mma_commit_elect(&o_done[t]);
            }
            if (j < it.n[t]) {
              // S_t,j = Q_t K_j^T
              if ((j == 0 &&
                   !warp_wait_bounded(&q_full[t], nq[t] & 1, a.wait_limit_ns, a.status, WAIT_SITE_ATTN)) ||
                  (!k_ready &&
                   !warp_wait_bounded(&k_full[gj & 1], (gj >> 1) & 1, a.wait_limit_ns, a.status, WAIT_SITE_ATTN))) {
                ok = false;
                break;
              }
              k_ready = true;
              tc_fence_after();
              const uint64_t qd = t ? dq1 : dq0;
              const uint64_t kd = (gj & 1) ? dk1 : dk0;
#pragma unroll
              for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t off_q = (kk >> 2) * tt::Q_HALF + (kk & 3) * 32;
                const uint32_t off_k = (kk >> 2) * tt::KV_HALF + (kk & 3) * 32;
                mma_bf16_ss_elect(t_s, qd + static_cast<uint64_t>(off_q >> 4), kd + static_cast<uint64_t>(off_k >> 4),
                            tt::IDESC_S, kk > 0 ? 1u : 0u);
              }
              mma_commit_elect(&s_full[t]);
              if (j == it.n[t] - 1) mma_commit_elect(&q_empty[t]);
            }
          }
          if (!ok) break;
          if (j >= 1) mma_commit_elect(&v_empty[(gj - 1) & 1]);
          if (j < it.n_max) mma_commit_elect(&k_empty[gj & 1]);
        }
#pragma unroll
        for (int t = 0; t < 2; ++t)
          if (it.n[t] > 0) {
            blk[t] += static_cast<uint32_t>(it.n[t]);
            ++nq[t];
          }
        gb += it.n_max;
      }
      if (!ok) *abort_flag = 1;
      mma_commit_elect(drain_bar);
      warp_wait_bounded(drain_bar, 0, a.wait_limit_ns, a.status, WAIT_SITE_ATTN);
    }
  } else {
    // ------------------------------------------------------------ softmax + output of tile t
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(tt::SOFTMAX_REGS));
    const int t = warp >> 2;
    const int quad = warp & 3;
    const int r_in = quad * 32 + lane;      // query row within the tile
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t t_s = tmem_base + lane_off + static_cast<uint32_t>(t * tt::BQ);
    const uint32_t t_o = tmem_base + lane_off + tt::O_COL + static_cast<uint32_t>(t * D);
    const float sl2 = a.scale_log2;
    uint32_t blk = 0, items = 0;            // key blocks and items of this tile slot so far
    bool ok = true;
    for (int rr = 0; rr < rounds && ok; ++rr) {
      TtItem it;
      if (!tt_item(a, rr, it)) continue;
      const int n = t == 0 ? it.n[0] : it.n[1];
      if (n == 0) continue;
      const int qt = it.q0 + t * tt::BQ;
      const int q = qt + r_in;
      float m_ref = -INFINITY;   // reference max of the scaled scores (log2 units)
      float l_run = 0.f;
      for (int j = 0; j < n && ok; ++j) {
        // waits are made warp-uniform: tcgen05.ld/st are warp-collective instructions
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(&s_full[t], (blk + j) & 1, a.wait_limit_ns, a.status,
                                                       WAIT_SITE_ATTN))) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t sr[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld_32x32b_x32(t_s + c * 32, sr[c]);
        tmem_ld_wait();
        const int k0 = j * tt::BK;
        // Keys k0 + i with i <= lim are visible to this row (causal, and inside the
        // sequence); a block every row of the tile sees whole takes the mask-free path.
        const int lim = min(a.causal ? q - k0 : tt::BK - 1, a.S - 1 - k0);
        const bool whole = k0 + tt::BK <= a.S && (!a.causal || k0 + tt::BK - 1 <= qt);
        if (!whole) {
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (c * 32 + i > lim) sr[c][i] = __float_as_uint(-INFINITY);
        }
        // row max of the raw scores (8 independent chains), then scaled (the scale is positive)
        float mc[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const int c4 = c >> 1, o = (c & 1) * 16;
          mc[c] = __uint_as_float(sr[c4][o]);
#pragma unroll
          for (int i = 1; i < 15; i += 2)
            mc[c] = max3f(mc[c], __uint_as_float(sr[c4][o + i]), __uint_as_float(sr[c4][o + i + 1]));
          mc[c] = fmaxf(mc[c], __uint_as_float(sr[c4][o + 15]));
        }
        const float mx =
            fmaxf(max3f(mc[0], mc[1], mc[2]), max3f(mc[3], max3f(mc[4], mc[5], mc[6]), mc[7])) * sl2;
        const bool move = mx > m_ref + RESCALE_LOG2;
        const float m_new = move ? mx : m_ref;
        // O_t is idle here: S_t,j was issued after O_t += P_t,{j-1} V_{j-1}, and its
        // commit tracks every earlier MMA of the issuing lane.  Rescale it in place.
        if (j > 0 && __any_sync(0xffffffffu, move)) {
          const float alpha = move ? exp2f(m_ref - m_new) : 1.0f;
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld_32x32b_x32(t_o + c * 32, o);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st_32x32b_x32(t_o + c * 32, o);
          }
          tmem_st_wait();
          l_run *= alpha;
        }
        const float m_use = m_new == -INFINITY ? 0.f : m_new;
        m_ref = m_new;
        // P = exp2(s * scale - m) in fp16, two keys per 32-bit column, stored over the first
        // 64 columns of S_t's buffer; masked scores are -inf and give 0.  The row sum is
        // taken over the fp32 values.
        float ls0 = 0.f, ls1 = 0.f;
        const float neg_m = -m_use;
#pragma unroll
        for (int hlf = 0; hlf < 2; ++hlf) {
          uint32_t pk[32];
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              float x0, x1;
              fma2_bc(x0, x1, __uint_as_float(sr[hlf * 2 + cc][2 * i]),
                      __uint_as_float(sr[hlf * 2 + cc][2 * i + 1]), sl2, neg_m);
              const float e0 = ex2_approx(x0), e1 = ex2_approx(x1);
              add2_acc(ls0, ls1, e0, e1);
              pk[cc * 16 + i] = pack_f16x2(e0, e1);
            }
          }
          tmem_st_32x32b_x32(t_s + hlf * 32, pk);
        }
        tmem_st_wait();
        l_run += ls0 + ls1;
        // publish P_t,j (tensor memory) to the tensor core; O_t is released with it
        tc_fence_before();
        mbar_arrive(&p_full[t]);
      }
      if (!ok) break;
      // epilogue: O_t / l to global, then hand O_t back to the MMA warp
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(&o_done[t], items & 1, a.wait_limit_ns, a.status,
                                                     WAIT_SITE_ATTN))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float inv = 1.f / l_run;
      if (a.lse && q < a.S) a.lse[static_cast<int64_t>(it.bh) * a.lse_ld + q] = m_ref + log2f(l_run);
      uint16_t* dst =
          static_cast<uint16_t*>(a.O) + (static_cast<int64_t>(it.b) * a.S + q) * (a.H * D) + it.head * D;
      uint32_t o[4][32];
#pragma unroll
      for (int c = 0; c < D / 32; ++c) tmem_ld_32x32b_x32(t_o + c * 32, o[c]);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&o_empty[t]);
      if (q < a.S) {
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          if (a.o_f16) {
            float m = 0.f;
#pragma unroll
            for (int i = 0; i < 32; ++i) m = fmaxf(m, fabsf(__uint_as_float(o[c][i])));
            note_f16_range(a.status, m * inv, DEV_RANGE_ATTN_O);
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            uint4 w;
            uint32_t* wp = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float lo = __uint_as_float(o[c][u * 8 + 2 * e]) * inv;
              const float hi = __uint_as_float(o[c][u * 8 + 2 * e + 1]) * inv;
              wp[e] = a.o_f16 ? pack_f16x2(lo, hi) : pack_bf16x2(lo, hi);
            }
            reinterpret_cast<uint4*>(dst + c * 32)[u] = w;
          }
        }
      }
      blk += static_cast<uint32_t>(n);
      ++items;
    }
    if (!ok) *abort_flag = 1;
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 9) {
    __syncwarp();
    tmem_dealloc(tmem_base, tt::TMEM_COLS);
  }
}

}  // namespace

// TPB_ATTN_ONE_TILE=1 selects the one-tile kernel (two CTAs per SM, 64-key blocks);
// by default each CTA takes two query tiles (one CTA per SM, 128-key blocks).
bool attention_one_tile() {
  static const int v = [] {
    const char* e = getenv("TPB_ATTN_ONE_TILE");
    return (e && e[0] == '1') ? 1 : 0;
  }();
  return v != 0;
}

int attention_kv_rows() { return attention_one_tile() ? BKV : tt::BK; }

tp_status launch_attention(const AttnArgs& a, cudaStream_t stream) {
  static int attr_set[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return TP_ERR_CUDA;
  const bool one = attention_one_tile();
  if (dev < 64 && !(attr_set[dev] & (one ? 1 : 2))) {
    if (one) {
      if (cudaFuncSetAttribute(tp_attention_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES) !=
          cudaSuccess)
        return TP_ERR_CUDA;
    } else {
      // setmaxnreg moves registers between the warpgroups of the launch: the softmax
      // warpgroups' raise must be covered by what the control warpgroup gives back, so
      // the kernel has to start with at least (2 * 232 + 40) / 3 registers per thread.
      cudaFuncAttributes fa;
      if (cudaFuncGetAttributes(&fa, tp_attention_tt_kernel) != cudaSuccess) return TP_ERR_CUDA;
      if (fa.numRegs < tt::MIN_LAUNCH_REGS) {
        char msg[160];
        snprintf(msg, sizeof(msg), "attention kernel built with %d registers per thread, its register split needs %d",
                 fa.numRegs, tt::MIN_LAUNCH_REGS);
        return set_error(TP_ERR_UNSUPPORTED, msg);
      }
      if (cudaFuncSetAttribute(tp_attention_tt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               tt::SMEM_BYTES) != cudaSuccess)
        return TP_ERR_CUDA;
    }
    attr_set[dev] |= one ? 1 : 2;
  }
  if (a.S <= 0 || a.B == 0 || a.H - a.head0 <= 0) return TP_OK;
  trace_before(stream, "attention");
  tp_status st;
  if (one) {
    const int nqb = (a.S + BQ - 1) / BQ;
    dim3 grid(nqb, a.H - a.head0, a.B);
    st = launch_ex(tp_attention_kernel, grid, dim3(THREADS), SMEM_BYTES, stream, 1, a);
  } else {
    // persistent: one CTA per SM (at most one per work item), items handed out longest first
    const int npairs = (a.S + 2 * tt::BQ - 1) / (2 * tt::BQ);
    const long long items = static_cast<long long>(npairs) * (a.H - a.head0) * a.B;
    dim3 grid(static_cast<unsigned>(items < sm_count() ? items : sm_count()));
    st = launch_ex(tp_attention_tt_kernel, grid, dim3(tt::THREADS), tt::SMEM_BYTES, stream, 1, a);
  }
  if (st != TP_OK) return st;
  trace_after(stream, "attention");
  return TP_OK;
}

}  // namespace tpb
