// Per-head causal (or full) attention with online softmax on tcgen05 tensor cores.
//
// "Tensor Parallelism > Combining Column and Row Parallelism", paragraphs on
// multi-head attention and head independence: each head attends over the full
// sequence on its own, so a head group's shard runs with no communication.
// All heads of all groups run in one launch; groups differ only in which
// heads they own.
//
// One CTA per (128 queries, head, batch), two CTAs per SM, 192 threads:
//   warp 0      TMA: Q once, then K_j (double-buffered) and V_j, 64 keys per block
//   warp 1      TMEM allocation; one thread issues S_j = Q K_j^T into one of two
//               TMEM score buffers, and O += P_j V_j into the TMEM output accumulator
//   warps 2..5  one query row per thread: row max of S_j, P_j = exp2(s - m) in
//               fp16 written back over S_j in tensor memory, row sum.
// O += P_j V_j reads P_j from tensor memory (A operand in TMEM) and V_j from shared
// memory, so P is double-buffered with the scores and the softmax of block j does not
// wait for P_{j-1} V_{j-1}.  While the softmax warps work on S_j, the tensor core
// already computes S_{j+1}.
// The running max is only moved (and O, l rescaled in place) when a row's max grows
// by more than 2^8, so P stays <= 256 and the final O / l is unchanged; O never
// leaves TMEM until the end.
// Q, K, V are [B*H][S][d] fp16 (d = 128); O is written to [B*S, H*d] (bf16 or
// fp16), the layout the row-parallel output projection reads.  Q, K and P are
// fp16 because the scores' rounding error grows with |Q||K|: bf16 Q and K cost
// up to ~5e-3 relative error at hidden size 8192, fp16 about 8x less.
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

}  // namespace

tp_status launch_attention(const AttnArgs& a, cudaStream_t stream) {
  static int attr_set[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return TP_ERR_CUDA;
  if (dev < 64 && !attr_set[dev]) {
    if (cudaFuncSetAttribute(tp_attention_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES) !=
        cudaSuccess)
      return TP_ERR_CUDA;
    attr_set[dev] = 1;
  }
  const int nqb = (a.S + BQ - 1) / BQ;
  if (nqb == 0 || a.B == 0) return TP_OK;
  dim3 grid(nqb, a.H - a.head0, a.B);
  trace_before(stream);
  const tp_status st = launch_ex(tp_attention_kernel, grid, dim3(THREADS), SMEM_BYTES, stream, 1, a);
  if (st != TP_OK) return st;
  trace_after(stream, "attention");
  return TP_OK;
}

}  // namespace tpb
