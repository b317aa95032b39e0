// Per-head causal (or full) attention with online softmax on tcgen05 tensor cores.
//
// "Tensor Parallelism > Combining Column and Row Parallelism", paragraphs on
// multi-head attention and head independence: each head attends over the full
// sequence on its own, so a head group's shard runs with no communication.
// All heads of all groups run in one launch; groups differ only in which
// heads they own.
//
// One CTA per (128-query block, head, batch), 192 threads:
//   warp 0      TMA: Q once, then K_j and V_j (128 keys each) into a 2-stage ring
//   warp 1      TMEM allocation; one thread issues S_j = Q K_j^T and PV_j = P_j V_j
//   warps 2..5  one query row per thread: row max and exp2 of S_j read from TMEM,
//               P_j (fp16) written to shared memory in the MMA's swizzled layout,
//               running max / sum, O kept in fp32 registers and rescaled per block.
// Q, K, V are [B*H][S][d] fp16 (d = 128); O is written to [B*S, H*d] (bf16 or
// fp16), the layout the row-parallel output projection reads.  Q, K and P are
// fp16 because the scores' rounding error grows with |Q||K|: bf16 Q and K cost
// up to ~5e-3 relative error at hidden size 8192, fp16 about 8x less.
#include "tp_internal.h"
#include "tp_ptx.cuh"

namespace tpb {

namespace {

constexpr int BQ = 128;      // queries per CTA
constexpr int BKV = 128;     // keys per block
constexpr int D = 128;       // head dim
constexpr int HALF_BYTES = 128 * 64 * 2;  // one [128 rows x 64 cols] bf16 swizzled box: 16 KB
constexpr int TILE_BYTES = 2 * HALF_BYTES;  // [128 x 128] bf16: 32 KB
constexpr int KV_STAGES = 2;
constexpr int THREADS = 192;
constexpr int SOFTMAX_THREADS = 128;
constexpr int SMEM_BYTES = 1024 + TILE_BYTES /*Q*/ + KV_STAGES * 2 * TILE_BYTES /*K,V*/ + TILE_BYTES /*P*/ + 256;
constexpr uint32_t TMEM_COLS = 256;  // S: [0,128), PV: [128,256)
constexpr uint32_t IDESC_S = idesc_f16_f32(BQ, BKV, 0, 0);    // Q K-major, K K-major (N = keys); fp16
constexpr uint32_t IDESC_PV = idesc_f16_f32(BQ, D, 0, 1);     // P K-major, V N-major (N = d); fp16

__device__ __forceinline__ void tma_load_3d(void* smem_dst, const void* tmap, uint64_t* bar, int32_t x, int32_t y,
                                            int32_t z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::
          "r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

__global__ void __launch_bounds__(THREADS, 1) tp_attention_kernel(const __grid_constant__ AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + TILE_BYTES;                       // [KV_STAGES] tiles
  uint8_t* sV = sK + KV_STAGES * TILE_BYTES;           // [KV_STAGES] tiles
  uint8_t* sP = sV + KV_STAGES * TILE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sP + TILE_BYTES);
  uint64_t* q_full = bars + 0;
  uint64_t* kv_full = bars + 1;               // [KV_STAGES]
  uint64_t* kv_empty = bars + 1 + KV_STAGES;  // [KV_STAGES]
  uint64_t* s_full = bars + 1 + 2 * KV_STAGES;
  uint64_t* p_full = s_full + 1;
  uint64_t* pv_full = s_full + 2;
  uint64_t* drain_bar = s_full + 3;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(s_full + 4);
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
    for (int s = 0; s < KV_STAGES; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(p_full, SOFTMAX_THREADS);
    mbar_init(pv_full, 1);
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

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&a.tmQ);
      tma_prefetch_desc(&a.tmK);
      tma_prefetch_desc(&a.tmV);
      mbar_arrive_expect_tx(q_full, TILE_BYTES);
      tma_load_3d(sQ, &a.tmQ, q_full, 0, q0, bh);
      tma_load_3d(sQ + HALF_BYTES, &a.tmQ, q_full, 64, q0, bh);
      int issued = 0;
      for (int j = 0; j < nkv; ++j) {
        const int st = j % KV_STAGES;
        const uint32_t ph = static_cast<uint32_t>(j / KV_STAGES) & 1u;
        if (*abort_flag) break;
        if (!mbar_wait_bounded(&kv_empty[st], ph ^ 1u, a.wait_limit_ns, a.status, WAIT_SITE_ATTN)) {
          *abort_flag = 1;
          break;
        }
        mbar_arrive_expect_tx(&kv_full[st], 2 * TILE_BYTES);
        uint8_t* k_dst = sK + st * TILE_BYTES;
        uint8_t* v_dst = sV + st * TILE_BYTES;
        tma_load_3d(k_dst, &a.tmK, &kv_full[st], 0, j * BKV, bh);
        tma_load_3d(k_dst + HALF_BYTES, &a.tmK, &kv_full[st], 64, j * BKV, bh);
        tma_load_3d(v_dst, &a.tmV, &kv_full[st], 0, j * BKV, bh);
        tma_load_3d(v_dst + HALF_BYTES, &a.tmV, &kv_full[st], 64, j * BKV, bh);
        ++issued;
      }
      // wait for our own copies in flight
      mbar_wait_bounded(q_full, 0, a.wait_limit_ns, a.status, WAIT_SITE_ATTN);
      for (int j = issued - KV_STAGES > 0 ? issued - KV_STAGES : 0; j < issued; ++j)
        mbar_wait_bounded(&kv_full[j % KV_STAGES], static_cast<uint32_t>(j / KV_STAGES) & 1u, a.wait_limit_ns,
                          a.status, WAIT_SITE_ATTN);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t qa = smem_u32(sQ);
      const uint32_t pa = smem_u32(sP);
      const uint32_t t_s = tmem_base;
      const uint32_t t_pv = tmem_base + 128;
      bool ok = mbar_wait_bounded(q_full, 0, a.wait_limit_ns, a.status, WAIT_SITE_ATTN);
      if (!ok) *abort_flag = 1;
      for (int j = 0; j <= nkv && ok; ++j) {
        if (j < nkv) {
          const int st = j % KV_STAGES;
          if (!mbar_wait_bounded(&kv_full[st], static_cast<uint32_t>(j / KV_STAGES) & 1u, a.wait_limit_ns,
                                 a.status, WAIT_SITE_ATTN)) {
            *abort_flag = 1; ok = false; break;
          }
        }
        if (j > 0) {
          // softmax has read S_{j-1} and PV_{j-2} and written P_{j-1}
          if (!mbar_wait_bounded(p_full, static_cast<uint32_t>(j - 1) & 1u, a.wait_limit_ns, a.status,
                                 WAIT_SITE_ATTN)) {
            *abort_flag = 1; ok = false; break;
          }
        }
        tc_fence_after();
        if (j < nkv) {
          const uint32_t ka = smem_u32(sK + (j % KV_STAGES) * TILE_BYTES);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * HALF_BYTES + (kk & 3) * 32;
            mma_bf16_ss(t_s, smem_desc_sw128(qa + off, 16, 1024), smem_desc_sw128(ka + off, 16, 1024), IDESC_S,
                        kk > 0 ? 1u : 0u);
          }
          mma_commit(s_full);
        }
        if (j > 0) {
          const int jp = j - 1;
          const uint32_t va = smem_u32(sV + (jp % KV_STAGES) * TILE_BYTES);
#pragma unroll
          for (int kk = 0; kk < BKV / 16; ++kk) {
            const uint32_t poff = (kk >> 2) * HALF_BYTES + (kk & 3) * 32;
            mma_bf16_ss(t_pv, smem_desc_sw128(pa + poff, 16, 1024),
                        smem_desc_sw128(va + kk * 16 * 128, HALF_BYTES, 1024), IDESC_PV, kk > 0 ? 1u : 0u);
          }
          mma_commit(pv_full);
          mma_commit(&kv_empty[jp % KV_STAGES]);
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
    const uint32_t t_s = tmem_base + lane_off;
    const uint32_t t_pv = tmem_base + 128 + lane_off;
    const float sl2 = a.scale_log2;
    float o[D];
#pragma unroll
    for (int i = 0; i < D; ++i) o[i] = 0.f;
    float m_run = -INFINITY;   // running max of scaled scores (log2 units)
    float l_run = 0.f;
    float alpha_pending = 0.f; // rescale factor to apply together with PV_{j-1}
    bool ok = true;
    uint8_t* p_row = sP + r * 128;
    const int rsw = r & 7;
    for (int j = 0; j < nkv && ok; ++j) {
      // waits are made warp-uniform: tcgen05.ld is a warp-collective instruction
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(s_full, static_cast<uint32_t>(j) & 1u, a.wait_limit_ns,
                                                     a.status, WAIT_SITE_ATTN))) {
        *abort_flag = 1; ok = false; break;
      }
      tc_fence_after();
      const int k0 = j * BKV;
      // pass 1: row max over visible keys
      float mx = -INFINITY;
#pragma unroll 1
      for (int c = 0; c < BKV / 32; ++c) {
        uint32_t sr[32];
        tmem_ld_32x32b_x32(t_s + c * 32, sr);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int kidx = k0 + c * 32 + i;
          const bool vis = kidx < a.S && (!a.causal || kidx <= q);
          if (vis) mx = fmaxf(mx, __uint_as_float(sr[i]) * sl2);
        }
      }
      const float m_new = fmaxf(m_run, mx);
      const float m_use = m_new == -INFINITY ? 0.f : m_new;
      const float alpha = exp2f(m_run - m_use);  // 0 on the first block
      // before overwriting sP: PV_{j-1} must be complete; fold it into O
      if (j > 0) {
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(pv_full, static_cast<uint32_t>(j - 1) & 1u,
                                                       a.wait_limit_ns, a.status, WAIT_SITE_ATTN))) {
          *abort_flag = 1; ok = false; break;
        }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t pr[32];
          tmem_ld_32x32b_x32(t_pv + c * 32, pr);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[c * 32 + i] = o[c * 32 + i] * alpha_pending + __uint_as_float(pr[i]);
        }
      }
      // pass 2: P = exp2(s - m), rounded to fp16, written in the 128B-swizzled K-major layout
      float lsum = 0.f;
#pragma unroll 1
      for (int c = 0; c < BKV / 32; ++c) {
        uint32_t sr[32];
        tmem_ld_32x32b_x32(t_s + c * 32, sr);
        tmem_ld_wait();
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float pv2[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int kidx = k0 + c * 32 + 2 * i + e;
            const bool vis = kidx < a.S && (!a.causal || kidx <= q);
            pv2[e] = vis ? exp2f(__uint_as_float(sr[2 * i + e]) * sl2 - m_use) : 0.f;
          }
          __half2 hb = __floats2half2_rn(pv2[0], pv2[1]);
          lsum += __low2float(hb) + __high2float(hb);
          pk[i] = *reinterpret_cast<uint32_t*>(&hb);
        }
        // 32 keys = 4 chunks of 8; key block (c*32)/64, chunk within the 128B row
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int key = c * 32 + u * 8;
          const int blk = key >> 6;
          const int chunk = (key & 63) >> 3;
          uint4* dst = reinterpret_cast<uint4*>(p_row + blk * HALF_BYTES + ((chunk ^ rsw) << 4));
          *dst = make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
        }
      }
      l_run = l_run * alpha + lsum;
      m_run = m_new;
      alpha_pending = alpha;
      // publish P_j to the tensor core (async proxy) and release S_j
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    if (ok && nkv > 0) {
      if (__all_sync(0xffffffffu, mbar_wait_bounded(pv_full, static_cast<uint32_t>(nkv - 1) & 1u,
                                                    a.wait_limit_ns, a.status, WAIT_SITE_ATTN))) {
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t pr[32];
          tmem_ld_32x32b_x32(t_pv + c * 32, pr);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[c * 32 + i] = o[c * 32 + i] * alpha_pending + __uint_as_float(pr[i]);
        }
        if (q < a.S) {
          const float inv = 1.f / l_run;
          uint16_t* dst = static_cast<uint16_t*>(a.O) + (static_cast<int64_t>(b) * a.S + q) * (a.H * D) + head * D;
          if (a.o_f16) {
#pragma unroll
            for (int c = 0; c < D / 8; ++c) {
              uint4 u;
              u.x = pack_f16x2(o[c * 8 + 0] * inv, o[c * 8 + 1] * inv);
              u.y = pack_f16x2(o[c * 8 + 2] * inv, o[c * 8 + 3] * inv);
              u.z = pack_f16x2(o[c * 8 + 4] * inv, o[c * 8 + 5] * inv);
              u.w = pack_f16x2(o[c * 8 + 6] * inv, o[c * 8 + 7] * inv);
              reinterpret_cast<uint4*>(dst)[c] = u;
            }
          } else {
#pragma unroll
            for (int c = 0; c < D / 8; ++c) {
              uint4 u;
              u.x = pack_bf16x2(o[c * 8 + 0] * inv, o[c * 8 + 1] * inv);
              u.y = pack_bf16x2(o[c * 8 + 2] * inv, o[c * 8 + 3] * inv);
              u.z = pack_bf16x2(o[c * 8 + 4] * inv, o[c * 8 + 5] * inv);
              u.w = pack_bf16x2(o[c * 8 + 6] * inv, o[c * 8 + 7] * inv);
              reinterpret_cast<uint4*>(dst)[c] = u;
            }
          }
        }
      } else {
        *abort_flag = 1;
      }
    }
  }

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
  tp_attention_kernel<<<grid, THREADS, SMEM_BYTES, stream>>>(a);
  if (cudaGetLastError() != cudaSuccess) return TP_ERR_CUDA;
  trace_after(stream, "attention");
  return TP_OK;
}

}  // namespace tpb
