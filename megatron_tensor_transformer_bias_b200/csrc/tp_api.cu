// C-ABI entry points of libtpblock (declared in include/tpblock.h): argument
// validation, workspace layout, tensor-map construction and the launch
// sequence of each block.  Every check runs before the first launch; a failed
// check returns an error code and launches nothing.
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <string>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "tp_internal.h"

namespace tpb {

// ---------------------------------------------------------------- per-device facts
__device__ uint32_t g_status_word;

namespace {
constexpr int MAX_DEV = 64;
int g_sm_count[MAX_DEV] = {0};
// Device address of g_status_word per device, looked up once.  A cudaDeviceReset
// unloads the module, so the cached address is stale after one: the library does not
// support resetting a device it has used.
std::atomic<uint32_t*> g_status_ptr[MAX_DEV];
std::atomic<uint64_t> g_wait_limit_ns{2000000000ull};
thread_local std::string t_last_error;

int current_device() {
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess) return -1;
  return d;
}

tp_status fail(tp_status s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
tp_status fail(tp_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  t_last_error = buf;
  return s;
}

// ---------------------------------------------------------------- tracing
struct TraceRec {
  const char* name;
  cudaEvent_t start, stop;
};
thread_local bool t_trace_on = false;
thread_local int t_trace_cap = 0;
thread_local std::vector<TraceRec> t_trace;
thread_local std::vector<cudaEvent_t> t_event_pool;
thread_local cudaEvent_t t_pending_start = nullptr;

cudaEvent_t pool_event(size_t i) {
  while (t_event_pool.size() <= i) {
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    t_event_pool.push_back(e);
  }
  return t_event_pool[i];
}
}  // namespace

int sm_count() {
  const int d = current_device();
  if (d < 0 || d >= MAX_DEV) return 148;
  if (!g_sm_count[d]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, d) != cudaSuccess || n <= 0) n = 148;
    g_sm_count[d] = n;
  }
  return g_sm_count[d];
}

uint32_t* device_status_ptr() {
  const int d = current_device();
  if (d < 0 || d >= MAX_DEV) return nullptr;
  uint32_t* cached = g_status_ptr[d].load();
  if (!cached) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
    cached = static_cast<uint32_t*>(p);
    g_status_ptr[d].store(cached);
  }
  return cached;
}

uint64_t wait_limit_ns() { return g_wait_limit_ns.load(); }

bool pdl_enabled() {
  static int v = -1;
  if (v < 0) {
    const char* e = getenv("TPB_PDL");
    v = (e && e[0] == '0') ? 0 : 1;
  }
  return v == 1;
}

tp_status set_error(tp_status s, const char* msg) {
  t_last_error = msg;
  return s;
}

// Every launch is also an NVTX range named after the kernel (start/end ranges, so an
// error return between the two cannot unbalance a stack); a profiler that records NVTX
// shows them on the host timeline, without one the calls do nothing.
thread_local nvtxRangeId_t t_nvtx_launch = 0;

void trace_before(cudaStream_t stream, const char* name) {
  t_nvtx_launch = nvtxRangeStartA(name);
  if (!t_trace_on || static_cast<int>(t_trace.size()) >= t_trace_cap) return;
  t_pending_start = pool_event(2 * t_trace.size());
  if (t_pending_start) cudaEventRecord(t_pending_start, stream);
}

void trace_after(cudaStream_t stream, const char* name) {
  if (t_nvtx_launch) {
    nvtxRangeEnd(t_nvtx_launch);
    t_nvtx_launch = 0;
  }
  if (!t_trace_on || !t_pending_start || static_cast<int>(t_trace.size()) >= t_trace_cap) return;
  cudaEvent_t stop = pool_event(2 * t_trace.size() + 1);
  if (!stop) return;
  cudaEventRecord(stop, stream);
  t_trace.push_back({name, t_pending_start, stop});
  t_pending_start = nullptr;
}

// ---------------------------------------------------------------- tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

tp_status make_tmap_2d(CUtensorMap* map, const void* base, int f16, uint64_t inner, uint64_t outer,
                       uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(TP_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                   const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(TP_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return TP_OK;
}

tp_status make_tmap_mn(CUtensorMap* map, const void* base, int f16, uint64_t mn_cols, uint64_t k_rows,
                       uint64_t row_stride_bytes) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(TP_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  // [k_rows, mn_cols] row-major seen as (64 columns of a block, k_rows, mn_cols / 64 blocks)
  cuuint64_t dims[3] = {64, k_rows, mn_cols / 64};
  cuuint64_t strides[2] = {row_stride_bytes, 128};
  cuuint32_t box[3] = {64, 64, 2};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                   const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(TP_ERR_CUDA, "cuTensorMapEncodeTiled(mn) failed (%d)", static_cast<int>(r));
  return TP_OK;
}

tp_status make_tmap_out(CUtensorMap* map, void* base, int f16, uint64_t cols, uint64_t rows,
                        uint64_t row_stride_bytes) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(TP_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                   CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(TP_ERR_CUDA, "cuTensorMapEncodeTiled(out) failed (%d)", static_cast<int>(r));
  return TP_OK;
}

// fp32 output map of a grouped GEMM: (cols, rows, groups) with the given row and group
// strides, box {16 columns, 32 rows, 1 group}, 64-byte swizzle: a tile's stores clip at its
// own group's edge.
tp_status make_tmap_out_f32_3d(CUtensorMap* map, void* base, uint64_t cols, uint64_t rows, uint64_t groups,
                               uint64_t row_stride_bytes, uint64_t group_stride_bytes) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(TP_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[3] = {cols, rows, groups};
  cuuint64_t strides[2] = {row_stride_bytes, group_stride_bytes};
  cuuint32_t box[3] = {16, 32, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(TP_ERR_CUDA, "cuTensorMapEncodeTiled(out f32) failed (%d)", static_cast<int>(r));
  return TP_OK;
}

static tp_status make_tmap_f16_3d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                                   uint64_t s1_bytes, uint64_t s2_bytes, uint32_t b0, uint32_t b1) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(TP_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {s1_bytes, s2_bytes};
  cuuint32_t box[3] = {b0, b1, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(TP_ERR_CUDA, "cuTensorMapEncodeTiled(3d) failed (%d)", static_cast<int>(r));
  return TP_OK;
}

tp_status make_tmap_attn(CUtensorMap* map, const void* base, int BH, int S, int d, uint32_t box_rows) {
  // [B*H][S][d] fp16: inner d (box 64), then S (box box_rows), then heads (box 1).
  return make_tmap_f16_3d(map, base, static_cast<uint64_t>(d), static_cast<uint64_t>(S),
                           static_cast<uint64_t>(BH), static_cast<uint64_t>(d) * 2,
                           static_cast<uint64_t>(S) * d * 2, 64, box_rows);
}

// [B*S, H*d] fp16 (token rows, head-major columns) seen as (d, H, S, B): box {64, 1, rows, 1}
// is `rows` rows of one head's 64 columns, the same shared-memory tile as make_tmap_attn's.
tp_status make_tmap_rows_by_head(CUtensorMap* map, const void* base, int B, int S, int H, int d, uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(TP_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(S),
                        static_cast<cuuint64_t>(B)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(H) * d * 2,
                           static_cast<cuuint64_t>(S) * H * d * 2};
  cuuint32_t box[4] = {64, 1, box_rows, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(TP_ERR_CUDA, "cuTensorMapEncodeTiled(4d) failed (%d)", static_cast<int>(r));
  return TP_OK;
}

}  // namespace tpb

using namespace tpb;

// ---------------------------------------------------------------- validation helpers
namespace {

constexpr size_t WS_ALIGN = 256;
inline size_t align_up(size_t x) { return (x + WS_ALIGN - 1) / WS_ALIGN * WS_ALIGN; }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

tp_status check_ptr(const void* p, const char* what, bool need) {
  if (!p) return need ? fail(TP_ERR_INVALID_ARG, "%s is NULL", what) : TP_OK;
  if (!aligned16(p)) return fail(TP_ERR_INVALID_ARG, "%s is not 16-byte aligned", what);
  return TP_OK;
}

tp_status check_shards(const tp_shard* W, int t, int64_t cols, const char* what) {
  if (!W) return fail(TP_ERR_INVALID_ARG, "%s shard array is NULL", what);
  for (int i = 0; i < t; ++i) {
    if (W[i].dtype != TP_BF16 && W[i].dtype != TP_FP16)
      return fail(TP_ERR_INVALID_ARG, "%s[%d].dtype=%d (weights are TP_BF16 or TP_FP16)", what, i, W[i].dtype);
    if (W[i].dtype != W[0].dtype) return fail(TP_ERR_INVALID_ARG, "%s shards mix dtypes", what);
    if (!W[i].ptr) return fail(TP_ERR_INVALID_ARG, "%s[%d].ptr is NULL", what, i);
    if (!aligned16(W[i].ptr)) return fail(TP_ERR_INVALID_ARG, "%s[%d].ptr is not 16-byte aligned", what, i);
    if (W[i].ld < cols) return fail(TP_ERR_INVALID_ARG, "%s[%d].ld=%lld < %lld columns", what, i,
                                    static_cast<long long>(W[i].ld), static_cast<long long>(cols));
    if (W[i].ld % 8) return fail(TP_ERR_INVALID_ARG, "%s[%d].ld=%lld is not a multiple of 8", what, i,
                                 static_cast<long long>(W[i].ld));
  }
  return TP_OK;
}

tp_status check_bias_array(const void* const* b, int t, const char* what) {
  if (!b) return TP_OK;
  for (int i = 0; i < t; ++i)
    if (b[i] && !aligned16(b[i])) return fail(TP_ERR_INVALID_ARG, "%s[%d] is not 16-byte aligned", what, i);
  return TP_OK;
}

inline int is_f16(const tp_shard* W) { return W[0].dtype == TP_FP16 ? 1 : 0; }

#define TP_TRY(expr)                   \
  do {                                 \
    tp_status _s = (expr);             \
    if (_s != TP_OK) return _s;        \
  } while (0)

// ---------------------------------------------------------------- partials-mode workspace
// The row GEMM's fp32 partials [t, M, n], then the arrival counters of the in-epilogue
// reduction (one 32-bit word per 32-row x 128-column region of the output).
size_t row_partials_ws(int64_t M, int64_t n, int t) {
  return align_up(static_cast<size_t>(t) * M * n * 4) + align_up(partial_counter_count(M, n) * 4);
}
uint32_t* row_partials_counters(float* P, int64_t M, int64_t n, int t) {
  return reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(P) + align_up(static_cast<size_t>(t) * M * n * 4));
}

// Partials mode sums the t partials with the fixed-order reduce kernel after the row GEMM.
// TPB_REDUCE_IN_GEMM=1 takes the sum inside the row GEMM instead (the last shard's tiles add
// the stored partials 0..t-2 and their own; same order, same bits).  On one B200 the in-GEMM
// form is the slower one: the t-1 stored partials come back from DRAM in the last 1/t of
// the launch, when the row tiles of every region finish at once.
bool separate_reduce() {
  static int v = -1;
  if (v < 0) {
    const char* e = getenv("TPB_REDUCE_IN_GEMM");
    v = (e && e[0] == '1') ? 0 : 1;
  }
  return v == 1;
}

// Zero the arrival counters of a partials-mode row GEMM (before the sub-layer's first
// launch, so that its kernels stay chained by programmatic dependent launch).
tp_status zero_row_counters(float* P, int64_t M, int64_t n, int t, cudaStream_t stream) {
  if (separate_reduce()) return TP_OK;
  const cudaError_t e =
      cudaMemsetAsync(row_partials_counters(P, M, n, t), 0, partial_counter_count(M, n) * 4, stream);
  if (e != cudaSuccess) return fail(TP_ERR_CUDA, "cudaMemsetAsync of the reduction counters: %s", cudaGetErrorString(e));
  return TP_OK;
}

// ---------------------------------------------------------------- FFN (bf16)
size_t ffn_bf16_ws(int64_t M, int64_t h, int64_t f, int t, tp_reduce_mode mode) {
  size_t s = align_up(static_cast<size_t>(M) * f * 2);
  if (mode == TP_REDUCE_PARTIALS) s += row_partials_ws(M, h, t);
  return s;
}

tp_status validate_ffn_bf16_dims(int64_t M, int64_t h, int64_t f, int t) {
  if (M < 0 || h <= 0 || f <= 0) return fail(TP_ERR_INVALID_ARG, "sizes must be positive (M>=0)");
  if (t < 1 || t > TP_MAX_SHARDS) return fail(TP_ERR_INVALID_ARG, "t=%d outside [1, %d]", t, TP_MAX_SHARDS);
  if (f % t) return fail(TP_ERR_INVALID_ARG, "f=%lld is not divisible by t=%d", static_cast<long long>(f), t);
  if (h % 64) return fail(TP_ERR_UNSUPPORTED, "bf16 path needs h %% 64 == 0 (h=%lld)", static_cast<long long>(h));
  if ((f / t) % 64)
    return fail(TP_ERR_UNSUPPORTED, "bf16 path needs (f/t) %% 64 == 0 (f/t=%lld)", static_cast<long long>(f / t));
  if (M > (1LL << 31) - 1 || h > (1LL << 31) - 1 || f > (1LL << 31) - 1)
    return fail(TP_ERR_UNSUPPORTED, "dimension too large");
  return TP_OK;
}

// Column-parallel GEMM: out[:, g*ncol + n] = act(X W_g + b_g), X [M, k].
// X has W's dtype; out is written in out_type.
tp_status run_column(const void* X, int64_t M, int64_t k, int64_t ncol, int t, const tp_shard* W,
                     const void* const* b, int act, void* out, int out_type, int64_t ld_out, cudaStream_t stream) {
  GemmArgs a;
  memset(&a, 0, sizeof(a));
  const int f16 = is_f16(W);
  TP_TRY(make_tmap_2d(&a.tmA, X, f16, k, M, k * 2, 64, GEMM_BM));
  for (int i = 0; i < t; ++i) TP_TRY(make_tmap_mn(&a.tmB[i], W[i].ptr, f16, ncol, k, W[i].ld * 2));
  a.M = static_cast<int>(M); a.N = static_cast<int>(ncol); a.Kg = static_cast<int>(k); a.G = t;
  a.concat = 0; a.a_k_per_group = 0;
  a.epi = EPI_ACT; a.act = act; a.ab_f16 = f16;
  a.out = out; a.ld_out = ld_out; a.out_col_per_group = ncol; a.out_type = out_type;
  if (out_type != OUT_F32) {
    TP_TRY(make_tmap_out(&a.tmOut, out, out_type == OUT_F16, static_cast<uint64_t>(ld_out), M, ld_out * 2));
    a.tma_store = 1;
  }
  for (int i = 0; i < t; ++i) a.bias_g[i] = b ? b[i] : nullptr;
  a.status = device_status_ptr(); a.wait_limit_ns = wait_limit_ns();
  return launch_gemm(a, stream, "gemm_column_act");
}

// Row-parallel GEMM + reduction: out = sum_g A[:, g*kg:(g+1)*kg] W_g + bias + resid.
// A has W's dtype; out is bf16 or fp32 (out_fp32).
tp_status run_row(const void* A, int64_t M, int64_t kg, int64_t n, int t, const tp_shard* W, const void* bias,
                  const void* resid, int resid_fp32, void* out, int out_fp32, tp_reduce_mode mode, float* P,
                  cudaStream_t stream) {
  GemmArgs a;
  memset(&a, 0, sizeof(a));
  const int f16 = is_f16(W);
  TP_TRY(make_tmap_2d(&a.tmA, A, f16, kg * t, M, kg * t * 2, 64, GEMM_BM));
  for (int i = 0; i < t; ++i) TP_TRY(make_tmap_mn(&a.tmB[i], W[i].ptr, f16, n, kg, W[i].ld * 2));
  a.ab_f16 = f16;
  a.M = static_cast<int>(M); a.N = static_cast<int>(n); a.Kg = static_cast<int>(kg); a.G = t;
  a.a_k_per_group = static_cast<int>(kg);
  a.status = device_status_ptr(); a.wait_limit_ns = wait_limit_ns();
  if (mode == TP_REDUCE_FUSED) {
    a.concat = 1;
    a.epi = EPI_BIAS_RESID;
    a.out = out; a.ld_out = n; a.out_type = out_fp32 ? OUT_F32 : OUT_BF16;
    if (!out_fp32) {
      TP_TRY(make_tmap_out(&a.tmOut, out, 0, static_cast<uint64_t>(n), M, n * 2));
      a.tma_store = 1;
    }
    a.bias = bias; a.resid = resid; a.ld_resid = n; a.resid_fp32 = resid_fp32;
    return launch_gemm(a, stream, "gemm_row_fused_reduce");
  }
  a.concat = 0;
  a.epi = EPI_PARTIAL_F32;
  a.out = P; a.ld_out = n; a.out_group_stride = M * n;
  if (separate_reduce()) {
    TP_TRY(make_tmap_out_f32_3d(&a.tmOut, P, n, M, t, n * 4, M * n * 4));
    a.tma_store = 1;
    TP_TRY(launch_gemm(a, stream, "gemm_row_partials"));
    return launch_reduce_partials(P, t, M, n, bias, 0, resid, resid_fp32, out, out_fp32, stream);
  }
  // step 3 in the epilogue of the last shard's tiles: partials 0..t-2 are stored, the last
  // one is added to them straight from the accumulator, in the order 0..t-1
  a.counters = row_partials_counters(P, M, n, t);
  a.red_out = out; a.red_out_f32 = out_fp32;
  TP_TRY(make_tmap_out_f32_3d(&a.tmOut, P, n, M, t, n * 4, M * n * 4));
  a.tma_store = 1;
  if (!out_fp32) TP_TRY(make_tmap_out(&a.tmOut2, out, 0, static_cast<uint64_t>(n), M, n * 2));
  a.bias = bias; a.resid = resid; a.ld_resid = n; a.resid_fp32 = resid_fp32;
  return launch_gemm(a, stream, "gemm_row_partials");
}

// X has W1's dtype; act(Z) is stored in W2's dtype.
tp_status ffn_bf16(const void* X, int64_t M, int64_t h, int64_t f, int t, const tp_shard* W1,
                   const void* const* b1, const tp_shard* W2, const void* b2, const void* resid, int resid_fp32,
                   void* out, int out_fp32, tp_reduce_mode mode, int act, void* ws, cudaStream_t stream) {
  if (M == 0) return TP_OK;
  const int64_t fs = f / t;
  uint16_t* Zh = static_cast<uint16_t*>(ws);
  float* P = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + align_up(static_cast<size_t>(M) * f * 2));
  if (mode == TP_REDUCE_PARTIALS) TP_TRY(zero_row_counters(P, M, h, t, stream));
  TP_TRY(run_column(X, M, h, fs, t, W1, b1, act, Zh, is_f16(W2) ? OUT_F16 : OUT_BF16, f, stream));
  return run_row(Zh, M, fs, h, t, W2, b2, resid, resid_fp32, out, out_fp32, mode, P, stream);
}

tp_status validate_ffn(const void* X, int64_t M, int64_t h, int64_t f, int t, const tp_shard* W1,
                       const void* const* b1, const tp_shard* W2, const void* b2, const void* residual, void* out,
                       tp_dtype dtype, tp_reduce_mode mode, int act, void* ws, size_t ws_bytes) {
  if (dtype != TP_BF16 && dtype != TP_FP32) return fail(TP_ERR_INVALID_ARG, "unknown dtype %d", dtype);
  if (mode != TP_REDUCE_FUSED && mode != TP_REDUCE_PARTIALS) return fail(TP_ERR_INVALID_ARG, "unknown mode");
  if (act != TP_ACT_GELU && act != TP_ACT_RELU) return fail(TP_ERR_INVALID_ARG, "unknown activation %d", act);
  if (dtype == TP_BF16) {
    TP_TRY(validate_ffn_bf16_dims(M, h, f, t));
  } else {
    if (M < 0 || h <= 0 || f <= 0) return fail(TP_ERR_INVALID_ARG, "sizes must be positive (M>=0)");
    if (t < 1 || t > TP_MAX_SHARDS) return fail(TP_ERR_INVALID_ARG, "t=%d outside [1, %d]", t, TP_MAX_SHARDS);
    if (f % t) return fail(TP_ERR_INVALID_ARG, "f is not divisible by t");
    if (h % 4) return fail(TP_ERR_UNSUPPORTED, "fp32 path needs h %% 4 == 0");
    if (M * (f > h ? f : h) > (1LL << 31) || M > 65535LL * 16)
      return fail(TP_ERR_UNSUPPORTED, "fp32 path is for small blocks");
  }
  TP_TRY(check_ptr(X, "X", true));
  TP_TRY(check_ptr(out, "out", true));
  TP_TRY(check_ptr(b2, "b2", false));
  TP_TRY(check_ptr(residual, "residual", false));
  if (out == X || (residual && out == residual)) return fail(TP_ERR_INVALID_ARG, "out aliases an input");
  TP_TRY(check_shards(W1, t, f / t, "W1"));
  TP_TRY(check_shards(W2, t, h, "W2"));
  TP_TRY(check_bias_array(b1, t, "b1"));
  if (dtype == TP_BF16 && is_f16(W1)) return fail(TP_ERR_INVALID_ARG, "W1 must have X's dtype (bf16)");
  if (dtype == TP_FP32 && (W1[0].dtype != TP_BF16 || W2[0].dtype != TP_BF16))
    return fail(TP_ERR_INVALID_ARG, "fp32 FFN: leave the shards' dtype field at 0");
  const size_t need = tp_ffn_workspace_bytes(M, h, f, t, dtype, mode);
  if (need && (!ws || ws_bytes < need))
    return fail(TP_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, ws ? ws_bytes : 0);
  if (ws && (reinterpret_cast<uintptr_t>(ws) % WS_ALIGN))
    return fail(TP_ERR_INVALID_ARG, "workspace is not 256-byte aligned");
  return TP_OK;
}

// ---------------------------------------------------------------- FFN backward (bf16)
// Workspace: act(Z) [M, f] bf16 | act'(Z) [M, f] fp16 | dZ [M, f] bf16.
struct FfnBwdWs {
  uint16_t *A, *G, *dZ;
};

size_t ffn_bwd_ws_bytes(int64_t M, int64_t h, int64_t f) {
  (void)h;
  const size_t mf = align_up(static_cast<size_t>(M) * f * 2);
  return 3 * mf;
}

FfnBwdWs ffn_bwd_ws_layout(void* ws, int64_t M, int64_t f) {
  const size_t mf = align_up(static_cast<size_t>(M) * f * 2);
  uint8_t* p = static_cast<uint8_t*>(ws);
  return {reinterpret_cast<uint16_t*>(p), reinterpret_cast<uint16_t*>(p + mf), reinterpret_cast<uint16_t*>(p + 2 * mf)};
}

tp_status ffn_backward_bf16(const void* X, int64_t M, int64_t h, int64_t f, int t, const tp_shard* W1,
                            const void* const* b1, const tp_shard* W2, const void* dY, const void* dX_add, void* dX,
                            float* dW1, float* db1, float* dW2, float* db2, int act, void* ws, cudaStream_t stream) {
  const int64_t fs = f / t;
  FfnBwdWs w = ffn_bwd_ws_layout(ws, M, f);
  uint32_t* status = device_status_ptr();
  const uint64_t lim = wait_limit_ns();
  // 1. recompute step 1: act(Z_i) (bf16) and act'(Z_i) (fp16), Z_i = X W1_i + b1_i
  {
    GemmArgs a;
    memset(&a, 0, sizeof(a));
    TP_TRY(make_tmap_2d(&a.tmA, X, 0, h, M, h * 2, 64, GEMM_BM));
    for (int i = 0; i < t; ++i) TP_TRY(make_tmap_mn(&a.tmB[i], W1[i].ptr, 0, fs, h, W1[i].ld * 2));
    TP_TRY(make_tmap_out(&a.tmOut, w.A, 0, static_cast<uint64_t>(f), M, f * 2));
    TP_TRY(make_tmap_out(&a.tmOut2, w.G, 1, static_cast<uint64_t>(f), M, f * 2));
    a.M = static_cast<int>(M); a.N = static_cast<int>(fs); a.Kg = static_cast<int>(h); a.G = t;
    a.epi = EPI_ACT_GRAD; a.act = act;
    a.out = w.A; a.ld_out = f; a.out_col_per_group = fs; a.out_type = OUT_BF16; a.tma_store = 1;
    for (int i = 0; i < t; ++i) a.bias_g[i] = b1 ? b1[i] : nullptr;
    a.status = status; a.wait_limit_ns = lim;
    TP_TRY(launch_gemm(a, stream, "gemm_bwd_recompute"));
  }
  // 2. dZ_i = (dY W2_i^T) * act'(Z_i): the row layer's input gradient is local to each shard
  {
    GemmArgs a;
    memset(&a, 0, sizeof(a));
    TP_TRY(make_tmap_2d(&a.tmA, dY, 0, h, M, h * 2, 64, GEMM_BM));
    for (int i = 0; i < t; ++i) TP_TRY(make_tmap_2d(&a.tmB[i], W2[i].ptr, 0, h, fs, W2[i].ld * 2, 64, 128));
    TP_TRY(make_tmap_out(&a.tmOut, w.dZ, 0, static_cast<uint64_t>(f), M, f * 2));
    a.M = static_cast<int>(M); a.N = static_cast<int>(fs); a.Kg = static_cast<int>(h); a.G = t;
    a.b_kmajor = 1;
    a.epi = EPI_MUL_GRAD; a.grad_mul = w.G; a.ld_grad = f;
    a.out = w.dZ; a.ld_out = f; a.out_col_per_group = fs; a.out_type = OUT_BF16; a.tma_store = 1;
    a.status = status; a.wait_limit_ns = lim;
    TP_TRY(launch_gemm(a, stream, "gemm_bwd_dz"));
  }
  // 3. dW2_i = act(Z_i)^T dY (rows i*f/t.. of dW2)
  {
    GemmArgs a;
    memset(&a, 0, sizeof(a));
    TP_TRY(make_tmap_mn(&a.tmA, w.A, 0, f, M, f * 2));
    for (int i = 0; i < t; ++i) TP_TRY(make_tmap_mn(&a.tmB[i], dY, 0, h, M, h * 2));
    a.M = static_cast<int>(fs); a.N = static_cast<int>(h); a.Kg = static_cast<int>(M); a.G = t;
    a.a_mn = 1; a.a_m_per_group = static_cast<int>(fs);
    a.epi = EPI_PARTIAL_F32;
    a.out = dW2; a.ld_out = h; a.out_group_stride = fs * h;
    TP_TRY(make_tmap_out_f32_3d(&a.tmOut, dW2, h, fs, t, h * 4, fs * h * 4));
    a.tma_store = 1;
    a.status = status; a.wait_limit_ns = lim;
    TP_TRY(launch_gemm(a, stream, "gemm_bwd_dw2"));
  }
  // 4. dW1_i = X^T dZ_i (columns i*f/t.. of dW1)
  {
    GemmArgs a;
    memset(&a, 0, sizeof(a));
    TP_TRY(make_tmap_mn(&a.tmA, X, 0, h, M, h * 2));
    for (int i = 0; i < t; ++i) TP_TRY(make_tmap_mn(&a.tmB[i], w.dZ + i * fs, 0, fs, M, f * 2));
    a.M = static_cast<int>(h); a.N = static_cast<int>(fs); a.Kg = static_cast<int>(M); a.G = t;
    a.a_mn = 1; a.a_m_per_group = 0;
    a.epi = EPI_PARTIAL_F32;
    a.out = dW1; a.ld_out = f; a.out_group_stride = fs;
    TP_TRY(make_tmap_out_f32_3d(&a.tmOut, dW1, fs, h, t, f * 4, fs * 4));
    a.tma_store = 1;
    a.status = status; a.wait_limit_ns = lim;
    TP_TRY(launch_gemm(a, stream, "gemm_bwd_dw1"));
  }
  // 5. dX = sum_i dZ_i W1_i^T (+ dX_add): the column layer's input gradient is the sum over
  //    shards -- the backward pass's reduction, taken in one accumulator over the shards' K-slices
  {
    GemmArgs a;
    memset(&a, 0, sizeof(a));
    TP_TRY(make_tmap_2d(&a.tmA, w.dZ, 0, f, M, f * 2, 64, GEMM_BM));
    for (int i = 0; i < t; ++i) TP_TRY(make_tmap_2d(&a.tmB[i], W1[i].ptr, 0, fs, h, W1[i].ld * 2, 64, 128));
    TP_TRY(make_tmap_out(&a.tmOut, dX, 0, static_cast<uint64_t>(h), M, h * 2));
    a.M = static_cast<int>(M); a.N = static_cast<int>(h); a.Kg = static_cast<int>(fs); a.G = t;
    a.concat = 1; a.a_k_per_group = static_cast<int>(fs); a.b_kmajor = 1;
    a.epi = EPI_BIAS_RESID; a.bias = nullptr; a.resid = dX_add; a.ld_resid = h; a.resid_fp32 = 0;
    a.out = dX; a.ld_out = h; a.out_type = OUT_BF16; a.tma_store = 1;
    a.status = status; a.wait_limit_ns = lim;
    TP_TRY(launch_gemm(a, stream, "gemm_bwd_dx"));
  }
  // 6. bias gradients: column sums of dZ and dY in a fixed order
  if (db1) TP_TRY(launch_colsum(w.dZ, M, f, f, db1, stream));
  if (db2) TP_TRY(launch_colsum(dY, M, h, h, db2, stream));
  return TP_OK;
}

// ---------------------------------------------------------------- attention (bf16)
struct AttnWs {
  uint16_t *q, *k, *v, *o;
  float* P;
};

size_t attn_ws_bytes_i(int64_t B, int64_t S, int64_t h, int64_t H, int64_t d, int t, tp_reduce_mode mode) {
  const size_t qkv = align_up(static_cast<size_t>(B) * S * H * d * 2);
  size_t s = 4 * qkv;
  if (mode == TP_REDUCE_PARTIALS) s += row_partials_ws(B * S, h, t);
  return s;
}

AttnWs attn_ws_layout(void* ws, int64_t B, int64_t S, int64_t H, int64_t d) {
  const size_t qkv = align_up(static_cast<size_t>(B) * S * H * d * 2);
  uint8_t* p = static_cast<uint8_t*>(ws);
  AttnWs w;
  w.q = reinterpret_cast<uint16_t*>(p);
  w.k = reinterpret_cast<uint16_t*>(p + qkv);
  w.v = reinterpret_cast<uint16_t*>(p + 2 * qkv);
  w.o = reinterpret_cast<uint16_t*>(p + 3 * qkv);
  w.P = reinterpret_cast<float*>(p + 4 * qkv);
  return w;
}

tp_status validate_attn_dims(int B, int S, int h, int H, int d, int t) {
  if (B < 0 || S < 0 || h <= 0 || H <= 0 || d <= 0) return fail(TP_ERR_INVALID_ARG, "bad attention sizes");
  if (t < 1 || t > TP_MAX_SHARDS) return fail(TP_ERR_INVALID_ARG, "t=%d outside [1, %d]", t, TP_MAX_SHARDS);
  if (H % t) return fail(TP_ERR_INVALID_ARG, "heads=%d is not divisible by t=%d", H, t);
  if (d != 128) return fail(TP_ERR_UNSUPPORTED, "head dim d=%d (only 128 is implemented)", d);
  if (h % 64) return fail(TP_ERR_UNSUPPORTED, "h %% 64 != 0");
  if (((H / t) * d) % 64) return fail(TP_ERR_UNSUPPORTED, "(heads/t)*d %% 64 != 0");
  if (1LL * B * S > (1LL << 31) - 1 || B > 65535 || H > 65535) return fail(TP_ERR_UNSUPPORTED, "too many tokens");
  return TP_OK;
}

tp_status attn_bf16(const void* X, int B, int S, int h, int H, int d, int t, const tp_shard* Wqkv,
                    const void* const* bqkv, const tp_shard* Wo, const void* bo, const void* resid, int resid_fp32,
                    int causal, void* out, int out_fp32, tp_reduce_mode mode, void* ws, cudaStream_t stream) {
  const int64_t M = static_cast<int64_t>(B) * S;
  if (M == 0) return TP_OK;
  const int Hg = H / t;
  const int64_t ncol = 3LL * Hg * d;
  AttnWs w = attn_ws_layout(ws, B, S, H, d);
  if (mode == TP_REDUCE_PARTIALS) TP_TRY(zero_row_counters(w.P, M, h, t, stream));
  // QKV projection, column-parallel by head group, scattered to [B, H, S, d].
  {
    GemmArgs a;
    memset(&a, 0, sizeof(a));
    const int f16 = is_f16(Wqkv);  // X has Wqkv's dtype
    TP_TRY(make_tmap_2d(&a.tmA, X, f16, h, M, static_cast<uint64_t>(h) * 2, 64, GEMM_BM));
    for (int i = 0; i < t; ++i)
      TP_TRY(make_tmap_mn(&a.tmB[i], Wqkv[i].ptr, f16, ncol, h, Wqkv[i].ld * 2));
    a.ab_f16 = f16;
    a.M = static_cast<int>(M); a.N = static_cast<int>(ncol); a.Kg = h; a.G = t;
    a.concat = 0; a.a_k_per_group = 0;
    a.epi = EPI_QKV; a.act = ACT_NONE;
    for (int i = 0; i < t; ++i) a.bias_g[i] = bqkv ? bqkv[i] : nullptr;
    a.q = w.q; a.k = w.k; a.v = w.v; a.S = S; a.H = H; a.Hg = Hg; a.d = d;
    a.status = device_status_ptr(); a.wait_limit_ns = wait_limit_ns();
    TP_TRY(launch_gemm(a, stream, "gemm_qkv"));
  }
  // Per-head attention over every head (head groups are independent).
  {
    AttnArgs a;
    memset(&a, 0, sizeof(a));
    TP_TRY(make_tmap_attn(&a.tmQ, w.q, B * H, S, d, 128));  // 128-query tiles
    TP_TRY(make_tmap_attn(&a.tmK, w.k, B * H, S, d, attention_kv_rows()));  // key blocks of the kernel
    TP_TRY(make_tmap_attn(&a.tmV, w.v, B * H, S, d, attention_kv_rows()));
    a.O = w.o; a.o_f16 = is_f16(Wo);
    a.B = B; a.S = S; a.H = H; a.d = d; a.causal = causal; a.head0 = 0;
    a.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(d));
    a.status = device_status_ptr(); a.wait_limit_ns = wait_limit_ns();
    TP_TRY(launch_attention(a, stream));
  }
  // Output projection, row-parallel, and the reduction of the head groups' partials.
  return run_row(w.o, M, static_cast<int64_t>(Hg) * d, h, t, Wo, bo, resid, resid_fp32, out, out_fp32, mode, w.P,
                 stream);
}

// ---------------------------------------------------------------- attention backward
struct AttnBwdWs {
  AttnWs fwd;          // q, k, v, o as in the forward
  uint16_t* dO;        // [M, H*d] fp16
  uint16_t* dqkv;      // [M, 3*H*d] bf16, head groups' [dQ | dK | dV] column blocks
  float* lse;          // [B*H][S_pad]
  float* Dv;           // [B*H][S_pad]
};

int64_t attn_s_pad(int64_t S) { return (S + 127) / 128 * 128; }

size_t attn_bwd_ws_bytes(int64_t B, int64_t S, int64_t h, int64_t H, int64_t d) {
  const size_t qkv = align_up(static_cast<size_t>(B) * S * H * d * 2);
  const size_t vec = align_up(static_cast<size_t>(B) * H * attn_s_pad(S) * 4);
  (void)h;
  return 4 * qkv + qkv + 3 * qkv + 2 * vec;
}

AttnBwdWs attn_bwd_ws_layout(void* ws, int64_t B, int64_t S, int64_t H, int64_t d) {
  const size_t qkv = align_up(static_cast<size_t>(B) * S * H * d * 2);
  const size_t vec = align_up(static_cast<size_t>(B) * H * attn_s_pad(S) * 4);
  uint8_t* p = static_cast<uint8_t*>(ws);
  AttnBwdWs w;
  w.fwd = attn_ws_layout(ws, B, S, H, d);
  w.dO = reinterpret_cast<uint16_t*>(p + 4 * qkv);
  w.dqkv = reinterpret_cast<uint16_t*>(p + 5 * qkv);
  w.lse = reinterpret_cast<float*>(p + 8 * qkv);
  w.Dv = reinterpret_cast<float*>(p + 8 * qkv + vec);
  return w;
}

// Gradients of the attention sub-layer by the chain rule, shard (head group) by shard:
// recompute Q, K, V and O (with the softmax rows' log2-sum-exp), then the row-parallel
// projection's gradients (local per group), the attention gradients (per head), the
// column-parallel projection's weight gradients (local) and its input gradient (the sum
// over groups, in one accumulator).
tp_status attn_backward_bf16(const void* X, int B, int S, int h, int H, int d, int t, const tp_shard* Wqkv,
                             const void* const* bqkv, const tp_shard* Wo, const void* dY, const void* dX_add,
                             int causal, void* dX, float* dWqkv, float* dbqkv, float* dWo, float* dbo, void* ws,
                             cudaStream_t stream) {
  const int64_t M = static_cast<int64_t>(B) * S;
  const int Hg = H / t;
  const int64_t n = static_cast<int64_t>(Hg) * d;   // one group's columns of O / dO
  const int64_t ncol = 3 * n;                       // one group's columns of QKV / dQKV
  const int64_t Hd = static_cast<int64_t>(H) * d;
  const int64_t S_pad = attn_s_pad(S);
  AttnBwdWs w = attn_bwd_ws_layout(ws, B, S, H, d);
  uint32_t* status = device_status_ptr();
  const uint64_t lim = wait_limit_ns();
  const float scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(d));
  // 1. recompute Q, K, V (the forward's QKV projection)
  {
    GemmArgs a;
    memset(&a, 0, sizeof(a));
    TP_TRY(make_tmap_2d(&a.tmA, X, 0, h, M, static_cast<uint64_t>(h) * 2, 64, GEMM_BM));
    for (int i = 0; i < t; ++i) TP_TRY(make_tmap_mn(&a.tmB[i], Wqkv[i].ptr, 0, ncol, h, Wqkv[i].ld * 2));
    a.M = static_cast<int>(M); a.N = static_cast<int>(ncol); a.Kg = h; a.G = t;
    a.epi = EPI_QKV; a.act = ACT_NONE;
    for (int i = 0; i < t; ++i) a.bias_g[i] = bqkv ? bqkv[i] : nullptr;
    a.q = w.fwd.q; a.k = w.fwd.k; a.v = w.fwd.v; a.S = S; a.H = H; a.Hg = Hg; a.d = d;
    a.status = status; a.wait_limit_ns = lim;
    TP_TRY(launch_gemm(a, stream, "gemm_qkv"));
  }
  // 2. recompute O (bf16) and each softmax row's log2-sum-exp
  {
    AttnArgs a;
    memset(&a, 0, sizeof(a));
    TP_TRY(make_tmap_attn(&a.tmQ, w.fwd.q, B * H, S, d, 128));
    TP_TRY(make_tmap_attn(&a.tmK, w.fwd.k, B * H, S, d, attention_kv_rows()));
    TP_TRY(make_tmap_attn(&a.tmV, w.fwd.v, B * H, S, d, attention_kv_rows()));
    a.O = w.fwd.o; a.o_f16 = 0;
    a.B = B; a.S = S; a.H = H; a.d = d; a.causal = causal; a.head0 = 0;
    a.scale_log2 = scale_log2;
    a.lse = w.lse; a.lse_ld = static_cast<int>(S_pad);
    a.status = status; a.wait_limit_ns = lim;
    TP_TRY(launch_attention(a, stream));
  }
  // 3. dbo = column sums of dY
  if (dbo) TP_TRY(launch_colsum(dY, M, h, h, dbo, stream));
  // 4. dWo_i = O_i^T dY (rows i*n.. of dWo): the row-parallel projection's weight gradient
  {
    GemmArgs a;
    memset(&a, 0, sizeof(a));
    TP_TRY(make_tmap_mn(&a.tmA, w.fwd.o, 0, Hd, M, Hd * 2));
    for (int i = 0; i < t; ++i) TP_TRY(make_tmap_mn(&a.tmB[i], dY, 0, h, M, h * 2));
    a.M = static_cast<int>(n); a.N = h; a.Kg = static_cast<int>(M); a.G = t;
    a.a_mn = 1; a.a_m_per_group = static_cast<int>(n);
    a.epi = EPI_PARTIAL_F32;
    a.out = dWo; a.ld_out = h; a.out_group_stride = n * h;
    TP_TRY(make_tmap_out_f32_3d(&a.tmOut, dWo, h, n, t, h * 4, n * h * 4));
    a.tma_store = 1;
    a.status = status; a.wait_limit_ns = lim;
    TP_TRY(launch_gemm(a, stream, "gemm_attn_bwd_dwo"));
  }
  // 5. dO_i = dY Wo_i^T (fp16): the row-parallel projection's input gradient, local to group i
  {
    GemmArgs a;
    memset(&a, 0, sizeof(a));
    TP_TRY(make_tmap_2d(&a.tmA, dY, 0, h, M, static_cast<uint64_t>(h) * 2, 64, GEMM_BM));
    for (int i = 0; i < t; ++i) TP_TRY(make_tmap_2d(&a.tmB[i], Wo[i].ptr, 0, h, n, Wo[i].ld * 2, 64, 128));
    TP_TRY(make_tmap_out(&a.tmOut, w.dO, 1, static_cast<uint64_t>(Hd), M, Hd * 2));
    a.M = static_cast<int>(M); a.N = static_cast<int>(n); a.Kg = h; a.G = t;
    a.b_kmajor = 1;
    a.epi = EPI_ACT; a.act = ACT_NONE;
    a.out = w.dO; a.ld_out = Hd; a.out_col_per_group = n; a.out_type = OUT_F16; a.tma_store = 1;
    a.status = status; a.wait_limit_ns = lim;
    TP_TRY(launch_gemm(a, stream, "gemm_attn_bwd_do"));
  }
  // 6. per-head attention gradients into dQKV
  {
    AttnBwdArgs a;
    memset(&a, 0, sizeof(a));
    TP_TRY(make_tmap_attn(&a.tmQ, w.fwd.q, B * H, S, d, 128));
    TP_TRY(make_tmap_attn(&a.tmK, w.fwd.k, B * H, S, d, 128));
    TP_TRY(make_tmap_attn(&a.tmV, w.fwd.v, B * H, S, d, 128));
    TP_TRY(make_tmap_rows_by_head(&a.tmdO, w.dO, B, S, H, d, 128));
    TP_TRY(make_tmap_attn(&a.tmQs, w.fwd.q, B * H, S, d, 64));
    TP_TRY(make_tmap_attn(&a.tmKs, w.fwd.k, B * H, S, d, 64));
    TP_TRY(make_tmap_attn(&a.tmVs, w.fwd.v, B * H, S, d, 64));
    TP_TRY(make_tmap_rows_by_head(&a.tmdOs, w.dO, B, S, H, d, 64));
    TP_TRY(make_tmap_f16_3d(&a.tmOut, w.dqkv, static_cast<uint64_t>(3 * Hd), static_cast<uint64_t>(S),
                            static_cast<uint64_t>(B), static_cast<uint64_t>(3 * Hd) * 2,
                            static_cast<uint64_t>(S) * 3 * Hd * 2, 64, 128));
    a.lse = w.lse; a.Dv = w.Dv; a.dqkv = w.dqkv; a.ld_dqkv = 3 * Hd;
    a.B = B; a.S = S; a.H = H; a.Hg = Hg; a.head0 = 0; a.causal = causal; a.S_pad = static_cast<int>(S_pad);
    a.scale_log2 = scale_log2; a.scale = 1.f / sqrtf(static_cast<float>(d));
    a.status = status; a.wait_limit_ns = lim;
    TP_TRY(launch_attention_backward(a, w.dO, w.fwd.o, 0, stream));
  }
  // 7. dWqkv_i = X^T dQKV_i (columns i*3n.. of dWqkv): the column-parallel weight gradient
  {
    GemmArgs a;
    memset(&a, 0, sizeof(a));
    TP_TRY(make_tmap_mn(&a.tmA, X, 0, h, M, static_cast<uint64_t>(h) * 2));
    for (int i = 0; i < t; ++i) TP_TRY(make_tmap_mn(&a.tmB[i], w.dqkv + i * ncol, 0, ncol, M, 3 * Hd * 2));
    a.M = h; a.N = static_cast<int>(ncol); a.Kg = static_cast<int>(M); a.G = t;
    a.a_mn = 1; a.a_m_per_group = 0;
    a.epi = EPI_PARTIAL_F32;
    a.out = dWqkv; a.ld_out = 3 * Hd; a.out_group_stride = ncol;
    TP_TRY(make_tmap_out_f32_3d(&a.tmOut, dWqkv, ncol, h, t, 3 * Hd * 4, ncol * 4));
    a.tma_store = 1;
    a.status = status; a.wait_limit_ns = lim;
    TP_TRY(launch_gemm(a, stream, "gemm_attn_bwd_dwqkv"));
  }
  // 8. dbqkv = column sums of dQKV
  if (dbqkv) TP_TRY(launch_colsum(w.dqkv, M, 3 * Hd, 3 * Hd, dbqkv, stream));
  // 9. dX = sum_i dQKV_i Wqkv_i^T (+ dX_add): the sum over head groups, in one accumulator
  {
    GemmArgs a;
    memset(&a, 0, sizeof(a));
    TP_TRY(make_tmap_2d(&a.tmA, w.dqkv, 0, 3 * Hd, M, 3 * Hd * 2, 64, GEMM_BM));
    for (int i = 0; i < t; ++i) TP_TRY(make_tmap_2d(&a.tmB[i], Wqkv[i].ptr, 0, ncol, h, Wqkv[i].ld * 2, 64, 128));
    TP_TRY(make_tmap_out(&a.tmOut, dX, 0, static_cast<uint64_t>(h), M, h * 2));
    a.M = static_cast<int>(M); a.N = h; a.Kg = static_cast<int>(ncol); a.G = t;
    a.concat = 1; a.a_k_per_group = static_cast<int>(ncol); a.b_kmajor = 1;
    a.epi = EPI_BIAS_RESID; a.bias = nullptr; a.resid = dX_add; a.ld_resid = h; a.resid_fp32 = 0;
    a.out = dX; a.ld_out = h; a.out_type = OUT_BF16; a.tma_store = 1;
    a.status = status; a.wait_limit_ns = lim;
    TP_TRY(launch_gemm(a, stream, "gemm_attn_bwd_dx"));
  }
  return TP_OK;
}

tp_status validate_attn(const void* X, int B, int S, int h, int H, int d, int t, const tp_shard* Wqkv,
                        const void* const* bqkv, const tp_shard* Wo, const void* bo, const void* residual,
                        void* out, tp_reduce_mode mode, void* ws, size_t ws_bytes) {
  if (mode != TP_REDUCE_FUSED && mode != TP_REDUCE_PARTIALS) return fail(TP_ERR_INVALID_ARG, "unknown mode");
  TP_TRY(validate_attn_dims(B, S, h, H, d, t));
  TP_TRY(check_ptr(X, "X", true));
  TP_TRY(check_ptr(out, "out", true));
  TP_TRY(check_ptr(bo, "bo", false));
  TP_TRY(check_ptr(residual, "residual", false));
  if (out == X || (residual && out == residual)) return fail(TP_ERR_INVALID_ARG, "out aliases an input");
  TP_TRY(check_shards(Wqkv, t, 3LL * (H / t) * d, "Wqkv"));
  TP_TRY(check_shards(Wo, t, h, "Wo"));
  TP_TRY(check_bias_array(bqkv, t, "bqkv"));
  if (is_f16(Wqkv)) return fail(TP_ERR_INVALID_ARG, "Wqkv must have X's dtype (bf16)");
  const size_t need = attn_ws_bytes_i(B, S, h, H, d, t, mode);
  if (!ws || ws_bytes < need) return fail(TP_ERR_WORKSPACE, "workspace of %zu bytes needed", need);
  if (reinterpret_cast<uintptr_t>(ws) % WS_ALIGN) return fail(TP_ERR_INVALID_ARG, "workspace not 256-byte aligned");
  return TP_OK;
}

}  // namespace

// ================================================================ public C ABI
// NVTX range around one public call (pushed on entry, popped on every return).
struct ApiRange {
  explicit ApiRange(const char* name) { nvtxRangePushA(name); }
  ~ApiRange() { nvtxRangePop(); }
  ApiRange(const ApiRange&) = delete;
  ApiRange& operator=(const ApiRange&) = delete;
};

extern "C" {

size_t tp_ffn_workspace_bytes(int64_t M, int64_t h, int64_t f, int t, tp_dtype dtype, tp_reduce_mode mode) {
  if (M <= 0 || h <= 0 || f <= 0 || t < 1) return 0;
  if (dtype == TP_FP32) return align_up(static_cast<size_t>(M) * f * 4) + align_up(static_cast<size_t>(t) * M * h * 4);
  return ffn_bf16_ws(M, h, f, t, mode);
}

tp_status tp_ffn_forward_act(const void* X, int64_t M, int64_t h, int64_t f, int t, const tp_shard* W1,
                             const void* const* b1, const tp_shard* W2, const void* b2, const void* residual,
                             void* out, tp_dtype dtype, tp_reduce_mode mode, tp_activation act, void* ws,
                             size_t ws_bytes, tp_stream_t stream) {
  ApiRange range("tp_ffn_forward_act");
  TP_TRY(validate_ffn(X, M, h, f, t, W1, b1, W2, b2, residual, out, dtype, mode, act, ws, ws_bytes));
  if (M == 0) return TP_OK;
  const int kact = act == TP_ACT_GELU ? ACT_GELU : ACT_RELU;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dtype == TP_FP32) {
    float* Z = static_cast<float*>(ws);
    float* P = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + align_up(static_cast<size_t>(M) * f * 4));
    return launch_ffn_fp32(static_cast<const float*>(X), M, h, f, t, W1, b1, W2, static_cast<const float*>(b2),
                           static_cast<const float*>(residual), static_cast<float*>(out), kact, Z, P, s);
  }
  return ffn_bf16(X, M, h, f, t, W1, b1, W2, b2, residual, 0, out, 0, mode, kact, ws, s);
}

tp_status tp_ffn_forward(const void* X, int64_t M, int64_t h, int64_t f, int t, const tp_shard* W1,
                         const void* const* b1, const tp_shard* W2, const void* b2, const void* residual, void* out,
                         tp_dtype dtype, tp_reduce_mode mode, void* ws, size_t ws_bytes, tp_stream_t stream) {
  return tp_ffn_forward_act(X, M, h, f, t, W1, b1, W2, b2, residual, out, dtype, mode, TP_ACT_GELU, ws, ws_bytes,
                            stream);
}

tp_status tp_column_linear_forward(const void* X, int64_t M, int64_t k, int64_t n, int t, const tp_shard* W,
                                   const void* const* b, int act, void* out, tp_stream_t stream) {
  ApiRange range("tp_column_linear_forward");
  if (M < 0 || k <= 0 || n <= 0) return fail(TP_ERR_INVALID_ARG, "sizes must be positive (M>=0)");
  if (t < 1 || t > TP_MAX_SHARDS) return fail(TP_ERR_INVALID_ARG, "t outside [1, %d]", TP_MAX_SHARDS);
  if (n % t) return fail(TP_ERR_INVALID_ARG, "n is not divisible by t");
  if (k % 64 || (n / t) % 64) return fail(TP_ERR_UNSUPPORTED, "needs k %% 64 == 0 and (n/t) %% 64 == 0");
  if (act != -1 && act != TP_ACT_GELU && act != TP_ACT_RELU) return fail(TP_ERR_INVALID_ARG, "unknown act");
  TP_TRY(check_ptr(X, "X", true));
  TP_TRY(check_ptr(out, "out", true));
  TP_TRY(check_shards(W, t, n / t, "W"));
  TP_TRY(check_bias_array(b, t, "b"));
  if (M == 0) return TP_OK;
  const int kact = act == -1 ? ACT_NONE : (act == TP_ACT_GELU ? ACT_GELU : ACT_RELU);
  return run_column(X, M, k, n / t, t, W, b, kact, out, is_f16(W) ? OUT_F16 : OUT_BF16, n,
                    static_cast<cudaStream_t>(stream));
}

size_t tp_row_linear_workspace_bytes(int64_t M, int64_t n, int t, tp_reduce_mode mode) {
  if (mode != TP_REDUCE_PARTIALS || M <= 0 || n <= 0 || t < 1) return 0;
  return row_partials_ws(M, n, t);
}

tp_status tp_row_linear_forward(const void* A, int64_t M, int64_t k, int64_t n, int t, const tp_shard* W,
                                const void* bias, const void* residual, void* out, tp_reduce_mode mode, void* ws,
                                size_t ws_bytes, tp_stream_t stream) {
  ApiRange range("tp_row_linear_forward");
  if (M < 0 || k <= 0 || n <= 0) return fail(TP_ERR_INVALID_ARG, "sizes must be positive (M>=0)");
  if (t < 1 || t > TP_MAX_SHARDS) return fail(TP_ERR_INVALID_ARG, "t outside [1, %d]", TP_MAX_SHARDS);
  if (k % t) return fail(TP_ERR_INVALID_ARG, "k is not divisible by t");
  if ((k / t) % 64 || n % 64) return fail(TP_ERR_UNSUPPORTED, "needs (k/t) %% 64 == 0 and n %% 64 == 0");
  if (mode != TP_REDUCE_FUSED && mode != TP_REDUCE_PARTIALS) return fail(TP_ERR_INVALID_ARG, "unknown mode");
  TP_TRY(check_ptr(A, "A", true));
  TP_TRY(check_ptr(out, "out", true));
  TP_TRY(check_ptr(bias, "bias", false));
  TP_TRY(check_ptr(residual, "residual", false));
  TP_TRY(check_shards(W, t, n, "W"));
  const size_t need = tp_row_linear_workspace_bytes(M, n, t, mode);
  if (need && (!ws || ws_bytes < need)) return fail(TP_ERR_WORKSPACE, "workspace of %zu bytes needed", need);
  if (M == 0) return TP_OK;
  if (ws && reinterpret_cast<uintptr_t>(ws) % WS_ALIGN)
    return fail(TP_ERR_INVALID_ARG, "workspace is not 256-byte aligned");
  if (mode == TP_REDUCE_PARTIALS)
    TP_TRY(zero_row_counters(static_cast<float*>(ws), M, n, t, static_cast<cudaStream_t>(stream)));
  return run_row(A, M, k / t, n, t, W, bias, residual, 0, out, 0, mode, static_cast<float*>(ws),
                 static_cast<cudaStream_t>(stream));
}

size_t tp_ffn_backward_workspace_bytes(int64_t M, int64_t h, int64_t f, int t) {
  if (M <= 0 || h <= 0 || f <= 0 || t < 1) return 0;
  return ffn_bwd_ws_bytes(M, h, f);
}

tp_status tp_ffn_backward(const void* X, int64_t M, int64_t h, int64_t f, int t, const tp_shard* W1,
                          const void* const* b1, const tp_shard* W2, const void* dY, const void* dX_add, void* dX,
                          float* dW1, float* db1, float* dW2, float* db2, tp_activation act, void* ws,
                          size_t ws_bytes, tp_stream_t stream) {
  ApiRange range("tp_ffn_backward");
  if (act != TP_ACT_GELU && act != TP_ACT_RELU) return fail(TP_ERR_INVALID_ARG, "unknown activation %d", act);
  TP_TRY(validate_ffn_bf16_dims(M, h, f, t));
  // with no rows, X, dY and dX are never touched and may be NULL
  TP_TRY(check_ptr(X, "X", M > 0));
  TP_TRY(check_ptr(dY, "dY", M > 0));
  TP_TRY(check_ptr(dX_add, "dX_add", false));
  TP_TRY(check_ptr(dX, "dX", M > 0));
  TP_TRY(check_ptr(dW1, "dW1", true));
  TP_TRY(check_ptr(dW2, "dW2", true));
  TP_TRY(check_ptr(db1, "db1", false));
  TP_TRY(check_ptr(db2, "db2", false));
  TP_TRY(check_shards(W1, t, f / t, "W1"));
  TP_TRY(check_shards(W2, t, h, "W2"));
  TP_TRY(check_bias_array(b1, t, "b1"));
  if (is_f16(W1) || is_f16(W2)) return fail(TP_ERR_UNSUPPORTED, "the backward pass takes bf16 W1 and W2");
  if (M > 0 && (dX == X || dX == dY || dX == dX_add)) return fail(TP_ERR_INVALID_ARG, "dX aliases an input");
  if (M > 0x7FFFFFFF / 2) return fail(TP_ERR_UNSUPPORTED, "too many rows");
  const size_t need = tp_ffn_backward_workspace_bytes(M, h, f, t);
  if (need && (!ws || ws_bytes < need))
    return fail(TP_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, ws ? ws_bytes : 0);
  if (ws && (reinterpret_cast<uintptr_t>(ws) % WS_ALIGN))
    return fail(TP_ERR_INVALID_ARG, "workspace is not 256-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (M == 0) {
    // no rows: every weight and bias gradient is zero
    if (cudaMemsetAsync(dW1, 0, static_cast<size_t>(h) * f * 4, s) != cudaSuccess ||
        cudaMemsetAsync(dW2, 0, static_cast<size_t>(f) * h * 4, s) != cudaSuccess ||
        (db1 && cudaMemsetAsync(db1, 0, static_cast<size_t>(f) * 4, s) != cudaSuccess) ||
        (db2 && cudaMemsetAsync(db2, 0, static_cast<size_t>(h) * 4, s) != cudaSuccess))
      return fail(TP_ERR_CUDA, "cudaMemsetAsync of the gradients failed");
    return TP_OK;
  }
  return ffn_backward_bf16(X, M, h, f, t, W1, b1, W2, dY, dX_add, dX, dW1, db1, dW2, db2,
                           act == TP_ACT_GELU ? ACT_GELU : ACT_RELU, ws, s);
}

size_t tp_attn_workspace_bytes(int B, int S, int h, int heads, int d, int t, tp_reduce_mode mode) {
  if (B <= 0 || S <= 0 || h <= 0 || heads <= 0 || d <= 0 || t < 1) return 0;
  return attn_ws_bytes_i(B, S, h, heads, d, t, mode);
}

tp_status tp_attn_forward(const void* X, int B, int S, int h, int heads, int d, int t, const tp_shard* Wqkv,
                          const void* const* bqkv, const tp_shard* Wo, const void* bo, const void* residual,
                          int causal, void* out, tp_reduce_mode mode, void* ws, size_t ws_bytes,
                          tp_stream_t stream) {
  ApiRange range("tp_attn_forward");
  if (1LL * B * S == 0) {
    TP_TRY(validate_attn_dims(B > 0 ? B : 1, S > 0 ? S : 1, h, heads, d, t));
    return TP_OK;
  }
  TP_TRY(validate_attn(X, B, S, h, heads, d, t, Wqkv, bqkv, Wo, bo, residual, out, mode, ws, ws_bytes));
  return attn_bf16(X, B, S, h, heads, d, t, Wqkv, bqkv, Wo, bo, residual, 0, causal ? 1 : 0, out, 0, mode, ws,
                   static_cast<cudaStream_t>(stream));
}

size_t tp_attn_backward_workspace_bytes(int B, int S, int h, int heads, int d, int t) {
  if (B <= 0 || S <= 0 || h <= 0 || heads <= 0 || d <= 0 || t < 1) return 0;
  return attn_bwd_ws_bytes(B, S, h, heads, d);
}

tp_status tp_attn_backward(const void* X, int B, int S, int h, int heads, int d, int t, const tp_shard* Wqkv,
                           const void* const* bqkv, const tp_shard* Wo, const void* dY, const void* dX_add,
                           int causal, void* dX, float* dWqkv, float* dbqkv, float* dWo, float* dbo, void* ws,
                           size_t ws_bytes, tp_stream_t stream) {
  ApiRange range("tp_attn_backward");
  TP_TRY(validate_attn_dims(B, S, h, heads, d, t));
  const int64_t M = static_cast<int64_t>(B) * S;
  const int64_t Hd = static_cast<int64_t>(heads) * d;
  // with no tokens, X, dY and dX are never touched and may be NULL
  TP_TRY(check_ptr(X, "X", M > 0));
  TP_TRY(check_ptr(dY, "dY", M > 0));
  TP_TRY(check_ptr(dX_add, "dX_add", false));
  TP_TRY(check_ptr(dX, "dX", M > 0));
  TP_TRY(check_ptr(dWqkv, "dWqkv", true));
  TP_TRY(check_ptr(dWo, "dWo", true));
  TP_TRY(check_ptr(dbqkv, "dbqkv", false));
  TP_TRY(check_ptr(dbo, "dbo", false));
  TP_TRY(check_shards(Wqkv, t, 3LL * (heads / t) * d, "Wqkv"));
  TP_TRY(check_shards(Wo, t, h, "Wo"));
  TP_TRY(check_bias_array(bqkv, t, "bqkv"));
  if (is_f16(Wqkv) || is_f16(Wo)) return fail(TP_ERR_UNSUPPORTED, "the backward pass takes bf16 Wqkv and Wo");
  if (S > 65535 * 128) return fail(TP_ERR_UNSUPPORTED, "S > 65535 * 128 (the gradient kernels' grid)");
  if (M > 0 && (dX == X || dX == dY || dX == dX_add)) return fail(TP_ERR_INVALID_ARG, "dX aliases an input");
  const size_t need = tp_attn_backward_workspace_bytes(B, S, h, heads, d, t);
  if (need && (!ws || ws_bytes < need))
    return fail(TP_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, ws ? ws_bytes : 0);
  if (ws && (reinterpret_cast<uintptr_t>(ws) % WS_ALIGN))
    return fail(TP_ERR_INVALID_ARG, "workspace is not 256-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (M == 0) {
    // no tokens: every weight and bias gradient is zero
    if (cudaMemsetAsync(dWqkv, 0, static_cast<size_t>(h) * 3 * Hd * 4, s) != cudaSuccess ||
        cudaMemsetAsync(dWo, 0, static_cast<size_t>(Hd) * h * 4, s) != cudaSuccess ||
        (dbqkv && cudaMemsetAsync(dbqkv, 0, static_cast<size_t>(3 * Hd) * 4, s) != cudaSuccess) ||
        (dbo && cudaMemsetAsync(dbo, 0, static_cast<size_t>(h) * 4, s) != cudaSuccess))
      return fail(TP_ERR_CUDA, "cudaMemsetAsync of the gradients failed");
    return TP_OK;
  }
  return attn_backward_bf16(X, B, S, h, heads, d, t, Wqkv, bqkv, Wo, dY, dX_add, causal ? 1 : 0, dX, dWqkv, dbqkv,
                            dWo, dbo, ws, s);
}

size_t tp_layer_workspace_bytes(int B, int S, int h, int heads, int d, int64_t f, int t, tp_reduce_mode mode) {
  if (B <= 0 || S <= 0 || h <= 0 || heads <= 0 || d <= 0 || f <= 0 || t < 1) return 0;
  const int64_t M = static_cast<int64_t>(B) * S;
  const size_t a1 = align_up(static_cast<size_t>(M) * h * 2);
  const size_t h1 = align_up(static_cast<size_t>(M) * h * 4);
  const size_t a2 = a1;
  const size_t at = attn_ws_bytes_i(B, S, h, heads, d, t, mode);
  const size_t ff = ffn_bf16_ws(M, h, f, t, mode);
  return a1 + h1 + a2 + (at > ff ? at : ff);
}

tp_status tp_layer_forward(const void* X, int B, int S, int h, int heads, int d, int64_t f, int t, const void* ln1_g,
                           const void* ln1_b, const tp_shard* Wqkv, const void* const* bqkv, const tp_shard* Wo,
                           const void* bo, const void* ln2_g, const void* ln2_b, const tp_shard* W1,
                           const void* const* b1, const tp_shard* W2, const void* b2, float eps, int causal,
                           void* out, tp_reduce_mode mode, void* ws, size_t ws_bytes, tp_stream_t stream) {
  ApiRange range("tp_layer_forward");
  const int64_t M = static_cast<int64_t>(B) * S;
  if (mode != TP_REDUCE_FUSED && mode != TP_REDUCE_PARTIALS) return fail(TP_ERR_INVALID_ARG, "unknown mode");
  TP_TRY(validate_attn_dims(B > 0 ? B : 1, S > 0 ? S : 1, h, heads, d, t));
  TP_TRY(validate_ffn_bf16_dims(M, h, f, t));
  if (!(eps > 0.f)) return fail(TP_ERR_INVALID_ARG, "eps must be positive");
  if (M == 0) return TP_OK;
  TP_TRY(check_ptr(X, "X", true));
  TP_TRY(check_ptr(out, "out", true));
  if (out == X) return fail(TP_ERR_INVALID_ARG, "out aliases X");
  TP_TRY(check_ptr(ln1_g, "ln1_g", false));
  TP_TRY(check_ptr(ln1_b, "ln1_b", false));
  TP_TRY(check_ptr(ln2_g, "ln2_g", false));
  TP_TRY(check_ptr(ln2_b, "ln2_b", false));
  TP_TRY(check_ptr(bo, "bo", false));
  TP_TRY(check_ptr(b2, "b2", false));
  TP_TRY(check_shards(Wqkv, t, 3LL * (heads / t) * d, "Wqkv"));
  TP_TRY(check_shards(Wo, t, h, "Wo"));
  TP_TRY(check_shards(W1, t, f / t, "W1"));
  TP_TRY(check_shards(W2, t, h, "W2"));
  TP_TRY(check_bias_array(bqkv, t, "bqkv"));
  TP_TRY(check_bias_array(b1, t, "b1"));
  const size_t need = tp_layer_workspace_bytes(B, S, h, heads, d, f, t, mode);
  if (!ws || ws_bytes < need) return fail(TP_ERR_WORKSPACE, "workspace of %zu bytes needed", need);
  if (reinterpret_cast<uintptr_t>(ws) % WS_ALIGN) return fail(TP_ERR_INVALID_ARG, "workspace not 256-byte aligned");

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* p = static_cast<uint8_t*>(ws);
  const size_t a1b = align_up(static_cast<size_t>(M) * h * 2);
  const size_t h1b = align_up(static_cast<size_t>(M) * h * 4);
  uint16_t* a1 = reinterpret_cast<uint16_t*>(p);
  float* h1 = reinterpret_cast<float*>(p + a1b);
  uint16_t* a2 = reinterpret_cast<uint16_t*>(p + a1b + h1b);
  void* rest = p + a1b + h1b + a1b;
  // h1 = X + Attn(LN1(X)), kept in fp32; LN1's output takes Wqkv's dtype
  TP_TRY(launch_layernorm(X, 0, ln1_g, ln1_b, M, h, eps, a1, is_f16(Wqkv), s));
  TP_TRY(attn_bf16(a1, B, S, h, heads, d, t, Wqkv, bqkv, Wo, bo, X, 0, causal ? 1 : 0, h1, 1, mode, rest, s));
  // out = h1 + FFN(LN2(h1)); LN2's output takes W1's dtype
  TP_TRY(launch_layernorm(h1, 1, ln2_g, ln2_b, M, h, eps, a2, is_f16(W1), s));
  return ffn_bf16(a2, M, h, f, t, W1, b1, W2, b2, h1, 1, out, 0, mode, ACT_GELU, rest, s);
}

tp_status tp_layernorm_forward(const void* x, tp_dtype in_dtype, const void* gamma, const void* beta, int64_t M,
                               int64_t h, float eps, void* y, tp_dtype out_dtype, tp_stream_t stream) {
  ApiRange range("tp_layernorm_forward");
  if (in_dtype != TP_BF16 && in_dtype != TP_FP32) return fail(TP_ERR_INVALID_ARG, "unknown input dtype");
  if (out_dtype != TP_BF16 && out_dtype != TP_FP16) return fail(TP_ERR_INVALID_ARG, "unknown output dtype");
  if (M < 0 || h <= 0) return fail(TP_ERR_INVALID_ARG, "bad sizes");
  if (h % 8) return fail(TP_ERR_UNSUPPORTED, "h %% 8 != 0");
  if (h > 49152) return fail(TP_ERR_UNSUPPORTED, "h > 49152");
  if (!(eps > 0.f)) return fail(TP_ERR_INVALID_ARG, "eps must be positive");
  TP_TRY(check_ptr(x, "x", true));
  TP_TRY(check_ptr(y, "y", true));
  TP_TRY(check_ptr(gamma, "gamma", false));
  TP_TRY(check_ptr(beta, "beta", false));
  if (M > 0x7FFFFFFF) return fail(TP_ERR_UNSUPPORTED, "too many rows");
  return launch_layernorm(x, in_dtype == TP_FP32, gamma, beta, M, h, eps, y, out_dtype == TP_FP16,
                          static_cast<cudaStream_t>(stream));
}

tp_status tp_reduce_partials(const float* P, int t, int64_t M, int64_t h, const void* bias, const void* residual,
                             tp_dtype dtype, void* out, tp_stream_t stream) {
  ApiRange range("tp_reduce_partials");
  if (dtype != TP_BF16 && dtype != TP_FP32) return fail(TP_ERR_INVALID_ARG, "unknown dtype");
  if (t < 1 || M < 0 || h <= 0) return fail(TP_ERR_INVALID_ARG, "bad sizes");
  if (h % 4) return fail(TP_ERR_UNSUPPORTED, "h %% 4 != 0");
  TP_TRY(check_ptr(P, "P", true));
  TP_TRY(check_ptr(out, "out", true));
  TP_TRY(check_ptr(bias, "bias", false));
  TP_TRY(check_ptr(residual, "residual", false));
  const int f32 = dtype == TP_FP32;
  return launch_reduce_partials(P, t, M, h, bias, f32, residual, f32, out, f32, static_cast<cudaStream_t>(stream));
}

tp_status tp_activation_forward(const float* x, float* y, int64_t n, tp_activation act, tp_stream_t stream) {
  ApiRange range("tp_activation_forward");
  if (n < 0) return fail(TP_ERR_INVALID_ARG, "n must be >= 0");
  if (act != TP_ACT_GELU && act != TP_ACT_RELU) return fail(TP_ERR_INVALID_ARG, "unknown activation %d", act);
  if (n > 0 && (!x || !y)) return fail(TP_ERR_INVALID_ARG, "x or y is NULL");
  return launch_act(x, y, n, act == TP_ACT_GELU ? ACT_GELU : ACT_RELU, static_cast<cudaStream_t>(stream));
}

tp_status tp_get_device_status(tp_stream_t stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return fail(TP_ERR_CUDA, "stream synchronisation failed: %s", cudaGetErrorString(cudaGetLastError()));
  uint32_t v = 0;
  if (cudaMemcpyFromSymbol(&v, g_status_word, sizeof(v)) != cudaSuccess) return fail(TP_ERR_CUDA, "status read");
  const uint32_t zero = 0;
  if (cudaMemcpyToSymbol(g_status_word, &zero, sizeof(zero)) != cudaSuccess) return fail(TP_ERR_CUDA, "status clear");
  if (v == 0) return TP_OK;
  if ((v & 0xFF) == DEV_TIMEOUT) return fail(TP_ERR_TIMEOUT, "device wait ran out (site %u)", (v >> 8) & 0xFF);
  if (v & DEV_RANGE_MASK) {
    std::string where;
    if (v & DEV_RANGE_COLUMN) where += " column-layer output (act(Z));";
    if (v & DEV_RANGE_QKV) where += " Q/K/V;";
    if (v & DEV_RANGE_ATTN_O) where += " attention output O;";
    if (v & DEV_RANGE_LAYERNORM) where += " LayerNorm output;";
    if (v & DEV_RANGE_ATTN_GRAD) where += " attention backward P or dS;";
    return fail(TP_ERR_RANGE, "an fp16 intermediate exceeded 65504 in:%s", where.c_str());
  }
  return fail(TP_ERR_CUDA, "device status 0x%x", v);
}

void tp_set_wait_limit_ns(uint64_t ns) { g_wait_limit_ns.store(ns ? ns : 1); }

tp_status tp_selftest_bounded_wait(uint64_t limit_ns, tp_stream_t stream) {
  if (limit_ns == 0 || limit_ns > 10000000000ull) return fail(TP_ERR_INVALID_ARG, "limit must be in (0, 10 s]");
  return launch_selftest_wait(limit_ns, static_cast<cudaStream_t>(stream));
}

tp_status tp_trace_enable(int capacity) {
  if (capacity <= 0 || capacity > (1 << 20)) return fail(TP_ERR_INVALID_ARG, "bad trace capacity");
  t_trace.clear();
  t_trace.reserve(capacity);
  t_trace_cap = capacity;
  t_trace_on = true;
  return TP_OK;
}

void tp_trace_disable(void) { t_trace_on = false; }

int tp_trace_count(void) { return static_cast<int>(t_trace.size()); }

tp_status tp_trace_get(int i, const char** name, float* ms) {
  if (i < 0 || i >= static_cast<int>(t_trace.size())) return fail(TP_ERR_INVALID_ARG, "trace index out of range");
  if (name) *name = t_trace[i].name;
  if (ms) {
    if (cudaEventElapsedTime(ms, t_trace[i].start, t_trace[i].stop) != cudaSuccess)
      return fail(TP_ERR_CUDA, "event timing failed");
  }
  return TP_OK;
}

const char* tp_status_string(tp_status s) {
  switch (s) {
    case TP_OK: return "TP_OK";
    case TP_ERR_INVALID_ARG: return "TP_ERR_INVALID_ARG";
    case TP_ERR_UNSUPPORTED: return "TP_ERR_UNSUPPORTED";
    case TP_ERR_WORKSPACE: return "TP_ERR_WORKSPACE";
    case TP_ERR_CUDA: return "TP_ERR_CUDA";
    case TP_ERR_TIMEOUT: return "TP_ERR_TIMEOUT";
    case TP_ERR_RANGE: return "TP_ERR_RANGE";
  }
  return "TP_ERR_UNKNOWN";
}

const char* tp_last_error(void) { return t_last_error.c_str(); }

int tp_version(void) { return 1; }

}  // extern "C"
