// FFN block entry point that allocates nothing: its act(Z) scratch lives in a
// fixed-size static device array instead of a caller-provided workspace.
//
// Some callers cannot hand the library a workspace: code that runs inside a
// host framework which owns the whole device memory pool and forbids
// allocations it did not make, or latency-critical loops where a cudaMalloc
// (which may synchronise the device) is not allowed.  They still pass inputs
// and outputs; the intermediate act(Z) goes to `g_ffn_scratch` below.
//
// Limits and sharing:
//  * The scratch holds kScratchBytes = 16 MiB, i.e. M * f <= 8,388,608
//    bf16 elements; larger calls are rejected with TP_ERR_UNSUPPORTED.
//  * Every GPU that loads the library holds the array until the process exits.
//  * Every call on a device shares the one array, which keeps the last call's
//    contents.  Nothing in it has to start at zero: the column GEMM writes every
//    element of act(Z) before the row GEMM reads it.  Calls that overlap on the
//    GPU (for example on two streams) race on the array and give wrong results.
//  * The first call on each device looks up the array's device address
//    (cudaGetSymbolAddress, with that device current); make that first call
//    before any stream capture.  Later calls look it up again unless their
//    stream is capturing, so a device reset (which reloads the module and may
//    move the array) does not leave a stale address behind.
#include <atomic>
#include <cstdio>

#include <nvtx3/nvToolsExt.h>

#include "tp_internal.h"

namespace {

constexpr size_t kScratchBytes = 16u << 20;

// In host code this name is only a stand-in for the symbol: its device address
// comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_ffn_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::atomic<void*> g_scratch_addr[kMaxDevices];

// Device address of g_ffn_scratch on the current device: looked up on every call whose
// stream is not being captured, reused from the last lookup while it is.
tp_status scratch_address(cudaStream_t stream, void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return tpb::set_error(TP_ERR_CUDA, "cudaGetDevice failed");
  if (dev < 0 || dev >= kMaxDevices) return tpb::set_error(TP_ERR_UNSUPPORTED, "device index above 63");
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess)
    return tpb::set_error(TP_ERR_CUDA, "cudaStreamIsCapturing failed");
  void* p = cap == cudaStreamCaptureStatusNone ? nullptr : g_scratch_addr[dev].load();
  if (!p) {
    if (cap != cudaStreamCaptureStatusNone)
      return tpb::set_error(TP_ERR_INVALID_ARG, "first no-allocation call on this device is being captured");
    const cudaError_t e = cudaGetSymbolAddress(&p, g_ffn_scratch);
    if (e != cudaSuccess || !p) {
      char msg[160];
      snprintf(msg, sizeof(msg), "cudaGetSymbolAddress of the static scratch failed: %s", cudaGetErrorString(e));
      return tpb::set_error(TP_ERR_CUDA, msg);
    }
    g_scratch_addr[dev].store(p);
  }
  *out = p;
  return TP_OK;
}

tp_status ffn_noalloc(const void* X, int64_t M, int64_t h, int64_t f, int t, const tp_shard* W1,
                      const void* const* b1, const tp_shard* W2, const void* b2, const void* residual, void* out,
                      tp_stream_t stream) {
  if (M < 0 || h <= 0 || f <= 0) return tpb::set_error(TP_ERR_INVALID_ARG, "sizes must be positive (M>=0)");
  if (t < 1 || t > TP_MAX_SHARDS) return tpb::set_error(TP_ERR_INVALID_ARG, "t outside [1, 16]");
  if (!W1 || !W2) return tpb::set_error(TP_ERR_INVALID_ARG, "shard array is NULL");
  for (int i = 0; i < t; ++i)
    if (W1[i].dtype != TP_BF16 || W2[i].dtype != TP_BF16)
      return tpb::set_error(TP_ERR_UNSUPPORTED, "the no-allocation FFN takes bf16 W1 and W2 only");
  if (M * f > static_cast<int64_t>(kScratchBytes / 2)) {
    char msg[200];
    snprintf(msg, sizeof(msg),
             "act(Z) needs %lld bytes but the static scratch holds %zu (M * f must be <= %zu)",
             static_cast<long long>(M * f * 2), kScratchBytes, kScratchBytes / 2);
    return tpb::set_error(TP_ERR_UNSUPPORTED, msg);
  }
  if (out && (out == X || out == residual)) return tpb::set_error(TP_ERR_INVALID_ARG, "out aliases an input");
  if (M == 0) return TP_OK;
  void* scratch = nullptr;
  const tp_status s = scratch_address(static_cast<cudaStream_t>(stream), &scratch);
  if (s != TP_OK) return s;
  // step 1: act(Z) = GeLU(X W1_i + b1_i) for every shard, into the static scratch [M, f]
  const tp_status c = tp_column_linear_forward(X, M, h, f, t, W1, b1, TP_ACT_GELU, scratch, stream);
  if (c != TP_OK) return c;
  // steps 2-3: out = sum_i act(Z)_i W2_i + b2 + residual, shards summed in one accumulator
  return tp_row_linear_forward(scratch, M, f, h, t, W2, b2, residual, out, TP_REDUCE_FUSED, nullptr, 0, stream);
}

}  // namespace

extern "C" tp_status tp_ffn_forward_noalloc(const void* X, int64_t M, int64_t h, int64_t f, int t,
                                            const tp_shard* W1, const void* const* b1, const tp_shard* W2,
                                            const void* b2, const void* residual, void* out, tp_stream_t stream) {
  nvtxRangePushA("tp_ffn_forward_noalloc");
  const tp_status s = ffn_noalloc(X, M, h, f, t, W1, b1, W2, b2, residual, out, stream);
  nvtxRangePop();
  return s;
}
