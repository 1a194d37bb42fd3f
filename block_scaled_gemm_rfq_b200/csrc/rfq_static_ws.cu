// rfq_static_ws.cu -- rfq_linear for callers that cannot allocate device memory.
//
// rfq_linear needs a scratch buffer for the quantized activation (the codes and
// scales of Q(X) and Q(R) that the quantizer writes and the GEMM reads).  Some
// callers cannot provide one: a plug-in running inside a host application that
// owns the whole device memory pool and forbids raw cudaMalloc, or a
// latency-critical loop where an allocation (which can synchronize the device)
// is not allowed after start-up.  For them, rfq_linear_static_workspace uses a
// fixed scratch array that lives in this library's own device memory: a
// file-scope __device__ array of RFQ_STATIC_WORKSPACE_BYTES, reserved on every
// GPU that loads the library and held until the process exits.  The entry point
// itself allocates nothing.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "rfq.h"

namespace {

static __device__ __align__(256) uint8_t g_static_workspace[RFQ_STATIC_WORKSPACE_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_ws_mutex;
void* g_ws_address[kMaxDevices] = {};   // device address of g_static_workspace, per device

// Device address of the scratch array on the current device.  Host code cannot
// use the symbol itself (on the host it names a stand-in, not device memory), so
// the address is queried once per device, with that device current, and cached.
rfq_status_t static_workspace_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return RFQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return RFQ_ERR_UNSUPPORTED_DEVICE;
  std::lock_guard<std::mutex> lock(g_ws_mutex);
  if (g_ws_address[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_workspace) != cudaSuccess || p == nullptr) return RFQ_ERR_CUDA;
    g_ws_address[dev] = p;
  }
  *out = g_ws_address[dev];
  return RFQ_OK;
}

}  // namespace

extern "C" rfq_status_t rfq_linear_static_workspace(const void* x_bf16, int64_t M, int64_t K,
                                                    const void* qw_codes, const void* qw_scales, int64_t N,
                                                    void* y, rfq_out_t y_type, int use_residual,
                                                    cudaStream_t stream) {
  if (M < 0 || N < 0 || K < 0) return RFQ_ERR_INVALID_ARG;
  const size_t need = rfq_linear_workspace_bytes(M, K, use_residual);
  if (M > 0 && K > 0 && (need == 0 || need > static_cast<size_t>(RFQ_STATIC_WORKSPACE_BYTES)))
    return RFQ_ERR_UNSUPPORTED_SHAPE;   // the quantized activation does not fit the fixed scratch array
  if (M == 0 || N == 0) return rfq_linear(x_bf16, M, K, qw_codes, qw_scales, N, y, y_type, use_residual, nullptr, 0,
                                          stream);
  void* ws = nullptr;
  rfq_status_t st = static_workspace_address(&ws);
  if (st != RFQ_OK) return st;
  // Nothing in the array has to start at zero: the quantizer writes every code
  // and every scale byte (padding included) that the GEMM then reads.
  return rfq_linear(x_bf16, M, K, qw_codes, qw_scales, N, y, y_type, use_residual, ws,
                    static_cast<size_t>(RFQ_STATIC_WORKSPACE_BYTES), stream);
}
