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

#include "rfq.h"

namespace {

static __device__ __align__(256) uint8_t g_static_workspace[RFQ_STATIC_WORKSPACE_BYTES];

// Device address of the scratch array on the current device.  Host code cannot
// use the symbol itself (on the host it names a stand-in, not device memory), so
// the address is looked up on every call, with the caller's device current.  The
// lookup is a table read in the runtime; nothing is cached, so an address never
// outlives the context it belongs to (after cudaDeviceReset the library's device
// code is loaded again, possibly at another address).
rfq_status_t static_workspace_address(void** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_static_workspace) != cudaSuccess || p == nullptr) return RFQ_ERR_CUDA;
  *out = p;
  return RFQ_OK;
}

}  // namespace

extern "C" rfq_status_t rfq_linear_static_workspace(const void* x_bf16, int64_t M, int64_t K,
                                                    const void* qw_codes, const void* qw_scales, int64_t N,
                                                    void* y, rfq_out_t y_type, int use_residual,
                                                    cudaStream_t stream) {
  // The argument checks come in rfq_linear's order, so both entry points return the
  // same status for the same bad arguments; the size limit is checked last.
  if (M < 0 || N < 0 || K < 0) return RFQ_ERR_INVALID_ARG;
  if (y_type != RFQ_OUT_F32 && y_type != RFQ_OUT_BF16) return RFQ_ERR_INVALID_ARG;
  const size_t need = rfq_linear_workspace_bytes(M, K, use_residual);
  // Empty problems need no scratch, and shapes rfq_linear rejects (need == 0 for a
  // bad M x K, or N not a multiple of 8) go to it unchanged for its own status.
  if (M == 0 || N == 0 || K == 0 || need == 0 || (N % 8) != 0)
    return rfq_linear(x_bf16, M, K, qw_codes, qw_scales, N, y, y_type, use_residual, nullptr, 0, stream);
  if (need > static_cast<size_t>(RFQ_STATIC_WORKSPACE_BYTES))
    return RFQ_ERR_UNSUPPORTED_SHAPE;   // the quantized activation does not fit the fixed scratch array
  void* ws = nullptr;
  rfq_status_t st = static_workspace_address(&ws);
  if (st != RFQ_OK) return st;
  // Nothing in the array has to start at zero: the quantizer writes every code
  // and every scale byte (padding included) that the GEMM then reads.
  return rfq_linear(x_bf16, M, K, qw_codes, qw_scales, N, y, y_type, use_residual, ws,
                    static_cast<size_t>(RFQ_STATIC_WORKSPACE_BYTES), stream);
}
