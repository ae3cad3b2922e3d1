// moe_route_noalloc: moe_route for callers that cannot allocate device memory.
//
// moe_route needs a caller-allocated workspace for its internal per-block
// statistics (counts, ranks, probability partials, the dispatch scan). Some
// callers have no way to provide one: plugin-style interfaces of inference
// runtimes hand a kernel its input and output buffers but no allocator, and
// latency-critical callers must not call cudaMalloc on their hot path because
// it can synchronise the device and its cost is unbounded. This entry point
// keeps that scratch in a fixed-size array in this library's own device
// memory instead, so the caller passes only inputs and outputs.
//
// The array below is a device symbol: every GPU that loads this library holds
// kNoAllocScratchBytes of it until the process exits. In host code its name is
// only a host-side placeholder, never a device address, so the device address
// is looked up once per device with cudaGetSymbolAddress (with that device
// current) and cached; the first call on each device does this lookup.
//
// All calls on a device share the one array and it keeps whatever the last
// call left there. The route launch clears the parts that must start at zero
// (the status word and the per-expert row totals) at the start of every call;
// everything else is fully written before it is read. Two calls whose GPU work
// overlaps (for example on two streams without ordering between them) race on
// the array and give wrong results: order them on one stream.
#include "moe_internal.cuh"

#include <mutex>

namespace moe {

// 8 MiB (MOE_ROUTE_NOALLOC_MAX_SCRATCH_BYTES in the header). A shape needs
// moe_workspace_bytes(dims) of it: about 0.9 MB for T = 16384, d = 1024, K = 4,
// N = 64, about 6.1 MB for T = 131072, d = 2048, K = 8, N = 64.
constexpr size_t kNoAllocScratchBytes = MOE_ROUTE_NOALLOC_MAX_SCRATCH_BYTES;

static __device__ __align__(256) unsigned char g_route_scratch[kNoAllocScratchBytes];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {nullptr};

// Device address of g_route_scratch on the current device (looked up once).
int scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_route_scratch);
    if (e != cudaSuccess || p == nullptr) return MOE_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return MOE_OK;
}
}  // namespace

}  // namespace moe

extern "C" MOE_API int moe_route_noalloc(const moe_dims_t* dims, const uint16_t* x, const float* w_router,
                                         const float* router_bias, const float* tok_null_bias,
                                         float* logits_out, int32_t* topk_idx, float* topk_gate,
                                         int32_t* n_real, moe_stream_t stream) {
  using namespace moe;
  const int rc = check_dims(dims);
  if (rc != MOE_OK) return rc;
  if (dims->T == 0) return MOE_OK;
  if (!x || !w_router || !topk_idx || !topk_gate || !n_real) return MOE_ERR_INVALID_ARG;
  // The internal scratch of this shape must fit in the fixed array.
  if (ws_layout(*dims).total > kNoAllocScratchBytes) return MOE_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  const int sr = scratch_address(&scratch);
  if (sr != MOE_OK) return sr;
  return launch_route(*dims, x, w_router, router_bias, tok_null_bias, logits_out, topk_idx, topk_gate, n_real,
                      scratch, reinterpret_cast<cudaStream_t>(stream));
}
