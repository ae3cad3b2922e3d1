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
// The array below is a device symbol: every GPU that uses this entry point holds
// kNoAllocScratchBytes of it from the first call on that device until the process
// exits (with CUDA's lazy module loading the array is allocated when the module is
// first used on a device, not when the library is loaded). In host code its name is
// only a host-side placeholder, never a device address, so the device address is
// looked up with cudaGetSymbolAddress (with the device current) and cached per
// device and CUDA context; the first call on a device, and the first call after its
// context was replaced (cudaDeviceReset), does this lookup.
//
// All calls on a device share the one array and it keeps whatever the last
// call left there. The route launch clears the parts that must start at zero
// (the status word and the per-expert row totals) at the start of every call;
// everything else is fully written before it is read. Two calls whose GPU work
// overlaps (for example on two streams without ordering between them) race on
// the array and give wrong results: order them on one stream.
//
// Device-side failures (a bounded wait that ran out, an index guard) are recorded
// in the array's first word, as in a caller's workspace; moe_route_noalloc_device_status
// reads it.
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
CUcontext g_scratch_ctx[kMaxDevices] = {nullptr};

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

// cuCtxGetCurrent from the driver, through the runtime's entry-point query (the library
// links only the static runtime).
CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

// Device address of g_route_scratch on the current device, looked up again whenever the
// device's current context differs from the one the cached address belongs to. Before
// the runtime's first use on this thread no context is current yet; the lookup itself
// then binds the device's primary context, and it is read again afterwards.
int scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
  const CtxGetCurrentFn get = ctx_get_current();
  CUcontext ctx = nullptr;
  if (get == nullptr || get(&ctx) != CUDA_SUCCESS) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (ctx != nullptr && g_scratch_addr[dev] != nullptr && g_scratch_ctx[dev] == ctx) {
    *out = g_scratch_addr[dev];
    return MOE_OK;
  }
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_route_scratch);
  if (e != cudaSuccess || p == nullptr) return MOE_ERR_CUDA;
  if (ctx == nullptr && (get(&ctx) != CUDA_SUCCESS || ctx == nullptr)) return MOE_ERR_CUDA;
  g_scratch_addr[dev] = p;
  g_scratch_ctx[dev] = ctx;
  *out = p;
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

extern "C" MOE_API int moe_route_noalloc_device_status(moe_stream_t stream) {
  using namespace moe;
  void* scratch = nullptr;
  const int sr = scratch_address(&scratch);
  if (sr != MOE_OK) return sr;
  return moe_get_device_status(scratch, stream);
}

extern "C" MOE_API int moe_route_noalloc_selftest_bounded_wait(uint64_t limit_ns, moe_stream_t stream) {
  using namespace moe;
  void* scratch = nullptr;
  const int sr = scratch_address(&scratch);
  if (sr != MOE_OK) return sr;
  return moe_selftest_bounded_wait(scratch, limit_ns, stream);
}
