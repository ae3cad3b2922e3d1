// C ABI entry points of libmoe_null (declared in include/moe_null.h): argument
// checks on the host, then stream-ordered launches. No entry point allocates
// device memory or synchronises the host (except moe_get_device_status).
#include "moe_internal.cuh"

#include <climits>

namespace moe {

int cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev < 0 || dev >= 64) return 148;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

int check_dims(const moe_dims_t* d) {
  if (d == nullptr) return MOE_ERR_INVALID_ARG;
  if ((d->flags & ~(MOE_FLAG_ROUTER_FP32_CORES | MOE_FLAG_FFN_CTA_PAIR | MOE_FLAG_WGRAD_CTA_PAIR)) != 0u)
    return MOE_ERR_INVALID_ARG;
  if (d->T < 0 || d->d <= 0 || d->N < 1 || d->M < 0 || d->K < 1 || d->F <= 0 || d->F_shared <= 0)
    return MOE_ERR_INVALID_ARG;
  if (d->C < 0 || d->V < 0) return MOE_ERR_INVALID_ARG;
  if ((long long)d->K > (long long)d->N + d->M + d->C + d->V) return MOE_ERR_INVALID_ARG;
  if (d->C + d->V > 0) {  // MoE++ copy/constant experts: tensor-core router, one 80-row router tile
    if (d->C + d->V > kMaxPP || router_rows(*d) > kMaxRows) return MOE_ERR_UNSUPPORTED;
    if (route_fp32_cores(*d)) return MOE_ERR_UNSUPPORTED;
  }
  if (d->N > kMaxN || d->K > kMaxK) return MOE_ERR_UNSUPPORTED;
  if (d->d % 128 != 0 || d->d > 8192) return MOE_ERR_UNSUPPORTED;
  if (d->F % 64 != 0 || d->F > 16384 || d->F_shared % 64 != 0 || d->F_shared > 16384)
    return MOE_ERR_UNSUPPORTED;
  if ((long long)d->T * d->K >= (long long)INT_MAX) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

}  // namespace moe

using namespace moe;

#define MOE_CHECK(expr)              \
  do {                               \
    const int _r = (expr);           \
    if (_r != MOE_OK) return _r;     \
  } while (0)

static inline cudaStream_t S(moe_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

extern "C" {

int moe_abi_version(void) { return MOE_NULL_ABI_VERSION; }

const char* moe_status_string(int status) {
  switch (status) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported size or limit";
    case MOE_ERR_CUDA: return "CUDA call failed";
    case MOE_ERR_TIMEOUT: return "device-side wait timed out";
    case MOE_ERR_DEVICE_BOUNDS: return "device-side index out of range";
    default: return "unknown status";
  }
}

int moe_check_dims(const moe_dims_t* dims) { return check_dims(dims); }

size_t moe_workspace_bytes(const moe_dims_t* dims) {
  if (check_dims(dims) != MOE_OK) return 0;
  return ws_layout(*dims).total;
}

size_t moe_packed_gate_up_elems(const moe_dims_t* dims, int shared) {
  if (check_dims(dims) != MOE_OK) return 0;
  if (shared) return (size_t)2 * dims->F_shared * dims->d;
  return (size_t)dims->N * 2 * dims->F * dims->d;
}

size_t moe_aux_sums_count(const moe_dims_t* dims) {
  if (check_dims(dims) != MOE_OK) return 0;
  return aux_sums_count(*dims);
}

int moe_pack_gate_up(const moe_dims_t* dims, const uint16_t* w_gate, const uint16_t* w_up,
                     const uint16_t* ws_gate, const uint16_t* ws_up, uint16_t* gate_up,
                     uint16_t* shared_gate_up, moe_stream_t stream) {
  MOE_CHECK(check_dims(dims));
  if (gate_up && (!w_gate || !w_up)) return MOE_ERR_INVALID_ARG;
  if (shared_gate_up && (!ws_gate || !ws_up)) return MOE_ERR_INVALID_ARG;
  return launch_pack_gate_up(*dims, w_gate, w_up, ws_gate, ws_up, gate_up, shared_gate_up, S(stream));
}

size_t moe_router_split_elems(const moe_dims_t* dims) {
  if (check_dims(dims) != MOE_OK) return 0;
  return (size_t)3 * route_npw(*dims) * dims->d;
}

int moe_prepare_router(const moe_dims_t* dims, const float* w_router, uint16_t* router_split,
                       moe_stream_t stream) {
  MOE_CHECK(check_dims(dims));
  if (!w_router || !router_split) return MOE_ERR_INVALID_ARG;
  return launch_router_split(*dims, w_router, router_split, S(stream), nullptr);
}

int moe_route(const moe_dims_t* dims, const uint16_t* x, const float* w_router, const float* router_bias,
              const float* tok_null_bias, float* logits_out, int32_t* topk_idx, float* topk_gate,
              int32_t* n_real, void* workspace, moe_stream_t stream) {
  MOE_CHECK(check_dims(dims));
  if (dims->T == 0) return MOE_OK;
  if (!x || !w_router || !topk_idx || !topk_gate || !n_real || !workspace) return MOE_ERR_INVALID_ARG;
  return launch_route(*dims, x, w_router, router_bias, tok_null_bias, logits_out, topk_idx, topk_gate,
                      n_real, workspace, S(stream));
}

int moe_route_prepared(const moe_dims_t* dims, const uint16_t* x, const uint16_t* router_split,
                       const float* router_bias, const float* tok_null_bias, float* logits_out, int32_t* topk_idx,
                       float* topk_gate, int32_t* n_real, void* workspace, moe_stream_t stream) {
  MOE_CHECK(check_dims(dims));
  if (route_fp32_cores(*dims)) return MOE_ERR_INVALID_ARG;
  if (dims->T == 0) return MOE_OK;
  if (!x || !router_split || !topk_idx || !topk_gate || !n_real || !workspace) return MOE_ERR_INVALID_ARG;
  return launch_route(*dims, x, nullptr, router_bias, tok_null_bias, logits_out, topk_idx, topk_gate, n_real,
                      workspace, S(stream), router_split);
}

int moe_dispatch(const moe_dims_t* dims, const uint16_t* x, const int32_t* topk_idx, void* workspace,
                 int32_t* counts, int32_t* offsets, int32_t* perm_tok, int32_t* slot_row, uint16_t* xs,
                 moe_stream_t stream) {
  MOE_CHECK(check_dims(dims));
  if (dims->T == 0) return MOE_OK;
  if (!x || !topk_idx || !workspace || !counts || !offsets || !perm_tok || !slot_row) return MOE_ERR_INVALID_ARG;
  return launch_dispatch(*dims, x, topk_idx, workspace, counts, offsets, perm_tok, slot_row, xs, nullptr,
                         nullptr, nullptr, S(stream));
}

int moe_expert_ffn(const moe_dims_t* dims, const uint16_t* xs, const uint16_t* x, const int32_t* offsets,
                   const uint16_t* gate_up, const uint16_t* w_down, const uint16_t* shared_gate_up,
                   const uint16_t* shared_down, uint16_t* h, uint16_t* h_shared, uint16_t* ys,
                   uint16_t* shared_out, void* workspace, moe_stream_t stream) {
  MOE_CHECK(check_dims(dims));
  if (dims->T == 0) return MOE_OK;
  if (!xs || !x || !offsets || !gate_up || !w_down || !shared_gate_up || !shared_down || !h || !h_shared ||
      !ys || !shared_out || !workspace)
    return MOE_ERR_INVALID_ARG;
  return launch_expert_ffn(*dims, xs, x, offsets, gate_up, w_down, shared_gate_up, shared_down, h, h_shared,
                           ys, shared_out, workspace, S(stream));
}

int moe_expert_gate_up(const moe_dims_t* dims, const uint16_t* xs, const uint16_t* x, const int32_t* offsets,
                       const uint16_t* gate_up, const uint16_t* shared_gate_up, uint16_t* h, uint16_t* h_shared,
                       void* workspace, moe_stream_t stream) {
  MOE_CHECK(check_dims(dims));
  if (dims->T == 0) return MOE_OK;
  if (!xs || !x || !offsets || !gate_up || !shared_gate_up || !h || !h_shared || !workspace)
    return MOE_ERR_INVALID_ARG;
  return launch_gate_up(*dims, xs, x, offsets, gate_up, shared_gate_up, h, h_shared, workspace, S(stream));
}

int moe_expert_gate_up_gather(const moe_dims_t* dims, const uint16_t* x, const int32_t* perm_tok,
                              const int32_t* offsets, const uint16_t* gate_up, const uint16_t* shared_gate_up,
                              uint16_t* h, uint16_t* h_shared, void* workspace, moe_stream_t stream) {
  MOE_CHECK(check_dims(dims));
  if (dims->T == 0) return MOE_OK;
  if (!x || !perm_tok || !offsets || !gate_up || !shared_gate_up || !h || !h_shared || !workspace)
    return MOE_ERR_INVALID_ARG;
  return launch_gate_up_perm(*dims, nullptr, x, offsets, perm_tok, gate_up, shared_gate_up, h, h_shared, workspace,
                             S(stream));
}

int moe_expert_down(const moe_dims_t* dims, const int32_t* offsets, const uint16_t* h, const uint16_t* h_shared,
                    const uint16_t* w_down, const uint16_t* shared_down, uint16_t* ys, uint16_t* shared_out,
                    void* workspace, moe_stream_t stream) {
  MOE_CHECK(check_dims(dims));
  if (dims->T == 0) return MOE_OK;
  if (!offsets || !h || !h_shared || !w_down || !shared_down || !ys || !shared_out || !workspace)
    return MOE_ERR_INVALID_ARG;
  return launch_down(*dims, offsets, h, h_shared, w_down, shared_down, ys, shared_out, workspace, S(stream));
}

int moe_expert_gate_up_rows(const moe_dims_t* dims, int64_t rows_cap, const uint16_t* xs, const uint16_t* x,
                            const int32_t* offsets, const uint16_t* gate_up, const uint16_t* shared_gate_up,
                            uint16_t* h, uint16_t* h_shared, void* workspace, moe_stream_t stream) {
  MOE_CHECK(check_dims(dims));
  if (rows_cap < 1 || rows_cap >= (int64_t)INT_MAX) return rows_cap < 1 ? MOE_ERR_INVALID_ARG : MOE_ERR_UNSUPPORTED;
  if (!xs || !offsets || !gate_up || !h || !workspace) return MOE_ERR_INVALID_ARG;
  if (dims->T > 0 && (!x || !shared_gate_up || !h_shared)) return MOE_ERR_INVALID_ARG;
  return launch_gate_up_rows(*dims, (long long)rows_cap, xs, x, offsets, gate_up, shared_gate_up, h, h_shared,
                             workspace, S(stream));
}

int moe_expert_down_rows(const moe_dims_t* dims, int64_t rows_cap, const int32_t* offsets, const uint16_t* h,
                         const uint16_t* h_shared, const uint16_t* w_down, const uint16_t* shared_down, uint16_t* ys,
                         uint16_t* shared_out, void* workspace, moe_stream_t stream) {
  MOE_CHECK(check_dims(dims));
  if (rows_cap < 1 || rows_cap >= (int64_t)INT_MAX) return rows_cap < 1 ? MOE_ERR_INVALID_ARG : MOE_ERR_UNSUPPORTED;
  if (!offsets || !h || !w_down || !ys || !workspace) return MOE_ERR_INVALID_ARG;
  if (dims->T > 0 && (!h_shared || !shared_down || !shared_out)) return MOE_ERR_INVALID_ARG;
  return launch_down_rows(*dims, (long long)rows_cap, offsets, h, h_shared, w_down, shared_down, ys, shared_out,
                          workspace, S(stream));
}

int moe_expert_down_combine(const moe_dims_t* dims, const int32_t* offsets, const uint16_t* h,
                            const uint16_t* h_shared, const uint16_t* w_down, const uint16_t* shared_down,
                            uint16_t* ys, const float* topk_gate, const int32_t* slot_row, const int32_t* topk_idx,
                            const uint16_t* x, const uint16_t* const_vectors, uint16_t* y, void* workspace,
                            moe_stream_t stream) {
  MOE_CHECK(check_dims(dims));
  if (dims->T == 0) return MOE_OK;
  if (!offsets || !h || !h_shared || !w_down || !shared_down || !ys || !topk_gate || !slot_row || !y || !workspace)
    return MOE_ERR_INVALID_ARG;
  if (dims->C + dims->V > 0 && (!topk_idx || (dims->C > 0 && !x) || (dims->V > 0 && !const_vectors)))
    return MOE_ERR_INVALID_ARG;
  return launch_down_combine(*dims, offsets, h, h_shared, w_down, shared_down, ys, topk_gate, slot_row, topk_idx, x,
                             const_vectors, y, workspace, S(stream));
}

int moe_combine(const moe_dims_t* dims, const uint16_t* ys, const uint16_t* shared_out, const float* topk_gate,
                const int32_t* slot_row, const int32_t* topk_idx, const uint16_t* x, const uint16_t* const_vectors,
                uint16_t* y, moe_stream_t stream) {
  MOE_CHECK(check_dims(dims));
  if (dims->T == 0) return MOE_OK;
  if (!ys || !shared_out || !topk_gate || !slot_row || !y) return MOE_ERR_INVALID_ARG;
  if (dims->C + dims->V > 0 && (!topk_idx || (dims->C > 0 && !x) || (dims->V > 0 && !const_vectors)))
    return MOE_ERR_INVALID_ARG;
  return launch_combine(*dims, ys, shared_out, topk_gate, slot_row, topk_idx, x, const_vectors, y, S(stream));
}

int moe_combine_inplace(const moe_dims_t* dims, const uint16_t* ys, const float* topk_gate,
                        const int32_t* slot_row, const int32_t* topk_idx, const uint16_t* x,
                        const uint16_t* const_vectors, uint16_t* y, void* workspace, moe_stream_t stream) {
  MOE_CHECK(check_dims(dims));
  if (dims->T == 0) return MOE_OK;
  if (!ys || !topk_gate || !slot_row || !y || !workspace) return MOE_ERR_INVALID_ARG;
  if (dims->C + dims->V > 0 && (!topk_idx || (dims->C > 0 && !x) || (dims->V > 0 && !const_vectors)))
    return MOE_ERR_INVALID_ARG;
  return launch_combine(*dims, ys, y, topk_gate, slot_row, topk_idx, x, const_vectors, y, S(stream), workspace);
}

int moe_aux_sums(const moe_dims_t* dims, const void* workspace, double* sums, moe_stream_t stream) {
  MOE_CHECK(check_dims(dims));
  if (!workspace || !sums) return MOE_ERR_INVALID_ARG;
  if (dims->T == 0) return cuda_status(cudaMemsetAsync(sums, 0, sizeof(double) * aux_sums_count(*dims), S(stream)));
  return launch_aux(*dims, workspace, sums, nullptr, nullptr, nullptr, nullptr, S(stream));
}

int moe_aux_sums_accumulate(const moe_dims_t* dims, const void* workspace, double* sums, moe_stream_t stream) {
  MOE_CHECK(check_dims(dims));
  if (!workspace || !sums) return MOE_ERR_INVALID_ARG;
  if (dims->T == 0) return MOE_OK;
  return launch_aux(*dims, workspace, sums, nullptr, nullptr, nullptr, nullptr, S(stream), true);
}

int moe_aux_finalize(const moe_dims_t* dims, const double* sums, int32_t* counts_ext, float* P, float* losses,
                     moe_stream_t stream) {
  MOE_CHECK(check_dims(dims));
  if (!sums || !counts_ext || !P || !losses) return MOE_ERR_INVALID_ARG;
  return launch_aux(*dims, nullptr, nullptr, sums, counts_ext, P, losses, S(stream));
}

int moe_aux(const moe_dims_t* dims, const void* workspace, int32_t* counts_ext, float* P, float* losses,
            moe_stream_t stream) {
  MOE_CHECK(check_dims(dims));
  if (dims->T == 0) return MOE_OK;
  if (!workspace || !counts_ext || !P || !losses) return MOE_ERR_INVALID_ARG;
  return launch_aux(*dims, workspace, nullptr, nullptr, counts_ext, P, losses, S(stream));
}

int moe_forward(const moe_dims_t* dims, const moe_weights_t* w, const uint16_t* x, const float* tok_null_bias,
                const moe_outputs_t* out, void* workspace, moe_stream_t stream) {
  MOE_CHECK(check_dims(dims));
  if (dims->T == 0) return MOE_OK;
  if (!w || !out || !x || !workspace) return MOE_ERR_INVALID_ARG;
  if (!w->w_router || !w->gate_up || !w->w_down || !w->shared_gate_up || !w->shared_down)
    return MOE_ERR_INVALID_ARG;
  if (dims->V > 0 && !w->const_vectors) return MOE_ERR_INVALID_ARG;
  if (!out->topk_idx || !out->topk_gate || !out->n_real || !out->counts || !out->offsets || !out->perm_tok ||
      !out->slot_row || !out->h || !out->h_shared || !out->ys || !out->y || !out->counts_ext || !out->P ||
      !out->losses)
    return MOE_ERR_INVALID_ARG;
  // saved pre-activations: both buffers or neither, and only with the gathered copy xs
  if ((out->z != nullptr) != (out->z_shared != nullptr) || (out->z && !out->xs)) return MOE_ERR_INVALID_ARG;
  const cudaStream_t st = S(stream);
  MOE_CHECK(launch_route(*dims, x, w->w_router, w->router_bias, tok_null_bias, out->logits, out->topk_idx,
                         out->topk_gate, out->n_real, workspace, st, w->router_split));
  MOE_CHECK(launch_dispatch(*dims, x, out->topk_idx, workspace, out->counts, out->offsets, out->perm_tok,
                            out->slot_row, out->xs, out->counts_ext, out->P, out->losses, st));
  if (out->z) {
    // training: the pre-activations are kept for the backward pass (copy path only)
    MOE_CHECK(launch_gate_up_save(*dims, out->xs, x, out->offsets, w->gate_up, w->shared_gate_up, out->h,
                                  out->h_shared, out->z, out->z_shared, workspace, st));
  } else {
    // xs == NULL: gate/up gathers the routed rows of x by TMA (no copies written by dispatch)
    MOE_CHECK(launch_gate_up_perm(*dims, out->xs, x, out->offsets, out->xs ? nullptr : out->perm_tok, w->gate_up,
                                  w->shared_gate_up, out->h, out->h_shared, workspace, st));
  }
  if (out->shared_out == nullptr)  // the combine runs in the down GEMM's shared-expert tiles
    return launch_down_combine(*dims, out->offsets, out->h, out->h_shared, w->w_down, w->shared_down, out->ys,
                               out->topk_gate, out->slot_row, out->topk_idx, x, w->const_vectors, out->y,
                               workspace, st);
  MOE_CHECK(launch_down(*dims, out->offsets, out->h, out->h_shared, w->w_down, w->shared_down, out->ys,
                        out->shared_out, workspace, st));
  // in place (shared_out == y): only the tokens the route listed as having a source
  return launch_combine(*dims, out->ys, out->shared_out, out->topk_gate, out->slot_row, out->topk_idx, x,
                        w->const_vectors, out->y, st, out->shared_out == out->y ? workspace : nullptr);
}

int moe_get_device_status(const void* workspace, moe_stream_t stream) {
  if (!workspace) return MOE_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(S(stream)) != cudaSuccess) return MOE_ERR_CUDA;
  uint32_t st = 0;
  if (cudaMemcpy(&st, workspace, sizeof(st), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  if (st & kStatusTimeout) return MOE_ERR_TIMEOUT;
  if (st & kStatusBounds) return MOE_ERR_DEVICE_BOUNDS;
  return MOE_OK;
}

int moe_clear_device_status(void* workspace, moe_stream_t stream) {
  if (!workspace) return MOE_ERR_INVALID_ARG;
  return cuda_status(cudaMemsetAsync(workspace, 0, sizeof(uint32_t), S(stream)));
}

int moe_selftest_bounded_wait(void* workspace, uint64_t limit_ns, moe_stream_t stream) {
  if (!workspace) return MOE_ERR_INVALID_ARG;
  if (limit_ns < 1000ull || limit_ns > 10000000000ull) return MOE_ERR_INVALID_ARG;
  return launch_selftest_wait(workspace, (unsigned long long)limit_ns, S(stream));
}

}  // extern "C"
