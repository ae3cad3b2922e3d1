// C ABI entry points of the backward pass (declared in include/moe_null.h): host-side
// argument checks, then stream-ordered launches into the caller's backward workspace.
#include "moe_internal.cuh"

using namespace moe;

#define MOE_CHECK(expr)          \
  do {                           \
    const int _r = (expr);       \
    if (_r != MOE_OK) return _r; \
  } while (0)

static inline cudaStream_t S(moe_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

static int check_pp_inputs(const moe_dims_t* d, const int32_t* topk_idx, const uint16_t* x, const uint16_t* cv) {
  if (d->C + d->V > 0 && (!topk_idx || (d->C > 0 && !x) || (d->V > 0 && !cv))) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

// The five expert GEMMs. With w->w_router set, the router's input gradient ds W_r (from the
// split ds that the router backward left in the workspace) is added to dx_shared inside the
// shared expert's gate/up dgrad.
static int expert_ffn_bwd(const moe_dims_t& d, const moe_weights_t* w, const moe_saved_t* sv, const uint16_t* dys,
                          const uint16_t* dy, uint16_t* dxs, uint16_t* dx_shared, const moe_grads_t* g, void* ws,
                          cudaStream_t st) {
  const BwdLayout L = bwd_layout(d);
  uint32_t* status = ws_ptr<uint32_t>(ws, L.hdr);
  uint16_t* dh = ws_ptr<uint16_t>(ws, L.dh);
  uint16_t* dhs = ws_ptr<uint16_t>(ws, L.dhs);
  uint16_t* dz = ws_ptr<uint16_t>(ws, L.dz);
  uint16_t* dzs = ws_ptr<uint16_t>(ws, L.dzs);
  float* spart = ws_ptr<float>(ws, L.spart);
  uint16_t* dsplit = nullptr;
  uint16_t* w2 = nullptr;
  if (w->w_router) {
    dsplit = ws_ptr<uint16_t>(ws, L.dsplit);
    w2 = ws_ptr<uint16_t>(ws, L.w2);
    MOE_CHECK(launch_router_split2(d, w->w_router, w2, st));
  }
  MOE_CHECK(launch_dgrad_down(d, sv->offsets, dys, dy, w->w_down, w->shared_down, dh, dhs, status, st));
  if (sv->z && sv->z_shared)  // training mode: pre-activations saved by the forward
    MOE_CHECK(launch_swiglu_bwd_saved(d, sv->offsets, sv->z, sv->z_shared, dh, dhs, dz, dzs, status, st));
  else
    MOE_CHECK(launch_swiglu_backward(d, sv->offsets, sv->xs, sv->x, w->gate_up, w->shared_gate_up, dh, dhs, dz, dzs,
                                     status, st));
  MOE_CHECK(launch_wgrad_down(d, sv->offsets, dys, dy, sv->h, sv->h_shared, g->dw_down, g->dws_down, spart, status,
                              st));
  MOE_CHECK(launch_dgrad_gate_up(d, sv->offsets, dz, dzs, w->gate_up, w->shared_gate_up, dsplit, w2, dxs, dx_shared,
                                 status, st));
  return launch_wgrad_gate_up(d, sv->offsets, dz, dzs, sv->xs, sv->x, g->dw_gate, g->dw_up, g->dws_gate, g->dws_up,
                              spart, status, st);
}

static int router_wgrad(const moe_dims_t& d, const uint16_t* x, float* dw_router, float* dbias, void* ws,
                        cudaStream_t st) {
  const BwdLayout L = bwd_layout(d);
  float* part = ws_ptr<float>(ws, L.rpart);
  MOE_CHECK(launch_router_wgrad_tc(d, ws_ptr<uint16_t>(ws, L.dsplit), x, part, ws_ptr<uint32_t>(ws, L.hdr), st));
  return launch_router_wgrad_reduce(d, part, router_wgrad_split(d, nullptr), ws_ptr<float>(ws, L.bpart), dw_router,
                                    dbias, st);
}

static bool saved_ok(const moe_saved_t* s, const moe_dims_t* d) {
  return s && s->x && s->logits && s->topk_idx && s->topk_gate && s->offsets && s->slot_row && s->xs && s->h &&
         s->h_shared && s->ys && s->counts_ext && s->t_total >= (int64_t)d->T && s->t_total > 0 &&
         ((s->z != nullptr) == (s->z_shared != nullptr));
}

static bool expert_grads_ok(const moe_grads_t* g) {
  return g && g->dw_gate && g->dw_up && g->dw_down && g->dws_gate && g->dws_up && g->dws_down;
}

extern "C" {

size_t moe_backward_workspace_bytes(const moe_dims_t* dims) {
  if (check_dims(dims) != MOE_OK) return 0;
  return bwd_layout(*dims).total;
}

int moe_combine_backward(const moe_dims_t* dims, const uint16_t* dy, const uint16_t* ys, const float* topk_gate,
                         const int32_t* slot_row, const int32_t* topk_idx, const uint16_t* x,
                         const uint16_t* const_vectors, uint16_t* dys, float* dg, void* bwd_workspace,
                         moe_stream_t stream) {
  MOE_CHECK(check_dims(dims));
  if (dims->T == 0) return MOE_OK;
  if (!dy || !ys || !topk_gate || !slot_row || !dys || !dg || !bwd_workspace) return MOE_ERR_INVALID_ARG;
  MOE_CHECK(check_pp_inputs(dims, topk_idx, x, const_vectors));
  const BwdLayout L = bwd_layout(*dims);
  return launch_combine_bwd(*dims, dy, ys, topk_gate, slot_row, topk_idx, x, const_vectors, dys, dg,
                            ws_ptr<uint32_t>(bwd_workspace, L.hdr), S(stream));
}

int moe_router_backward(const moe_dims_t* dims, const float* logits, const int32_t* topk_idx, const float* topk_gate,
                        const float* dg, const int32_t* counts_ext, int64_t t_total, float alpha, float beta,
                        float* ds, float* dtok_null_bias, void* bwd_workspace, moe_stream_t stream) {
  MOE_CHECK(check_dims(dims));
  if (dims->T == 0) return MOE_OK;
  if (!logits || !topk_idx || !topk_gate || !dg || !counts_ext || !ds || !bwd_workspace) return MOE_ERR_INVALID_ARG;
  if (t_total < (int64_t)dims->T || t_total <= 0) return MOE_ERR_INVALID_ARG;
  const BwdLayout L = bwd_layout(*dims);
  return launch_router_bwd(*dims, logits, topk_idx, topk_gate, dg, counts_ext, (long long)t_total, alpha, beta, ds,
                           dtok_null_bias, ws_ptr<uint16_t>(bwd_workspace, L.dsplit),
                           ws_ptr<float>(bwd_workspace, L.bpart), S(stream));
}

int moe_router_weight_grad(const moe_dims_t* dims, const uint16_t* x, float* dw_router, float* dbias,
                           void* bwd_workspace, moe_stream_t stream) {
  MOE_CHECK(check_dims(dims));
  if (!dw_router) return MOE_ERR_INVALID_ARG;
  const size_t rows = (size_t)router_rows(*dims);
  if (dims->T == 0) {
    MOE_CHECK(cuda_status(cudaMemsetAsync(dw_router, 0, sizeof(float) * rows * dims->d, S(stream))));
    return dbias ? cuda_status(cudaMemsetAsync(dbias, 0, sizeof(float) * rows, S(stream))) : MOE_OK;
  }
  if (!x || !bwd_workspace) return MOE_ERR_INVALID_ARG;
  return router_wgrad(*dims, x, dw_router, dbias, bwd_workspace, S(stream));
}

int moe_expert_ffn_backward(const moe_dims_t* dims, const moe_weights_t* w, const moe_saved_t* saved,
                            const uint16_t* dys, const uint16_t* dy, uint16_t* dxs, uint16_t* dx_shared,
                            const moe_grads_t* g, void* bwd_workspace, moe_stream_t stream) {
  MOE_CHECK(check_dims(dims));
  if (dims->T == 0) return MOE_OK;
  if (!w || !w->gate_up || !w->w_down || !w->shared_gate_up || !w->shared_down) return MOE_ERR_INVALID_ARG;
  if (!saved || !saved->x || !saved->xs || !saved->offsets || !saved->h || !saved->h_shared) return MOE_ERR_INVALID_ARG;
  if ((saved->z != nullptr) != (saved->z_shared != nullptr)) return MOE_ERR_INVALID_ARG;
  if (!dys || !dy || !dxs || !dx_shared || !expert_grads_ok(g) || !bwd_workspace) return MOE_ERR_INVALID_ARG;
  return expert_ffn_bwd(*dims, w, saved, dys, dy, dxs, dx_shared, g, bwd_workspace, S(stream));
}

// The five GEMM stages of moe_expert_ffn_backward, one launch each (the weight gradients
// add the reduction of the shared expert's K chunks when T needs more than one).
int moe_expert_dgrad_down(const moe_dims_t* dims, const int32_t* offsets, const uint16_t* dys, const uint16_t* dy,
                          const uint16_t* w_down, const uint16_t* shared_down, void* bwd_workspace,
                          moe_stream_t stream) {
  MOE_CHECK(check_dims(dims));
  if (dims->T == 0) return MOE_OK;
  if (!offsets || !dys || !dy || !w_down || !shared_down || !bwd_workspace) return MOE_ERR_INVALID_ARG;
  const BwdLayout L = bwd_layout(*dims);
  void* ws = bwd_workspace;
  return launch_dgrad_down(*dims, offsets, dys, dy, w_down, shared_down, ws_ptr<uint16_t>(ws, L.dh),
                           ws_ptr<uint16_t>(ws, L.dhs), ws_ptr<uint32_t>(ws, L.hdr), S(stream));
}

int moe_expert_swiglu_backward(const moe_dims_t* dims, const uint16_t* xs, const uint16_t* x, const int32_t* offsets,
                               const uint16_t* gate_up, const uint16_t* shared_gate_up, void* bwd_workspace,
                               moe_stream_t stream) {
  MOE_CHECK(check_dims(dims));
  if (dims->T == 0) return MOE_OK;
  if (!xs || !x || !offsets || !gate_up || !shared_gate_up || !bwd_workspace) return MOE_ERR_INVALID_ARG;
  const BwdLayout L = bwd_layout(*dims);
  void* ws = bwd_workspace;
  return launch_swiglu_backward(*dims, offsets, xs, x, gate_up, shared_gate_up, ws_ptr<uint16_t>(ws, L.dh),
                                ws_ptr<uint16_t>(ws, L.dhs), ws_ptr<uint16_t>(ws, L.dz), ws_ptr<uint16_t>(ws, L.dzs),
                                ws_ptr<uint32_t>(ws, L.hdr), S(stream));
}

int moe_expert_swiglu_backward_saved(const moe_dims_t* dims, const int32_t* offsets, const uint16_t* z,
                                     const uint16_t* z_shared, void* bwd_workspace, moe_stream_t stream) {
  MOE_CHECK(check_dims(dims));
  if (dims->T == 0) return MOE_OK;
  if (!offsets || !z || !z_shared || !bwd_workspace) return MOE_ERR_INVALID_ARG;
  const BwdLayout L = bwd_layout(*dims);
  void* ws = bwd_workspace;
  return launch_swiglu_bwd_saved(*dims, offsets, z, z_shared, ws_ptr<uint16_t>(ws, L.dh), ws_ptr<uint16_t>(ws, L.dhs),
                                 ws_ptr<uint16_t>(ws, L.dz), ws_ptr<uint16_t>(ws, L.dzs), ws_ptr<uint32_t>(ws, L.hdr),
                                 S(stream));
}

int moe_expert_wgrad_down(const moe_dims_t* dims, const int32_t* offsets, const uint16_t* dys, const uint16_t* dy,
                          const uint16_t* h, const uint16_t* h_shared, uint16_t* dw_down, uint16_t* dws_down,
                          void* bwd_workspace, moe_stream_t stream) {
  MOE_CHECK(check_dims(dims));
  if (dims->T == 0) return MOE_OK;
  if (!offsets || !dys || !dy || !h || !h_shared || !dw_down || !dws_down || !bwd_workspace)
    return MOE_ERR_INVALID_ARG;
  const BwdLayout L = bwd_layout(*dims);
  void* ws = bwd_workspace;
  return launch_wgrad_down(*dims, offsets, dys, dy, h, h_shared, dw_down, dws_down, ws_ptr<float>(ws, L.spart),
                           ws_ptr<uint32_t>(ws, L.hdr), S(stream));
}

int moe_expert_dgrad_gate_up(const moe_dims_t* dims, const int32_t* offsets, const uint16_t* gate_up,
                             const uint16_t* shared_gate_up, const float* w_router, uint16_t* dxs,
                             uint16_t* dx_shared, void* bwd_workspace, moe_stream_t stream) {
  MOE_CHECK(check_dims(dims));
  if (dims->T == 0) return MOE_OK;
  if (!offsets || !gate_up || !shared_gate_up || !dxs || !dx_shared || !bwd_workspace) return MOE_ERR_INVALID_ARG;
  const BwdLayout L = bwd_layout(*dims);
  void* ws = bwd_workspace;
  uint16_t* dsplit = nullptr;
  uint16_t* w2 = nullptr;
  if (w_router) {
    dsplit = ws_ptr<uint16_t>(ws, L.dsplit);
    w2 = ws_ptr<uint16_t>(ws, L.w2);
    MOE_CHECK(launch_router_split2(*dims, w_router, w2, S(stream)));
  }
  return launch_dgrad_gate_up(*dims, offsets, ws_ptr<uint16_t>(ws, L.dz), ws_ptr<uint16_t>(ws, L.dzs), gate_up,
                              shared_gate_up, dsplit, w2, dxs, dx_shared, ws_ptr<uint32_t>(ws, L.hdr), S(stream));
}

int moe_expert_wgrad_gate_up(const moe_dims_t* dims, const int32_t* offsets, const uint16_t* xs, const uint16_t* x,
                             uint16_t* dw_gate, uint16_t* dw_up, uint16_t* dws_gate, uint16_t* dws_up,
                             void* bwd_workspace, moe_stream_t stream) {
  MOE_CHECK(check_dims(dims));
  if (dims->T == 0) return MOE_OK;
  if (!offsets || !xs || !x || !dw_gate || !dw_up || !dws_gate || !dws_up || !bwd_workspace)
    return MOE_ERR_INVALID_ARG;
  const BwdLayout L = bwd_layout(*dims);
  void* ws = bwd_workspace;
  return launch_wgrad_gate_up(*dims, offsets, ws_ptr<uint16_t>(ws, L.dz), ws_ptr<uint16_t>(ws, L.dzs), xs, x,
                              dw_gate, dw_up, dws_gate, dws_up, ws_ptr<float>(ws, L.spart),
                              ws_ptr<uint32_t>(ws, L.hdr), S(stream));
}

int moe_input_grad(const moe_dims_t* dims, const uint16_t* dx_shared, const uint16_t* dxs, const int32_t* slot_row,
                   const int32_t* topk_idx, const float* topk_gate, const uint16_t* dy, uint16_t* dx,
                   void* bwd_workspace, moe_stream_t stream) {
  MOE_CHECK(check_dims(dims));
  if (dims->T == 0) return MOE_OK;
  if (!dx_shared || !dxs || !slot_row || !dx || !bwd_workspace) return MOE_ERR_INVALID_ARG;
  if (dims->C > 0 && (!topk_idx || !topk_gate || !dy)) return MOE_ERR_INVALID_ARG;
  const BwdLayout L = bwd_layout(*dims);
  return launch_input_grad(*dims, dx_shared, dxs, slot_row, topk_idx, topk_gate, dy, dx,
                           ws_ptr<uint32_t>(bwd_workspace, L.hdr), S(stream));
}

int moe_backward(const moe_dims_t* dims, const moe_weights_t* w, const moe_saved_t* saved, const uint16_t* dy,
                 float alpha, float beta, const moe_grads_t* g, void* bwd_workspace, moe_stream_t stream) {
  MOE_CHECK(check_dims(dims));
  if (dims->T == 0) return MOE_OK;
  if (!w || !w->w_router || !w->gate_up || !w->w_down || !w->shared_gate_up || !w->shared_down)
    return MOE_ERR_INVALID_ARG;
  if (dims->V > 0 && !w->const_vectors) return MOE_ERR_INVALID_ARG;
  if (!saved_ok(saved, dims) || !dy || !expert_grads_ok(g) || !g->dx || !g->dw_router || !bwd_workspace)
    return MOE_ERR_INVALID_ARG;
  if (dims->V > 0 && !g->dconst) return MOE_ERR_INVALID_ARG;
  const moe_dims_t& d = *dims;
  const cudaStream_t st = S(stream);
  const BwdLayout L = bwd_layout(d);
  void* ws = bwd_workspace;
  uint32_t* status = ws_ptr<uint32_t>(ws, L.hdr);
  uint16_t* dys = ws_ptr<uint16_t>(ws, L.dys);
  uint16_t* dxs = ws_ptr<uint16_t>(ws, L.dxs);
  float* dg = ws_ptr<float>(ws, L.dg);
  float* ds = ws_ptr<float>(ws, L.ds);
  MOE_CHECK(cuda_status(cudaMemsetAsync(status, 0, sizeof(uint32_t), st)));
  MOE_CHECK(launch_combine_bwd(d, dy, saved->ys, saved->topk_gate, saved->slot_row, saved->topk_idx, saved->x,
                               w->const_vectors, dys, dg, status, st));
  MOE_CHECK(launch_router_bwd(d, saved->logits, saved->topk_idx, saved->topk_gate, dg, saved->counts_ext,
                              (long long)saved->t_total, alpha, beta, ds, g->dtok_null_bias,
                              ws_ptr<uint16_t>(ws, L.dsplit), ws_ptr<float>(ws, L.bpart), st));
  MOE_CHECK(router_wgrad(d, saved->x, g->dw_router, g->dbias, ws, st));
  // the shared expert's (and the router's) input gradient goes straight into dx; the input
  // gradient gather then adds the routed and copy-expert terms in place, skipping the tokens
  // that have none
  MOE_CHECK(expert_ffn_bwd(d, w, saved, dys, dy, dxs, g->dx, g, ws, st));
  MOE_CHECK(launch_input_grad(d, g->dx, dxs, saved->slot_row, saved->topk_idx, saved->topk_gate, dy, g->dx, status,
                              st));
  return launch_const_grad(d, saved->topk_idx, saved->topk_gate, dy, g->dconst, st);
}

}  // extern "C"
