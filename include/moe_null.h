/*
 * moe_null.h -- C ABI of the B200 (sm_100a) forward hot path of a token-choice
 * MoE layer with zero-compute null experts.
 *
 * The layer (Kilian et al., "Improving MoE Compute Efficiency by Composing
 * Weight and Data Sparsity", paper-review page, section 三 技术架构):
 *
 *   y = E_shared(x) + sum_{i in top-K, i real} g_i(x) * E_i(x)
 *
 * The router emits N real logits plus one null logit (Null Expert 机制); the
 * null logit is replicated M times before top-K, so the pool has N+M slots
 * (indices N..N+M-1 are the null copies, which compute nothing). Gates are
 * renormalised over the selected real experts only. The layer also emits the
 * load-balance statistics L_bal = N * sum_{i<N+M} f_i P_i (负载均衡损失) and the
 * Z-loss L_z = mean_t (log sum_{i<N+M} e^{s_i})^2 (Z-Loss).
 *
 * Optionally the pool also holds MoE++'s other zero-computation experts (MoE++
 * explainer page, 核心创新：三种零计算专家): C copy experts (output x) and V
 * constant experts (output a learned vector c_j), each with its own router row
 * after the null logit. Pool order: reals 0..N-1, null copies N..N+M-1, copy
 * experts N+M..N+M+C-1, constant experts N+M+C..N+M+C+V-1. They take gates like
 * real experts (renormalisation runs over every selected slot except null
 * copies) and cost no GEMM work: combine adds g x and g c_j. C = V = 0 is the
 * paper's layer.
 *
 * Conventions shared by every entry point:
 *  - All pointers except `dims`, `w` and `out` (host structs) are DEVICE
 *    pointers on the current CUDA device. bf16 tensors are passed as uint16_t
 *    bit patterns. All tensors are dense row-major.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream). Every call
 *    only enqueues work on it and returns; none synchronises the host except
 *    moe_get_device_status.
 *  - The caller allocates and owns every buffer, the workspace included. The
 *    library allocates no device memory and keeps no per-call state; it does
 *    cache, per device and process, the SM count and kernel attributes.
 *  - Return value: MOE_OK (0) or a negative moe_status_t. Argument errors are
 *    detected on the host before anything is enqueued. A failure detected on
 *    the device (a bounded wait that ran out, a guard) is recorded in a status
 *    word inside the workspace; read it with moe_get_device_status.
 *  - T = 0 is a no-op that returns MOE_OK.
 *  - Non-finite inputs give undefined routing.
 *  - Limits: 1 <= N <= 64, 0 <= M, 1 <= K <= 16, K <= N + M + C + V, d a
 *    multiple of 128 (128..8192), F and F_shared multiples of 64 (64..16384),
 *    T*K < 2^31; with C + V > 0 also N + 1 + C + V <= 80 (and the tensor-core
 *    router).
 *    Outside them: MOE_ERR_UNSUPPORTED (or MOE_ERR_INVALID_ARG for values that
 *    are never valid, e.g. K < 1, M < 0, T < 0).
 *
 * Workspace: moe_workspace_bytes(dims) bytes, 256-byte aligned. moe_route
 * writes it (it clears what must start at zero itself); moe_dispatch,
 * moe_aux*, moe_expert_ffn and moe_combine_inplace read it. Among what moe_route
 * leaves there is the list of tokens with a source (a real, copy or constant
 * expert among their K slots), which the in-place combine visits. One workspace serves one layer call at
 * a time: two calls in flight on different streams must use two workspaces.
 */
#ifndef MOE_NULL_H
#define MOE_NULL_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_NULL_ABI_VERSION 6

typedef void* moe_stream_t; /* a cudaStream_t */

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = -1,   /* null pointer, negative size, K < 1, ... */
  MOE_ERR_UNSUPPORTED = -2,   /* valid but outside this library's limits */
  MOE_ERR_CUDA = -3,          /* a CUDA runtime/driver call failed */
  MOE_ERR_TIMEOUT = -4,       /* a device-side bounded wait ran out */
  MOE_ERR_DEVICE_BOUNDS = -5  /* a device-side guard saw an out-of-range index */
} moe_status_t;

/* Layer sizes. T tokens, model width d, N real experts, M null copies, top-K,
 * routed expert ffn width F, shared expert ffn width F_shared. flags: 0 or a
 * combination of the MOE_FLAG_* bits below. Every call of one layer (route,
 * dispatch, workspace sizing, ...) must see the same flags. */
/* Router product on the fp32 CUDA cores instead of the tensor cores (see
 * moe_route). Both give logits within the fp32 dot-product error bound; this
 * path is several times slower on the router product. */
#define MOE_FLAG_ROUTER_FP32_CORES 1u

/* Expert GEMMs on CTA pairs: 256 x 256 tiles, one tcgen05 MMA shared by the
 * two CTAs of a cluster, where the column tiles are 256 wide (F and F_shared
 * multiples of 128 for gate/up, d a multiple of 256 for down); otherwise, and
 * by default, single-CTA 128 x 256 tiles. A pair loads a third less operand
 * data per flop but rounds each expert's rows up to 256 instead of 128; on
 * this part it is ahead only when experts hold thousands of rows. Same results
 * up to fp32 accumulation order. */
#define MOE_FLAG_FFN_CTA_PAIR 2u

/* Weight gradients of the backward's expert GEMMs (moe_expert_wgrad_down,
 * moe_expert_wgrad_gate_up, moe_backward) on CTA pairs: 256 output rows x 256
 * columns per tile, one tcgen05 MMA shared by the two CTAs of a cluster, where
 * the output rows per expert are a multiple of 256 (d for W_down, 2 F and
 * 2 F_shared for gate/up) and the columns a multiple of 256 (F and F_shared,
 * d); otherwise single-CTA tiles. The same fp32 sums in the same order as the
 * single-CTA tiles, so the same results bit for bit. */
#define MOE_FLAG_WGRAD_CTA_PAIR 4u

typedef struct moe_dims {
  int32_t T, d, N, M, K, F, F_shared;
  uint32_t flags;
  int32_t C, V;  /* MoE++ copy and constant experts (0, 0: null experts only) */
} moe_dims_t;

/* Weights of one layer (device pointers). */
typedef struct moe_weights {
  const float* w_router;        /* [N+1+C+V, d] fp32; row N is the null logit,
                                   rows N+1.. the copy, then constant experts   */
  const float* router_bias;     /* [N+1+C+V] fp32 or NULL (added to each logit) */
  const uint16_t* gate_up;      /* [N, 2F, d] bf16, from moe_pack_gate_up       */
  const uint16_t* w_down;       /* [N, d, F] bf16                               */
  const uint16_t* shared_gate_up; /* [2F_shared, d] bf16, from moe_pack_gate_up */
  const uint16_t* shared_down;  /* [d, F_shared] bf16                           */
  const uint16_t* const_vectors; /* [V, d] bf16 constant experts' outputs, or
                                    NULL when V = 0                             */
  const uint16_t* router_split;  /* [3 * P, d] bf16 from moe_prepare_router, or
                                    NULL: moe_forward then splits w_router for
                                    each call (tensor-core router only)         */
} moe_weights_t;

/* Outputs and intermediates of moe_forward (device pointers). R_cap = T*K. */
typedef struct moe_outputs {
  float* logits;        /* [T, N+1] fp32, or NULL to skip                        */
  int32_t* topk_idx;    /* [T, K] pool indices in rank order                     */
  float* topk_gate;     /* [T, K] fp32, 0 for null slots                         */
  int32_t* n_real;      /* [T] real experts per token                            */
  int32_t* counts;      /* [N] rows per expert                                   */
  int32_t* offsets;     /* [N+1] exclusive scan of counts; offsets[N] = R        */
  int32_t* perm_tok;    /* [R_cap] token of each expert-contiguous row (first R) */
  int32_t* slot_row;    /* [T, K] row of each slot in xs/h/ys, -1 for nulls      */
  uint16_t* xs;         /* [R_cap, d] bf16 gathered rows, or NULL: gate/up then
                           gathers the rows of x itself and no copies are written */
  uint16_t* h;          /* [R_cap, F] bf16 routed SwiGLU activations             */
  uint16_t* h_shared;   /* [T, F_shared] bf16 shared SwiGLU activations          */
  uint16_t* ys;         /* [R_cap, d] bf16 routed expert outputs                 */
  uint16_t* shared_out; /* [T, d] bf16 shared expert output; or y itself: the down
                           GEMM then writes it into y and the combine adds the routed
                           rows in place, skipping tokens that have none; or NULL:
                           the combine is folded into the down GEMM
                           (moe_expert_down_combine). y is the same in all three.   */
  uint16_t* y;          /* [T, d] bf16 layer output                              */
  int32_t* counts_ext;  /* [N+M+C+V] tokens per pool slot                        */
  float* P;             /* [N+M+C+V] mean routing probability per pool slot      */
  float* losses;        /* [2] = {L_bal, L_z}                                    */
  uint16_t* z;          /* [R_cap, 2F] bf16 gate/up pre-activations (packed order:
                           64-column panels of 64 gate then 64 up columns), or NULL.
                           Training: with z and z_shared set (and xs), the forward also
                           writes them and moe_backward skips their recomputation.     */
  uint16_t* z_shared;   /* [T, 2F_shared] bf16, or NULL (set both or neither)        */
} moe_outputs_t;

/* ABI version (MOE_NULL_ABI_VERSION) of the loaded library. */
MOE_API int moe_abi_version(void);

/* Static text for a moe_status_t value. Never NULL. */
MOE_API const char* moe_status_string(int status);

/* Host-side check of `dims` against the limits above. */
MOE_API int moe_check_dims(const moe_dims_t* dims);

/* Workspace size in bytes for `dims` (0 if dims are invalid). */
MOE_API size_t moe_workspace_bytes(const moe_dims_t* dims);

/* Element count (bf16) of the packed gate/up weights: routed N*2F*d and shared
 * 2*F_shared*d. Packing interleaves gate and up rows in panels of 64 rows
 * (64 gate rows of a panel, then the matching 64 up rows), so that one
 * tensor-core tile holds matching gate and up columns for the SwiGLU epilogue.
 * Either output pointer of moe_pack_gate_up may be NULL to skip that part. */
MOE_API size_t moe_packed_gate_up_elems(const moe_dims_t* dims, int shared);

/* One-time weight packing (device copy kernel). w_gate/w_up [N, F, d] ->
 * gate_up [N, 2F, d]; ws_gate/ws_up [F_shared, d] -> shared_gate_up
 * [2F_shared, d]. */
MOE_API int moe_pack_gate_up(const moe_dims_t* dims, const uint16_t* w_gate, const uint16_t* w_up,
                     const uint16_t* ws_gate, const uint16_t* ws_up, uint16_t* gate_up,
                     uint16_t* shared_gate_up, moe_stream_t stream);

/* Element count (bf16) of the router weight split into three bf16 terms for the
 * tensor-core router: 3 * P * d with P = N+1+C+V rounded up to a multiple of 16. */
MOE_API size_t moe_router_split_elems(const moe_dims_t* dims);

/* One-time preparation of the router weight for the tensor-core router (like
 * moe_pack_gate_up for the expert weights): router_split [3 * P, d] receives the
 * exact three-term bf16 split of w_router [N+1+C+V, d] (hi, mid and lo rows, zero
 * rows past N+1+C+V; see moe_route). Passed as moe_weights_t.router_split, it spares
 * moe_forward the split of every call. Redo it whenever w_router changes. */
MOE_API int moe_prepare_router(const moe_dims_t* dims, const float* w_router, uint16_t* router_split,
                               moe_stream_t stream);

/* Routing (section 三: Null Expert 机制, 阈值解释, 负载均衡损失, Z-Loss).
 *  s[t, j] = sum_c fp32(x[t,c]) * w_router[j,c] + bias[j] (+ tok_null_bias[t]
 *  for j = N), to fp32 accuracy: by default on the tensor cores, with each
 *  fp32 weight split exactly into three bf16 terms (hi + mid + lo; bf16
 *  products are exact, accumulation is fp32, the three partial sums are added
 *  in fp32), or, with MOE_FLAG_ROUTER_FP32_CORES, as an fp32 FMA product on the
 *  CUDA cores. x and w_router must be 16-byte aligned (x is read by TMA).
 *  Over the pool [s_0..s_{N-1}, s_N x M, s_{N+1}..s_{N+C+V}] (pool indices:
 *  reals, null copies, copy experts, constant experts): lse_t, p_{t,i}; top-K
 *  in (value desc, pool index asc) order -- a real logit equal to the null
 *  logit precedes every null copy, null copies fill N, N+1, ... and precede a
 *  copy or constant expert of equal logit; gates = softmax over the selected
 *  slots that are not null copies (0 for null copies, all 0 if only nulls).
 *  With M = 0 the null logit takes no part in anything.
 *  x [T, d] bf16; tok_null_bias [T] or NULL (added to the null logit);
 *  logits_out [T, N+1+C+V] or NULL; topk_idx [T, K] (pool indices); topk_gate
 *  [T, K]; n_real [T] (real experts only). Also fills the workspace with
 *  per-block statistics and the dispatch scan (counts, offsets). */
MOE_API int moe_route(const moe_dims_t* dims, const uint16_t* x, const float* w_router,
              const float* router_bias, const float* tok_null_bias, float* logits_out,
              int32_t* topk_idx, float* topk_gate, int32_t* n_real, void* workspace,
              moe_stream_t stream);

/* moe_route for the tensor-core router with its weight already split by
 * moe_prepare_router (router_split [3 * P, d] bf16): one launch fewer per call.
 * Same results as moe_route. Not for MOE_FLAG_ROUTER_FP32_CORES (MOE_ERR_INVALID_ARG). */
MOE_API int moe_route_prepared(const moe_dims_t* dims, const uint16_t* x, const uint16_t* router_split,
                               const float* router_bias, const float* tok_null_bias, float* logits_out,
                               int32_t* topk_idx, float* topk_gate, int32_t* n_real, void* workspace,
                               moe_stream_t stream);

/* moe_route without a workspace argument, for callers that cannot allocate
 * device memory: plugin-style interfaces that receive only their input and
 * output buffers, and hot paths that must not call cudaMalloc because it can
 * synchronise the device. The paper has no counterpart of this entry point; it
 * is a deployment convenience. Same inputs, outputs and results as moe_route.
 * Its internal scratch is a fixed MOE_ROUTE_NOALLOC_MAX_SCRATCH_BYTES array in
 * the library's own device memory, held by every GPU that uses this entry
 * point from its first call there until the process exits. Shapes whose
 * moe_workspace_bytes exceeds that size are rejected with MOE_ERR_UNSUPPORTED
 * before anything is enqueued. The first call on each device (and the first
 * after the device's context was replaced, e.g. by cudaDeviceReset) looks up
 * the array's device address; make that first call before any stream capture.
 * All calls on a device share the array (each call clears what must start at
 * zero): calls whose GPU work overlaps, e.g. on two unordered streams, race and
 * give wrong results. It allocates nothing and does not fill a workspace for
 * moe_dispatch. Device-side failures are recorded in the array's status word:
 * read it with moe_route_noalloc_device_status. */
#define MOE_ROUTE_NOALLOC_MAX_SCRATCH_BYTES ((size_t)8 << 20)
MOE_API int moe_route_noalloc(const moe_dims_t* dims, const uint16_t* x, const float* w_router,
                              const float* router_bias, const float* tok_null_bias, float* logits_out,
                              int32_t* topk_idx, float* topk_gate, int32_t* n_real,
                              moe_stream_t stream);

/* Synchronises `stream`, then returns MOE_OK or the first device-side error that a
 * moe_route_noalloc call on the current device recorded since the last call cleared
 * it (MOE_ERR_TIMEOUT, MOE_ERR_DEVICE_BOUNDS): the counterpart of
 * moe_get_device_status for the entry point without a workspace. */
MOE_API int moe_route_noalloc_device_status(moe_stream_t stream);

/* Test aid, as moe_selftest_bounded_wait, recording into the status word that
 * moe_route_noalloc_device_status reads; the next moe_route_noalloc call clears it. */
MOE_API int moe_route_noalloc_selftest_bounded_wait(uint64_t limit_ns, moe_stream_t stream);

/* Dispatch (section 三 / 实现: nulls sorted to the end and truncated). After
 * moe_route with the same workspace. counts [N], offsets [N+1]; the real slots
 * are laid out expert by expert, tokens ascending inside an expert: perm_tok
 * [T*K] (first offsets[N] entries valid), slot_row [T, K] (-1 for nulls), and
 * xs [T*K, d] bf16 with xs[slot_row[t,k]] = x[t], or xs = NULL to write no row
 * copies (moe_expert_gate_up_gather then reads the rows of x through
 * perm_tok). Null slots cause no memory traffic. Also reduces the aux
 * statistics into the workspace (see moe_aux). */
MOE_API int moe_dispatch(const moe_dims_t* dims, const uint16_t* x, const int32_t* topk_idx,
                 void* workspace, int32_t* counts, int32_t* offsets, int32_t* perm_tok,
                 int32_t* slot_row, uint16_t* xs, moe_stream_t stream);

/* Expert FFNs (section 三 / 核心公式; 实现: grouped matmul over the truncated
 * list). Two persistent tcgen05/TMEM/TMA grouped GEMMs with per-expert row
 * counts read from `offsets` on the device:
 *   h[r]  = bf16(silu(xs[r] Wg_e^T) * (xs[r] Wu_e^T)),  ys[r] = bf16(h[r] Wd_e^T)
 * for rows r in [offsets[e], offsets[e+1]); the shared expert is one more group
 * over all T rows of x: h_shared, shared_out. bf16 in, fp32 accumulation.
 * h [T*K, F], h_shared [T, F_shared], ys [T*K, d], shared_out [T, d]. */
MOE_API int moe_expert_ffn(const moe_dims_t* dims, const uint16_t* xs, const uint16_t* x,
                   const int32_t* offsets, const uint16_t* gate_up, const uint16_t* w_down,
                   const uint16_t* shared_gate_up, const uint16_t* shared_down, uint16_t* h,
                   uint16_t* h_shared, uint16_t* ys, uint16_t* shared_out, void* workspace,
                   moe_stream_t stream);

/* The two halves of moe_expert_ffn, for callers that time or schedule them
 * separately. moe_expert_gate_up writes h and h_shared (the SwiGLU grouped
 * GEMM); moe_expert_down reads them and writes ys and shared_out. */
MOE_API int moe_expert_gate_up(const moe_dims_t* dims, const uint16_t* xs, const uint16_t* x,
                       const int32_t* offsets, const uint16_t* gate_up,
                       const uint16_t* shared_gate_up, uint16_t* h, uint16_t* h_shared,
                       void* workspace, moe_stream_t stream);
/* moe_expert_gate_up without the gathered copy xs: the routed rows are fetched
 * from x by 16-byte asynchronous copies (cp.async) through perm_tok, the row -> token
 * map of moe_dispatch (row r of expert e's segment is token perm_tok[r]). Same
 * h and h_shared as moe_expert_gate_up on the xs that moe_dispatch would write.
 * x must be 16-byte aligned. */
MOE_API int moe_expert_gate_up_gather(const moe_dims_t* dims, const uint16_t* x, const int32_t* perm_tok,
                                      const int32_t* offsets, const uint16_t* gate_up,
                                      const uint16_t* shared_gate_up, uint16_t* h, uint16_t* h_shared,
                                      void* workspace, moe_stream_t stream);
MOE_API int moe_expert_down(const moe_dims_t* dims, const int32_t* offsets, const uint16_t* h,
                    const uint16_t* h_shared, const uint16_t* w_down, const uint16_t* shared_down,
                    uint16_t* ys, uint16_t* shared_out, void* workspace, moe_stream_t stream);

/* Expert parallelism (MoE tutorial page, 五、通信：All-to-All 为什么是成本中心: the
 * experts are spread over the GPUs, a dispatch all-to-all sends each token's rows to
 * the GPUs that hold its experts and a combine all-to-all brings the outputs back;
 * MoE++ page, 局限性与开放问题 / 分布式部署复杂度: the zero-computation experts live on
 * every GPU, so null slots are never sent). On the rank that holds a shard of the
 * routed experts, these run the two grouped GEMMs over the rows it received:
 *  - dims->N is the number of experts in the shard (the groups); dims->M and dims->K
 *    play no part (pass 0 and 1);
 *  - offsets [N+1] (device) delimit each expert's received rows, expert-contiguous;
 *  - gate_up [N, 2F, d] (packed as by moe_pack_gate_up) and w_down [N, d, F] are the
 *    shard's weights, e.g. pointers into the whole layer's at its first expert;
 *  - rows_cap (>= 1) is the row count of xs, h and ys, independent of T*K: a rank can
 *    receive up to world_size * T * K rows;
 *  - the shared expert runs as usual over the rank's own dims->T tokens of x into
 *    h_shared and shared_out (dims->T = 0: no shared expert, the routed rows still run).
 * Same per-row results as moe_expert_gate_up / moe_expert_down (a row's output does
 * not depend on which tile holds it). Single-CTA tiles. */
MOE_API int moe_expert_gate_up_rows(const moe_dims_t* dims, int64_t rows_cap, const uint16_t* xs,
                                    const uint16_t* x, const int32_t* offsets, const uint16_t* gate_up,
                                    const uint16_t* shared_gate_up, uint16_t* h, uint16_t* h_shared,
                                    void* workspace, moe_stream_t stream);
MOE_API int moe_expert_down_rows(const moe_dims_t* dims, int64_t rows_cap, const int32_t* offsets,
                                 const uint16_t* h, const uint16_t* h_shared, const uint16_t* w_down,
                                 const uint16_t* shared_down, uint16_t* ys, uint16_t* shared_out,
                                 void* workspace, moe_stream_t stream);

/* moe_expert_down + moe_combine in one launch (section 三 / 核心公式): the down
 * GEMM writes ys for the routed rows, and its shared-expert tiles, which come
 * after every routed tile, write y[t] = bf16(bf16(shared[t]) + sum over the
 * token's slots k, in rank order, of topk_gate[t,k] * out_k) with out_k as in
 * moe_combine: the same arithmetic, so y is bit-identical to moe_expert_down
 * followed by moe_combine, without the shared expert's output ever going to
 * memory. A shared tile first waits (bounded; MOE_ERR_TIMEOUT in the status word
 * if it runs out) until the launch's routed tiles have stored their rows, which
 * relies on the persistent grid (one CTA per SM) being resident at once. The
 * workspace must come from moe_route (which clears the two counters this call
 * uses; the call leaves them cleared). Always single-CTA tiles. topk_idx, x and
 * const_vectors are read only when C + V > 0. */
MOE_API int moe_expert_down_combine(const moe_dims_t* dims, const int32_t* offsets, const uint16_t* h,
                                    const uint16_t* h_shared, const uint16_t* w_down,
                                    const uint16_t* shared_down, uint16_t* ys, const float* topk_gate,
                                    const int32_t* slot_row, const int32_t* topk_idx, const uint16_t* x,
                                    const uint16_t* const_vectors, uint16_t* y, void* workspace,
                                    moe_stream_t stream);

/* Combine (section 三 / 核心公式): y[t] = bf16(shared_out[t] + sum over the
 * token's slots k, in rank order, of topk_gate[t,k] * out_k), out_k =
 * ys[slot_row[t,k]] for a real expert, x[t] for a copy expert, const_vectors[j]
 * for constant expert j, nothing for a null copy; fp32 accumulation, one
 * rounding. y [T, d]. topk_idx, x and const_vectors are read only when C + V >
 * 0 (they may be NULL otherwise). shared_out may be y itself (in place): a
 * token with no slot that has an output is then left as it is. */
MOE_API int moe_combine(const moe_dims_t* dims, const uint16_t* ys, const uint16_t* shared_out,
                const float* topk_gate, const int32_t* slot_row, const int32_t* topk_idx,
                const uint16_t* x, const uint16_t* const_vectors, uint16_t* y, moe_stream_t stream);

/* moe_combine in place (shared_out == y) over the route's list of tokens with a
 * source (section 三 / 核心公式 and Null Expert 机制: a token whose K slots are
 * all null copies takes only the shared expert, so y[t] = bf16(shared[t]) is
 * already its result). y [T, d] holds the shared expert's output on entry, as
 * moe_expert_down writes it with shared_out == y. workspace is the one moe_route
 * filled for this batch (same dims); the token list there decides which rows are
 * touched, and y is bit-identical to moe_combine(..., shared_out = y, ...). The
 * list's order depends on the route's timing; the result does not. A list entry
 * outside [0, T) is skipped and sets MOE_ERR_DEVICE_BOUNDS in the status word.
 * topk_idx, x and const_vectors are read only when C + V > 0. */
MOE_API int moe_combine_inplace(const moe_dims_t* dims, const uint16_t* ys, const float* topk_gate,
                                const int32_t* slot_row, const int32_t* topk_idx, const uint16_t* x,
                                const uint16_t* const_vectors, uint16_t* y, void* workspace,
                                moe_stream_t stream);

/* Number of doubles in the additive aux statistics of a token shard:
 * [counts_real (N) | null histogram (K+1), then the C+V copy/constant expert
 * counts | sum_t p (N+1+C+V: reals, the null logit, copy/constant experts) |
 * sum_t lse^2 | T]. */
MOE_API size_t moe_aux_sums_count(const moe_dims_t* dims);

/* Additive aux statistics of this call's tokens (layout above), for a
 * data-parallel all-reduce across ranks. After moe_route. sums: device. */
MOE_API int moe_aux_sums(const moe_dims_t* dims, const void* workspace, double* sums,
                 moe_stream_t stream);

/* moe_aux_sums added into `sums` (+=) instead of written over it: the statistics of
 * a batch processed in several calls (token chunks), summed on the device. */
MOE_API int moe_aux_sums_accumulate(const moe_dims_t* dims, const void* workspace, double* sums,
                                    moe_stream_t stream);

/* L_bal / L_z from (possibly all-reduced) sums (section 三 / 负载均衡损失,
 * Z-Loss): counts_ext [N+M+C+V] (null copy j counts the tokens with more than j
 * null slots), P [N+M+C+V] (null copies share the null probability), losses [2]
 * = {L_bal = N * sum_i f_i P_i with f_i = counts_ext_i / T_total, L_z}. */
MOE_API int moe_aux_finalize(const moe_dims_t* dims, const double* sums, int32_t* counts_ext,
                     float* P, float* losses, moe_stream_t stream);

/* moe_aux_sums + moe_aux_finalize on this call's tokens alone. */
MOE_API int moe_aux(const moe_dims_t* dims, const void* workspace, int32_t* counts_ext, float* P,
            float* losses, moe_stream_t stream);

/* The whole forward: route, dispatch (+aux), expert FFNs, combine. With
 * out->shared_out == NULL the combine runs inside the down GEMM
 * (moe_expert_down_combine) and the forward is six launches. With
 * out->xs == NULL the routed rows are never copied: dispatch writes only the
 * permutation and gate/up gathers rows of x (moe_expert_gate_up_gather). With
 * out->z and out->z_shared set (training; xs required) the gate/up GEMM also
 * writes the pre-activations for moe_backward. z and z_shared must both be set or
 * both NULL, else MOE_ERR_INVALID_ARG before anything is enqueued. */
MOE_API int moe_forward(const moe_dims_t* dims, const moe_weights_t* w, const uint16_t* x,
                const float* tok_null_bias, const moe_outputs_t* out, void* workspace,
                moe_stream_t stream);

/* Synchronises `stream`, then returns MOE_OK or the first device-side error
 * recorded in the workspace status word (MOE_ERR_TIMEOUT, ...). */
MOE_API int moe_get_device_status(const void* workspace, moe_stream_t stream);

/* Clears the workspace status word (enqueued on `stream`). */
MOE_API int moe_clear_device_status(void* workspace, moe_stream_t stream);

/* Test aid for the failure path: one CTA waits, with the same bounded wait
 * the GEMM uses, on a shared-memory barrier that nothing arrives at, gives up
 * after `limit_ns` nanoseconds (1e3..1e10), records MOE_ERR_TIMEOUT in the
 * workspace status word and returns. The context stays usable. */
MOE_API int moe_selftest_bounded_wait(void* workspace, uint64_t limit_ns, moe_stream_t stream);

/* ------------------------------------------------------------------------------------
 * Backward pass.
 *
 * The paper trains the layer end to end with the load-balance and Z losses added at
 * fixed weights (paper-review page, section 四 实验结果 / 训练配置: 2e-2 and 1e-3).
 * The backward differentiates the objective <y, dy> + alpha L_bal + beta L_z, dy the
 * upstream gradient of y. Top-K choices and the load fractions f_i are piecewise
 * constant in the logits and carry no gradient; the logits receive gradient through
 * the renormalised gates, through P_i in L_bal and through lse in L_z. As in the
 * forward, null slots cost nothing: the expert gradients run on the real rows only.
 * Each expert is SwiGLU. Its gate/up pre-activations z either come from the forward
 * (moe_outputs_t.z / z_shared: training mode; then the SwiGLU derivative is an elementwise
 * pass over z and dh) or are recomputed from xs on the tensor cores (fp32 in TMEM), with the
 * SwiGLU derivative taken in that GEMM's epilogue.
 *
 * Requirements: the forward ran with out->logits and out->xs non-NULL (the copy
 * path). Weight gradients of the experts are bf16; router, bias and constant-vector
 * gradients are fp32. Every gradient is written (not accumulated).
 *
 * Backward workspace: moe_backward_workspace_bytes(dims) bytes, 256-byte aligned,
 * separate from the forward workspace; its first word is a status word like the
 * forward workspace's (moe_get_device_status / moe_clear_device_status accept it).
 * moe_backward clears it. */

/* Forward tensors the backward reads (device pointers, all from moe_forward). */
typedef struct moe_saved {
  const uint16_t* x;          /* [T, d] bf16 layer input                              */
  const float* logits;        /* [T, N+1+C+V] fp32 router logits                      */
  const int32_t* topk_idx;    /* [T, K]                                               */
  const float* topk_gate;     /* [T, K]                                               */
  const int32_t* offsets;     /* [N+1]                                                */
  const int32_t* slot_row;    /* [T, K]                                               */
  const uint16_t* xs;         /* [R_cap, d] gathered routed rows                      */
  const uint16_t* h;          /* [R_cap, F] routed SwiGLU activations                 */
  const uint16_t* h_shared;   /* [T, F_shared]                                        */
  const uint16_t* ys;         /* [R_cap, d] routed expert outputs                     */
  const int32_t* counts_ext;  /* [N+M+C+V] slot counts over every data-parallel rank  */
  int64_t t_total;            /* tokens over every data-parallel rank (>= T)          */
  const uint16_t* z;          /* [R_cap, 2F] pre-activations saved by the forward, or
                                 NULL to recompute them on the tensor cores             */
  const uint16_t* z_shared;   /* [T, 2F_shared], or NULL (set both or neither)          */
} moe_saved_t;

/* Gradients (device pointers). */
typedef struct moe_grads {
  uint16_t* dx;               /* [T, d] bf16                                          */
  float* dw_router;           /* [N+1+C+V, d] fp32                                    */
  float* dbias;               /* [N+1+C+V] fp32, or NULL                              */
  float* dtok_null_bias;      /* [T] fp32 gradient of the per-token null offset, or NULL */
  uint16_t* dw_gate;          /* [N, F, d] bf16                                       */
  uint16_t* dw_up;            /* [N, F, d] bf16                                       */
  uint16_t* dw_down;          /* [N, d, F] bf16                                       */
  uint16_t* dws_gate;         /* [F_shared, d] bf16                                   */
  uint16_t* dws_up;           /* [F_shared, d] bf16                                   */
  uint16_t* dws_down;         /* [d, F_shared] bf16                                   */
  float* dconst;              /* [V, d] fp32 (V > 0), else NULL                       */
} moe_grads_t;

/* Backward workspace size in bytes (0 if dims are invalid). */
MOE_API size_t moe_backward_workspace_bytes(const moe_dims_t* dims);

/* Combine backward (核心公式): for each selected slot, dg[t,k] = <dy_t, out> where out
 * is the slot's expert output (its row of ys, x_t for a copy expert, c_j for a
 * constant expert; 0 for a null copy), and for a real slot dys[row] = bf16(g dy_t).
 * dy [T, d] bf16; dys [R_cap, d] bf16 (rows of real slots written); dg [T, K] fp32.
 * topk_idx, x and const_vectors are read only when C + V > 0. */
MOE_API int moe_combine_backward(const moe_dims_t* dims, const uint16_t* dy, const uint16_t* ys,
                                 const float* topk_gate, const int32_t* slot_row, const int32_t* topk_idx,
                                 const uint16_t* x, const uint16_t* const_vectors, uint16_t* dys, float* dg,
                                 void* bwd_workspace, moe_stream_t stream);

/* Router backward (Null Expert 机制, 负载均衡损失, Z-Loss): the logit gradient
 * ds [T, N+1+C+V] fp32 from the gate gradients dg, the forward logits and the global
 * slot counts: gates g = softmax over the selected non-null slots give
 * g_k (dg_k - sum_l g_l dg_l); alpha L_bal gives alpha (N/t_total) p_i (f_i - sum_l f_l p_l)
 * over the pool; beta L_z gives beta (2/t_total) lse_t p_i. The null logit's entry sums
 * its M copies. dtok_null_bias (optional, [T]) receives column N. The call also leaves in
 * the backward workspace ds as two bf16 terms (hi = bf16(ds), lo = bf16(ds - hi)) and
 * per-warp column sums of ds, which moe_router_weight_grad and the router term of
 * moe_expert_dgrad_gate_up read. */
MOE_API int moe_router_backward(const moe_dims_t* dims, const float* logits, const int32_t* topk_idx,
                                const float* topk_gate, const float* dg, const int32_t* counts_ext,
                                int64_t t_total, float alpha, float beta, float* ds, float* dtok_null_bias,
                                void* bwd_workspace, moe_stream_t stream);

/* dw_router = ds^T x ([N+1+C+V, d] fp32) on the tensor cores from the two-term ds that
 * moe_router_backward left in the workspace (x is bf16, so each product is exact; the
 * terms carry ds to 2^-16 relative), and dbias = sum_t ds (optional). Both are summed in
 * a fixed order (deterministic). */
MOE_API int moe_router_weight_grad(const moe_dims_t* dims, const uint16_t* x, float* dw_router, float* dbias,
                                   void* bwd_workspace, moe_stream_t stream);

/* Expert FFN backward (实现: grouped GEMMs over the real rows only): dgrad of the down
 * projection, the gate/up pre-activations recomputed with the SwiGLU derivative in the
 * same GEMM's epilogue, the down weight gradient, dgrad of gate/up and the gate/up weight
 * gradient, for the routed experts (rows of xs, upstream dys) and the shared expert
 * (rows of x, upstream dy). Writes dxs [R_cap, d] and dx_shared [T, d] (bf16) and
 * g->dw_gate/up/down and g->dws_gate/up/down. When w->w_router is set, dx_shared also
 * receives the router's input gradient ds W_r (two-term products hi*hi + hi*lo + lo*hi
 * on the tensor cores, as extra k-blocks of the shared expert's tiles), from the ds that
 * moe_router_backward left in the workspace. */
MOE_API int moe_expert_ffn_backward(const moe_dims_t* dims, const moe_weights_t* w, const moe_saved_t* saved,
                                    const uint16_t* dys, const uint16_t* dy, uint16_t* dxs, uint16_t* dx_shared,
                                    const moe_grads_t* g, void* bwd_workspace, moe_stream_t stream);

/* The five stages of moe_expert_ffn_backward, one GEMM launch each, for callers that
 * schedule or time them separately. dh and dz live in the backward workspace; call the
 * stages in this order:
 *   moe_expert_dgrad_down      dh = dys W_d (routed), dh_shared = dy W_sd
 *   moe_expert_swiglu_backward z = [xs W_g^T | xs W_u^T] recomputed in fp32 on the tensor
 *                              cores; its epilogue writes dz = [da | db] (packed order) with
 *                              da = dh b sigma(a) (1 + a (1 - sigma(a))), db = dh a sigma(a)
 *   moe_expert_wgrad_down      dw_down[e] = dys_e^T h_e, dws_down = dy^T h_shared
 *   moe_expert_dgrad_gate_up dxs = dz W_gu, dx_shared = dz_shared W_sgu (+ ds W_r when
 *                            w_router is not NULL)
 *   moe_expert_wgrad_gate_up dw_gate/dw_up[e] = dz_e^T xs_e (unpacked), shared from x */
MOE_API int moe_expert_dgrad_down(const moe_dims_t* dims, const int32_t* offsets, const uint16_t* dys,
                                  const uint16_t* dy, const uint16_t* w_down, const uint16_t* shared_down,
                                  void* bwd_workspace, moe_stream_t stream);
MOE_API int moe_expert_swiglu_backward(const moe_dims_t* dims, const uint16_t* xs, const uint16_t* x,
                                       const int32_t* offsets, const uint16_t* gate_up,
                                       const uint16_t* shared_gate_up, void* bwd_workspace, moe_stream_t stream);
/* Training-mode alternative to moe_expert_swiglu_backward: dz from the pre-activations the
 * forward saved (z [R_cap, 2F], z_shared [T, 2F_shared]) and the dh in the workspace. */
MOE_API int moe_expert_swiglu_backward_saved(const moe_dims_t* dims, const int32_t* offsets, const uint16_t* z,
                                             const uint16_t* z_shared, void* bwd_workspace, moe_stream_t stream);
MOE_API int moe_expert_wgrad_down(const moe_dims_t* dims, const int32_t* offsets, const uint16_t* dys,
                                  const uint16_t* dy, const uint16_t* h, const uint16_t* h_shared,
                                  uint16_t* dw_down, uint16_t* dws_down, void* bwd_workspace,
                                  moe_stream_t stream);
MOE_API int moe_expert_dgrad_gate_up(const moe_dims_t* dims, const int32_t* offsets, const uint16_t* gate_up,
                                     const uint16_t* shared_gate_up, const float* w_router, uint16_t* dxs,
                                     uint16_t* dx_shared, void* bwd_workspace, moe_stream_t stream);
MOE_API int moe_expert_wgrad_gate_up(const moe_dims_t* dims, const int32_t* offsets, const uint16_t* xs,
                                     const uint16_t* x, uint16_t* dw_gate, uint16_t* dw_up, uint16_t* dws_gate,
                                     uint16_t* dws_up, void* bwd_workspace, moe_stream_t stream);

/* Input gradient: dx[t] = dx_shared[t] (the shared expert's and the router's input
 * gradient) + sum over the token's real slots of dxs[slot_row] + sum over its copy-expert
 * slots of g dy[t], accumulated in fp32 in rank order and rounded once to bf16. dx_shared
 * may be dx itself (in place, as moe_backward runs it): a token with no real or copy-expert
 * slot is then left as it is, which is the same value bit for bit. */
MOE_API int moe_input_grad(const moe_dims_t* dims, const uint16_t* dx_shared, const uint16_t* dxs,
                           const int32_t* slot_row, const int32_t* topk_idx, const float* topk_gate,
                           const uint16_t* dy, uint16_t* dx, void* bwd_workspace, moe_stream_t stream);

/* The whole backward: combine, router, router weight gradient, expert FFNs, input
 * gradient and (V > 0) the constant experts' gradient. */
MOE_API int moe_backward(const moe_dims_t* dims, const moe_weights_t* w, const moe_saved_t* saved,
                         const uint16_t* dy, float alpha, float beta, const moe_grads_t* g, void* bwd_workspace,
                         moe_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* MOE_NULL_H */
