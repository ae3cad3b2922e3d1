// Internal declarations shared by the CUDA translation units of libmoe_null.
// Device helpers are thin inline-PTX wrappers for sm_100a: mbarriers, TMA
// tensor loads, tcgen05 (TMEM allocation, MMA, commit, loads) and fences.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "../../include/moe_null.h"

namespace moe {

// ------------------------------------------------------------------------------------
// Tiling constants of the route kernel (router product on tcgen05 + routing).
constexpr int kRouteTokens = 128;                          // tokens per route CTA (one M=128 tile)
constexpr int kRouteBK = 64;                               // d-columns per pipeline stage
constexpr int kRouteEpiThreads = 512;                      // 16 epilogue warps: 4 lanes per token
constexpr int kRouteThreads = 64 + kRouteEpiThreads;       // + TMA warp + MMA warp
constexpr int kFp32RouteTokens = 64;                       // tokens per CTA of the fp32 CUDA-core route
constexpr int kMaxN = 64;
constexpr int kMaxK = 16;
constexpr int kMaxPP = 16;     // MoE++ copy + constant experts
constexpr int kMaxRows = 80;   // router rows N + 1 + C + V (one tensor-core tile of three terms)

// Status bits recorded on the device (the host maps them to moe_status_t).
constexpr uint32_t kStatusTimeout = 1u;
constexpr uint32_t kStatusBounds = 2u;

// Byte offset of the per-expert row totals inside the workspace header.
constexpr size_t kHdrTotOffset = 16;
// Byte offset of the count of tokens with a source (int32): the route appends each token
// that takes a real expert or a copy or constant expert to the workspace's token list.
constexpr size_t kHdrSrcOffset = 384;
// Byte offset of the two counters of the down GEMM with the combine folded in: routed
// tiles whose ys rows are stored, and CTAs that have exited (the last one resets both).
constexpr size_t kHdrCombineOffset = 448;
// Bytes of the header that every route call clears: status word, per-expert totals, the
// count of tokens with a source and the down GEMM's counters.
constexpr size_t kHdrClearBytes = kHdrCombineOffset + 8;
static_assert(kHdrTotOffset + sizeof(int32_t) * kMaxN <= kHdrSrcOffset &&
                  kHdrSrcOffset + sizeof(int32_t) <= kHdrCombineOffset,
              "workspace header fields overlap");

// Default limit of every device-side wait, in ns of %globaltimer.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

// Workspace layout, computed identically on the host for every entry point.
struct WsLayout {
  int blk_tokens;    // tokens per route block (route_block_tokens)
  int nblk;          // route CTAs = ceil(T / blk_tokens)
  size_t hdr;        // uint32 status at 0; int32 per-expert totals at kHdrTotOffset; the count
                     // of tokens with a source at kHdrSrcOffset; the down GEMM's counters at
                     // kHdrCombineOffset (512 B)
  size_t counts_blk; // int32 [N][nblk]
  size_t bases;      // int32 [N][nblk]
  size_t ppart;      // float [nblk][N+1+C+V]
  size_t lsq;        // float [nblk]
  size_t hist;       // int32 [nblk][K+1+C+V]: null histogram, then copy/constant expert counts
  size_t lrank;      // int32 [T][K]
  size_t srctok;     // int32 [T]: the tokens with a source, in the order the route blocks
                     // appended them (the first header count entries are valid)
  size_t counts;     // int32 [N]
  size_t offsets;    // int32 [N+1]
  size_t sums;       // double [aux sums count]
  int nparts;        // first-level aux partials = min(kAuxParts, nblk)
  size_t auxp;       // double [nparts][aux_part_cols]
  size_t wprep;      // router weight prepared for this call: bf16 [3 * route_npw][d] (three
                     // terms hi, mid, lo) or, for the fp32 CUDA-core route, W_r^T fp32 [d][npad + 4]
  size_t total;
};

constexpr size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// First-level aux partials: each of up to kAuxParts CTAs reduces a fixed,
// contiguous slice of route blocks in fp64: [sum p (N+1) | null hist (K+1) | sum lse^2].
constexpr int kAuxParts = 64;
// MoE++ copy + constant experts, and the column counts that follow from them: router
// rows / logits (N real, the null logit, C + V), per-block probability sums (one per
// router row) and per-block slot counts (null histogram K+1, then one per C/V expert).
inline int pp_experts(const moe_dims_t& d) { return d.C + d.V; }
inline int router_rows(const moe_dims_t& d) { return d.N + 1 + pp_experts(d); }
inline int hist_cols(const moe_dims_t& d) { return d.K + 1 + pp_experts(d); }
inline int aux_part_cols(const moe_dims_t& d) { return router_rows(d) + hist_cols(d) + 1; }

// Rows per bf16 term of the split router weight: the router rows padded to a
// multiple of 16 (16 .. 80), so the three terms together are one MMA of N <= 240.
inline int route_npw(const moe_dims_t& d) { return (router_rows(d) + 15) / 16 * 16; }

// Real-logit count the fp32 CUDA-core route pads N to (8, 16, 32 or 64).
inline int route_fp32_npad(int N) { return N <= 8 ? 8 : N <= 16 ? 16 : N <= 32 ? 32 : 64; }

inline bool route_fp32_cores(const moe_dims_t& d) { return (d.flags & MOE_FLAG_ROUTER_FP32_CORES) != 0u; }

// Tokens per route block: the unit of the per-block statistics and ranks.
inline int route_block_tokens(const moe_dims_t& d) {
  return route_fp32_cores(d) ? kFp32RouteTokens : kRouteTokens;
}

// [counts_real (N) | slot counts (hist_cols) | probability sums (router_rows) | lse^2 | T]
inline size_t aux_sums_count(const moe_dims_t& d) {
  return (size_t)d.N + (size_t)hist_cols(d) + (size_t)router_rows(d) + 2;
}

inline WsLayout ws_layout(const moe_dims_t& d) {
  WsLayout L{};
  L.blk_tokens = route_block_tokens(d);
  L.nblk = (d.T + L.blk_tokens - 1) / L.blk_tokens;
  size_t o = 0;
  L.hdr = o; o += 512;
  L.counts_blk = o; o = align_up(o + sizeof(int32_t) * (size_t)d.N * L.nblk, 256);
  L.bases = o; o = align_up(o + sizeof(int32_t) * (size_t)d.N * L.nblk, 256);
  L.ppart = o; o = align_up(o + sizeof(float) * (size_t)router_rows(d) * L.nblk, 256);
  L.lsq = o; o = align_up(o + sizeof(float) * (size_t)L.nblk, 256);
  L.hist = o; o = align_up(o + sizeof(int32_t) * (size_t)hist_cols(d) * L.nblk, 256);
  L.lrank = o; o = align_up(o + sizeof(int32_t) * (size_t)d.T * d.K, 256);
  L.srctok = o; o = align_up(o + sizeof(int32_t) * (size_t)d.T, 256);
  L.counts = o; o = align_up(o + sizeof(int32_t) * (size_t)d.N, 256);
  L.offsets = o; o = align_up(o + sizeof(int32_t) * (size_t)(d.N + 1), 256);
  L.sums = o; o = align_up(o + sizeof(double) * aux_sums_count(d), 256);
  L.nparts = L.nblk < kAuxParts ? L.nblk : kAuxParts;
  L.auxp = o; o = align_up(o + sizeof(double) * (size_t)L.nparts * aux_part_cols(d), 256);
  L.wprep = o;
  o = align_up(o + (route_fp32_cores(d) ? sizeof(float) * (size_t)d.d * (route_fp32_npad(d.N) + 4)
                                        : sizeof(uint16_t) * 3 * (size_t)route_npw(d) * d.d),
               256);
  L.total = o;
  return L;
}

// Backward-pass workspace (moe_backward_workspace_bytes). R_cap = T*K rows.
int bwd_shared_split(const moe_dims_t& d, int* chunk_kb);
size_t bwd_split_partial_floats(const moe_dims_t& d);
int router_wgrad_split(const moe_dims_t& d, int* chunk_kb);
int router_bwd_grid(const moe_dims_t& d);
// Router rows padded to a multiple of 64: the width of each bf16 term of the split logit
// gradients and router weights that the backward's tensor-core products read.
inline int router_split_rows(const moe_dims_t& d) { return (router_rows(d) + 63) / 64 * 64; }

struct BwdLayout {
  size_t hdr;    // uint32 status at 0 (256 B)
  size_t dh;     // bf16 [R_cap, F] gradient of the routed SwiGLU activations
  size_t dhs;    // bf16 [T, F_shared] the shared expert's
  size_t dz;     // bf16 [R_cap, 2F] gradients of the gate/up pre-activations (packed order)
  size_t dzs;    // bf16 [T, 2F_shared]
  size_t dys;    // bf16 [R_cap, d] upstream gradient of each routed row: g * dy
  size_t dxs;    // bf16 [R_cap, d] input gradient of each routed row (the shared expert's
                 // input gradient goes straight into the caller's dx)
  size_t dg;     // fp32 [T, K] gate gradients
  size_t ds;     // fp32 [T, N+1+C+V] logit gradients
  size_t dsplit; // bf16 [T, 2 RP] logit gradients as two terms (hi | lo), RP = router_split_rows
  size_t w2;     // bf16 [2 RP, d] router weights as two terms (hi rows, then lo rows)
  size_t rpart;  // fp32 [chunks, 2 RP, d] partials of dsplit^T x
  size_t bpart;  // fp32 [router_bwd CTAs, rows] column sums of ds
  size_t spart;  // fp32 shared-expert weight-gradient K-chunk partials
  size_t total;
};

inline BwdLayout bwd_layout(const moe_dims_t& d) {
  BwdLayout L{};
  const size_t rcap = (size_t)d.T * d.K, T = (size_t)d.T;
  const size_t rows = (size_t)router_rows(d);
  const int nch = router_wgrad_split(d, nullptr);
  const size_t rp = (size_t)router_split_rows(d);
  size_t o = 0;
  L.hdr = o; o += 256;
  L.dh = o; o = align_up(o + 2 * rcap * d.F, 256);
  L.dhs = o; o = align_up(o + 2 * T * d.F_shared, 256);
  L.dz = o; o = align_up(o + 2 * rcap * 2 * d.F, 256);
  L.dzs = o; o = align_up(o + 2 * T * 2 * d.F_shared, 256);
  L.dys = o; o = align_up(o + 2 * rcap * d.d, 256);
  L.dxs = o; o = align_up(o + 2 * rcap * d.d, 256);
  L.dg = o; o = align_up(o + 4 * T * d.K, 256);
  L.ds = o; o = align_up(o + 4 * T * rows, 256);
  L.dsplit = o; o = align_up(o + 2 * T * 2 * rp, 256);
  L.w2 = o; o = align_up(o + 2 * 2 * rp * d.d, 256);
  L.rpart = o; o = align_up(o + 4 * (size_t)nch * 2 * rp * d.d, 256);
  L.bpart = o; o = align_up(o + 4 * (size_t)router_bwd_grid(d) * rows, 256);
  L.spart = o; o = align_up(o + 4 * bwd_split_partial_floats(d), 256);
  L.total = o;
  return L;
}

template <typename T>
inline T* ws_ptr(void* ws, size_t off) { return reinterpret_cast<T*>(static_cast<char*>(ws) + off); }
template <typename T>
inline const T* ws_ptr(const void* ws, size_t off) {
  return reinterpret_cast<const T*>(static_cast<const char*>(ws) + off);
}

// Host helpers implemented in api.cu.
int check_dims(const moe_dims_t* d);
int sm_count();
int cuda_status(cudaError_t e);

// Programmatic dependent launch. The layer's kernels are launched with
// programmatic stream serialization (launch_pdl): the GPU may start launching a
// kernel while its predecessor in the stream is still running, which hides the
// launch latency between the layer's kernels. Every kernel first waits in
// pdl_wait() until its predecessor has completed and its writes are visible (a
// no-op when the kernel was launched the ordinary way), and only then lets its
// own successor start launching, so no kernel ever runs ahead of earlier work.
template <typename... KArgs, typename... Args>
inline int launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                      const Args&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cuda_status(cudaLaunchKernelEx(&cfg, kern, args...));
}

// 2-D bf16 tensor map [rows, cols] (cols contiguous) with a box of box_rows x 64
// columns and the 128-byte swizzle (implemented in expert_ffn.cu).
bool make_tmap_bf16(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows);

// Launchers (each returns a moe_status_t after enqueuing).
// w_split: the three-term bf16 router weight prepared by moe_prepare_router, or null to
// split w_router into the workspace for this call (the tensor-core route; the fp32 route
// ignores it).
int launch_route(const moe_dims_t& d, const uint16_t* x, const float* w_router,
                 const float* bias, const float* tok_null_bias, float* logits_out,
                 int32_t* topk_idx, float* topk_gate, int32_t* n_real, void* ws,
                 cudaStream_t st, const uint16_t* w_split = nullptr);
// W_r fp32 [rows, d] -> the three bf16 terms [3 route_npw, d] (hi, mid, lo rows); with ws
// set, the same launch also clears the workspace header; with w3 null it only does that.
int launch_router_split(const moe_dims_t& d, const float* w_router, uint16_t* w3, cudaStream_t st,
                        void* ws = nullptr);
// The fp32 CUDA-core route (route_fp32.cu) and the per-expert scan both routes end with.
int launch_route_fp32(const moe_dims_t& d, const uint16_t* x, const float* w_router,
                      const float* bias, const float* tok_null_bias, float* logits_out,
                      int32_t* topk_idx, float* topk_gate, int32_t* n_real, void* ws,
                      cudaStream_t st);
int launch_route_scan(const moe_dims_t& d, void* ws, cudaStream_t st);
// The expert GEMMs on CTA pairs (expert_ffn_pair.cu), for shapes with 256-wide column tiles.
bool ffn_pair_gate_up_ok(const moe_dims_t& d);
bool ffn_pair_down_ok(const moe_dims_t& d);
int launch_gate_up_pair(const moe_dims_t& d, const uint16_t* xs, const uint16_t* x, const int32_t* offsets,
                        const uint16_t* gate_up, const uint16_t* sgate_up, uint16_t* h, uint16_t* h_shared,
                        void* ws, cudaStream_t st);
int launch_down_pair(const moe_dims_t& d, const int32_t* offsets, const uint16_t* h, const uint16_t* h_shared,
                     const uint16_t* w_down, const uint16_t* sdown, uint16_t* ys, uint16_t* shared_out, void* ws,
                     cudaStream_t st);
int launch_dispatch(const moe_dims_t& d, const uint16_t* x, const int32_t* topk_idx, void* ws,
                    int32_t* counts, int32_t* offsets, int32_t* perm_tok, int32_t* slot_row,
                    uint16_t* xs, int32_t* counts_ext, float* P, float* losses,
                    cudaStream_t st);
int launch_aux(const moe_dims_t& d, const void* ws, double* sums_out, const double* sums_in,
               int32_t* counts_ext, float* P, float* losses, cudaStream_t st,
               bool accumulate = false);
// ws (optional, in place only: shared_out == y): the workspace the route of this forward
// filled; the combine then visits only the tokens it listed as having a source.
int launch_combine(const moe_dims_t& d, const uint16_t* ys, const uint16_t* shared_out,
                   const float* topk_gate, const int32_t* slot_row, const int32_t* topk_idx, const uint16_t* x,
                   const uint16_t* const_vectors, uint16_t* y, cudaStream_t st, void* ws = nullptr);
// perm (optional): token of each routed row; when given, gate/up gathers the
// routed rows of x by TMA instead of reading a gathered copy xs (xs unused).
int launch_gate_up_perm(const moe_dims_t& d, const uint16_t* xs, const uint16_t* x, const int32_t* offsets,
                        const int32_t* perm, const uint16_t* gate_up, const uint16_t* sgate_up, uint16_t* h,
                        uint16_t* h_shared, void* ws, cudaStream_t st);
int launch_expert_ffn(const moe_dims_t& d, const uint16_t* xs, const uint16_t* x,
                      const int32_t* offsets, const uint16_t* gate_up, const uint16_t* w_down,
                      const uint16_t* sgate_up, const uint16_t* sdown, uint16_t* h,
                      uint16_t* h_shared, uint16_t* ys, uint16_t* shared_out, void* ws,
                      cudaStream_t st);
// gate/up that also writes the pre-activations z [T K, 2F] and zs [T, 2F_shared] (bf16, packed
// column order) for the backward pass; copy path (xs) only
int launch_gate_up_save(const moe_dims_t& d, const uint16_t* xs, const uint16_t* x, const int32_t* offsets,
                        const uint16_t* gate_up, const uint16_t* sgate_up, uint16_t* h, uint16_t* h_shared,
                        uint16_t* z, uint16_t* zs, void* ws, cudaStream_t st);
int launch_gate_up(const moe_dims_t& d, const uint16_t* xs, const uint16_t* x, const int32_t* offsets,
                   const uint16_t* gate_up, const uint16_t* sgate_up, uint16_t* h, uint16_t* h_shared,
                   void* ws, cudaStream_t st);
int launch_down(const moe_dims_t& d, const int32_t* offsets, const uint16_t* h, const uint16_t* h_shared,
                const uint16_t* w_down, const uint16_t* sdown, uint16_t* ys, uint16_t* shared_out, void* ws,
                cudaStream_t st);
int launch_gate_up_rows(const moe_dims_t& d, long long rows_cap, const uint16_t* xs, const uint16_t* x,
                        const int32_t* offsets, const uint16_t* gate_up, const uint16_t* sgate_up, uint16_t* h,
                        uint16_t* h_shared, void* ws, cudaStream_t st);
int launch_down_rows(const moe_dims_t& d, long long rows_cap, const int32_t* offsets, const uint16_t* h,
                     const uint16_t* h_shared, const uint16_t* w_down, const uint16_t* sdown, uint16_t* ys,
                     uint16_t* shared_out, void* ws, cudaStream_t st);
int launch_down_combine(const moe_dims_t& d, const int32_t* offsets, const uint16_t* h, const uint16_t* h_shared,
                        const uint16_t* w_down, const uint16_t* sdown, uint16_t* ys, const float* topk_gate,
                        const int32_t* slot_row, const int32_t* topk_idx, const uint16_t* x,
                        const uint16_t* const_vectors, uint16_t* y, void* ws, cudaStream_t st);
int launch_pack_gate_up(const moe_dims_t& d, const uint16_t* w_gate, const uint16_t* w_up,
                        const uint16_t* ws_gate, const uint16_t* ws_up, uint16_t* gate_up,
                        uint16_t* sgate_up, cudaStream_t st);
int launch_selftest_wait(void* ws, unsigned long long limit_ns, cudaStream_t st);

// Backward pass (backward.cu, expert_ffn_bwd.cu, expert_ffn.cu).
int launch_dgrad_down(const moe_dims_t& d, const int32_t* offsets, const uint16_t* dys, const uint16_t* dy,
                      const uint16_t* w_down, const uint16_t* sdown, uint16_t* dh, uint16_t* dh_shared,
                      uint32_t* status, cudaStream_t st);
int launch_swiglu_backward(const moe_dims_t& d, const int32_t* offsets, const uint16_t* xs, const uint16_t* x,
                           const uint16_t* gate_up, const uint16_t* sgate_up, const uint16_t* dh,
                           const uint16_t* dh_shared, uint16_t* dz, uint16_t* dzs, uint32_t* status,
                           cudaStream_t st);
// dsplit/w2 (optional, both or neither): the router's input gradient ds W_r is added to
// dx_shared as extra k-blocks of the shared expert's tiles
int launch_dgrad_gate_up(const moe_dims_t& d, const int32_t* offsets, const uint16_t* dz, const uint16_t* dzs,
                         const uint16_t* gate_up, const uint16_t* sgate_up, const uint16_t* dsplit,
                         const uint16_t* w2, uint16_t* dxs, uint16_t* dx_shared, uint32_t* status, cudaStream_t st);
int launch_wgrad_down(const moe_dims_t& d, const int32_t* offsets, const uint16_t* dys, const uint16_t* dy,
                      const uint16_t* h, const uint16_t* h_shared, uint16_t* dw_down, uint16_t* dws_down,
                      float* partials, uint32_t* status, cudaStream_t st);
int launch_wgrad_gate_up(const moe_dims_t& d, const int32_t* offsets, const uint16_t* dz, const uint16_t* dzs,
                         const uint16_t* xs, const uint16_t* x, uint16_t* dw_gate, uint16_t* dw_up,
                         uint16_t* dws_gate, uint16_t* dws_up, float* partials, uint32_t* status,
                         cudaStream_t st);
int launch_router_wgrad_tc(const moe_dims_t& d, const uint16_t* dsplit, const uint16_t* x, float* part,
                           uint32_t* status, cudaStream_t st);
int launch_router_split2(const moe_dims_t& d, const float* w_router, uint16_t* w2, cudaStream_t st);
int launch_router_wgrad_reduce(const moe_dims_t& d, const float* part, int nchunk, const float* bpart, float* dw,
                               float* dbias, cudaStream_t st);
int launch_combine_bwd(const moe_dims_t& d, const uint16_t* dy, const uint16_t* ys, const float* topk_gate,
                       const int32_t* slot_row, const int32_t* topk_idx, const uint16_t* x,
                       const uint16_t* const_vectors, uint16_t* dys, float* dg, uint32_t* status, cudaStream_t st);
int launch_router_bwd(const moe_dims_t& d, const float* logits, const int32_t* topk_idx, const float* topk_gate,
                      const float* dg, const int32_t* counts_ext, long long t_total, float alpha, float beta,
                      float* ds, float* dtnb, uint16_t* dsplit, float* bpart, cudaStream_t st);
// dx = dx_shared + sum over real slots of dxs rows + sum over copy slots of g dy (combine.cu)
int launch_input_grad(const moe_dims_t& d, const uint16_t* dx_shared, const uint16_t* dxs, const int32_t* slot_row,
                      const int32_t* topk_idx, const float* topk_gate, const uint16_t* dy, uint16_t* dx,
                      uint32_t* status, cudaStream_t st);
int launch_const_grad(const moe_dims_t& d, const int32_t* topk_idx, const float* topk_gate, const uint16_t* dy,
                      float* dconst, cudaStream_t st);
// dz from saved pre-activations and dh (elementwise, every routed row below offsets[N] and
// every shared row)
int launch_swiglu_bwd_saved(const moe_dims_t& d, const int32_t* offsets, const uint16_t* z, const uint16_t* zs,
                            const uint16_t* dh, const uint16_t* dhs, uint16_t* dz, uint16_t* dzs, uint32_t* status,
                            cudaStream_t st);

// ------------------------------------------------------------------------------------
// Device helpers.
#if defined(__CUDACC__)

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Wait for the predecessor kernel in the stream (see launch_pdl), then allow the
// successor to begin launching.
__device__ __forceinline__ void pdl_wait_then_release() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred P;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 P, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, P;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for the phase with parity `parity` of an mbarrier. Returns
// false (and records a timeout in *status) if `limit_ns` passed, or if
// *abort (CTA shared flag, may be null) became non-zero meanwhile.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity,
                                                  unsigned long long limit_ns,
                                                  volatile int* abort, uint32_t* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  uint32_t spins = 0;
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((++spins & 63u) == 0u) {
      if (abort != nullptr && *abort) return false;
      if (globaltimer_ns() - t0 > limit_ns) {
        if (status) atomicOr(status, kStatusTimeout);
        if (abort) *abort = 1;
        return false;
      }
    }
  }
}

// Release / acquire accesses of a counter in global memory (gpu scope).
__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void red_add_release_gpu(uint32_t* p, uint32_t v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Bounded wait until the counter *p reaches `target` (acquire). Returns false (and records
// a timeout in *status) if `limit_ns` passed, or if *abort became non-zero meanwhile.
__device__ __forceinline__ bool counter_wait_bounded(const uint32_t* p, uint32_t target,
                                                     unsigned long long limit_ns, volatile int* abort,
                                                     uint32_t* status) {
  if (ld_acquire_gpu(p) >= target) return true;
  const unsigned long long t0 = globaltimer_ns();
  while (true) {
    __nanosleep(128);
    if (ld_acquire_gpu(p) >= target) return true;
    if (abort != nullptr && *abort) return false;
    if (globaltimer_ns() - t0 > limit_ns) {
      if (status) atomicOr(status, kStatusTimeout);
      if (abort) *abort = 1;
      return false;
    }
  }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* tmap, uint32_t bar, int x,
                                            int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// TMEM allocation: warp-wide. The allocated base address is written to smem.
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, kind::f16 (bf16 inputs, fp32 accumulate).
__device__ __forceinline__ void tc_mma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                           uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on an mbarrier when all prior tcgen05 async ops of this thread finish.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}

// 32 lanes x 32 bit, 16 consecutive columns: thread i gets TMEM lane (base+i).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
// 32 lanes x 32 bit, 8 consecutive columns.
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                 "=r"(r[7])
               : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// bar.red.and over a named barrier: every participating thread gets the AND
// of all their predicates (a CTA-uniform decision among those threads).
__device__ __forceinline__ bool named_bar_and(int id, int nthreads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}

// Shared-memory matrix descriptor (tcgen05) for a K-major tile whose rows are
// 128 bytes (64 bf16) stored with the 128-byte swizzle, 8-row groups 1024 B
// apart: start address, LBO = 16 B (unused for this layout), SBO = 1024 B,
// descriptor version 1, layout type 2 (128-byte swizzle).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)64 << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor: D fp32, A bf16, B bf16, both K-major, shape M x N.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

// 16-byte asynchronous copy global -> shared (L2 only), completion tracked per thread.
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
// Arrive on an mbarrier once all of this thread's earlier cp.async copies have
// landed (the arrival is counted in the barrier's initial count: .noinc).
__device__ __forceinline__ void cp_async_mbar_arrive_noinc(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all_copies() { asm volatile("cp.async.wait_all;" ::: "memory"); }
// Make generic-proxy writes to shared memory (cp.async) visible to the async
// proxy (tcgen05 operand reads) for this thread's subsequent operations.
__device__ __forceinline__ void fence_proxy_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---- thread-block clusters of two CTAs (a CTA pair sharing one tcgen05 MMA)
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_id_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_count_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}
// Address of the same shared-memory object in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Arrive on an mbarrier that may live in the other CTA of the cluster.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// TMA tile load into this CTA's shared memory whose completion is counted on a
// barrier that may live in the other CTA of the pair (the pair's leader).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const void* tmap, uint32_t bar_cluster, int x,
                                                 int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(bar_cluster)
      : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// D[tmem] (+)= A * B^T over the pair: M = 256 (128 rows of A in each CTA), N
// from idesc with N/2 rows of B in each CTA; each CTA's TMEM holds its 128 rows.
__device__ __forceinline__ void tc_mma_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on a barrier (own or peer CTA) when this thread's prior pair MMAs finish.
__device__ __forceinline__ void tc_commit_pair(uint32_t bar_cluster) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar_cluster)
               : "memory");
}

__device__ __forceinline__ float bf16lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

#endif  // __CUDACC__

}  // namespace moe
