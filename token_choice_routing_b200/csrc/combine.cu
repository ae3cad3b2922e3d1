// moe_combine: y[t] = E_shared(x_t) + sum over the token's real slots of
// g_{t,k} * E_e(x_t) (Kilian et al., "Improving MoE Compute Efficiency by
// Composing Weight and Data Sparsity", review page, section 三 / 核心公式).
// Null experts output zero, so null slots (slot_row = -1) are skipped. MoE++
// copy experts add g x_t and constant expert j adds g c_j (MoE++ explainer page,
// 三种零计算专家); they have no ys row either, and are told apart by topk_idx.
// Written as a gather (each token reads its own rows of ys) so it is
// deterministic: fp32 accumulation in rank order, one bf16 rounding.
#include "moe_internal.cuh"

#include <algorithm>

namespace moe {

constexpr int kCombineThreads = 256;

// One warp per token, two 16-byte chunks per lane per pass. A slot's source row is coded
// as: >= 0 a row of ys, -1 nothing (null copy), -2 the token's row of x (copy expert),
// -3 - j constant vector j. The token's slots with a source are compacted (in rank order)
// and taken four at a time: in each pass the shared row's chunks and those slots' chunks
// are loaded together before any is used, so a token with up to four sources costs one
// round of loads per pass whatever K is; the next token's slot list is fetched while this
// one is combined. Sum order: shared, then the sources in rank order; fp32, one rounding.
// UNIT_ROWS (the backward's input gradient): rows of ys enter with weight 1, the gate
// having been applied upstream; copy slots still take g times their row of x.
// INPLACE (sh == y, the shared expert's output written into y by the down GEMM): a token
// without a source already holds its result, bf16(shared), and is skipped.
// THREADS: 256 for the persistent grid (one wave, each warp looping over tokens with the
// next token's slots prefetched), 64 for a grid of one token per warp (small batches).
// LISTED (in place only): the warps visit the route's list of tokens with a source
// (srctok[0 .. *nsrc)) instead of every token, so tokens without one cost no slot lookup
// and every warp gets an equal share of the tokens that have work. Each token's sum is the
// same either way, so y is the same bit for bit.
template <bool UNIT_ROWS, bool INPLACE, int THREADS, bool LISTED = false>
__global__ void __launch_bounds__(THREADS, 768 / THREADS)
combine_kernel(const uint16_t* __restrict__ ys, const uint16_t* sh, const float* __restrict__ gate,
               const int32_t* __restrict__ slot_row, const int32_t* __restrict__ topk_idx,
               const uint16_t* __restrict__ x, const uint16_t* __restrict__ cv, uint16_t* y, int T, int d, int K,
               long long rcap, int NM, int C, int V, uint32_t* status, const int32_t* __restrict__ srctok,
               const int32_t* __restrict__ nsrc) {
  static_assert(!LISTED || INPLACE, "a token list leaves the tokens it omits untouched: in place only");
  pdl_wait_then_release();
  const int lane = threadIdx.x & 31;
  const int wpb = THREADS / 32;
  const int nch = d >> 3;
  const int stride = gridDim.x * wpb;
  // visit i = 0 .. nvis-1: token i, or the i-th listed token
  const int nvis = LISTED ? min(max(__ldg(nsrc), 0), T) : T;
  auto token_at = [&](int i) {
    if (i >= nvis) return T;  // past the end: no slots, skipped
    if (!LISTED) return i;
    const int tt = __ldg(srctok + i);
    if (tt < 0 || tt >= T) {
      if (status) atomicOr(status, kStatusBounds);
      return T;
    }
    return tt;
  };
  int i = blockIdx.x * wpb + (threadIdx.x >> 5);
  int t = token_at(i);
  auto load_slot = [&](int tt, int& row, float& g) {
    row = -1;
    g = 0.f;
    if (tt < T && lane < K) {
      row = __ldg(slot_row + (size_t)tt * K + lane);
      g = __ldg(gate + (size_t)tt * K + lane);
      if (row >= rcap) {
        if (status) atomicOr(status, kStatusBounds);
        row = -1;
      }
      if (row < 0 && C + V > 0) {
        const int id = __ldg(topk_idx + (size_t)tt * K + lane) - NM;  // position among copy/constant
        if (id >= 0 && id < C) row = -2;
        else if (id >= C && id < C + V) row = -3 - (id - C);
      }
    }
  };
  auto fma8 = [](float (&a)[8], float gk, const uint4& v) {
    a[0] = fmaf(gk, bf16lo(v.x), a[0]); a[1] = fmaf(gk, bf16hi(v.x), a[1]);
    a[2] = fmaf(gk, bf16lo(v.y), a[2]); a[3] = fmaf(gk, bf16hi(v.y), a[3]);
    a[4] = fmaf(gk, bf16lo(v.z), a[4]); a[5] = fmaf(gk, bf16hi(v.z), a[5]);
    a[6] = fmaf(gk, bf16lo(v.w), a[6]); a[7] = fmaf(gk, bf16hi(v.w), a[7]);
  };
  int row, rown;
  float g, gn;
  load_slot(t, row, g);
  for (; i < nvis; i += stride) {
    const int tn = token_at(i + stride);
    load_slot(tn, rown, gn);  // next token's slots, in flight during this one
    const unsigned srcs = __ballot_sync(0xffffffffu, row != -1);  // lanes >= K hold -1
    if (INPLACE && srcs == 0u) {
      row = rown;
      g = gn;
      t = tn;
      continue;
    }
    // the shared row's pieces of the next pass are loaded before this pass's stores (in place
    // they are the same buffer, so the compiler would not move them above the stores itself)
    const uint4* shr = reinterpret_cast<const uint4*>(sh + (size_t)t * d);
    uint4 sa_n = (lane < nch) ? shr[lane] : make_uint4(0u, 0u, 0u, 0u);
    uint4 sb_n = (32 + lane < nch) ? shr[32 + lane] : make_uint4(0u, 0u, 0u, 0u);
    for (int c0 = 0; c0 < nch; c0 += 64) {
      const int ca = c0 + lane, cb = c0 + 32 + lane;
      const bool oka = ca < nch, okb = cb < nch;
      const uint4 sa = sa_n, sb = sb_n;
      float acc_a[8], acc_b[8];
      bool first = true;
      unsigned m = srcs;
      do {
        uint4 va[4], vb[4];
        float gq[4];
        int rq[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int k = m ? __ffs(m) - 1 : 0;
          rq[u] = __shfl_sync(0xffffffffu, row, k);
          gq[u] = __shfl_sync(0xffffffffu, g, k);
          if (m == 0u) rq[u] = -1;
          m &= m - 1u;
          if (UNIT_ROWS && rq[u] >= 0) gq[u] = 1.f;
          const uint16_t* srow = (rq[u] >= 0)    ? ys + (size_t)rq[u] * d
                                 : (rq[u] == -2) ? x + (size_t)t * d
                                 : (rq[u] <= -3) ? cv + (size_t)(-3 - rq[u]) * d
                                                 : ys;
          const uint4* src = reinterpret_cast<const uint4*>(srow);
          va[u] = (rq[u] != -1 && oka) ? __ldg(src + ca) : make_uint4(0u, 0u, 0u, 0u);
          vb[u] = (rq[u] != -1 && okb) ? __ldg(src + cb) : make_uint4(0u, 0u, 0u, 0u);
        }
        if (first) {
          acc_a[0] = bf16lo(sa.x); acc_a[1] = bf16hi(sa.x); acc_a[2] = bf16lo(sa.y); acc_a[3] = bf16hi(sa.y);
          acc_a[4] = bf16lo(sa.z); acc_a[5] = bf16hi(sa.z); acc_a[6] = bf16lo(sa.w); acc_a[7] = bf16hi(sa.w);
          acc_b[0] = bf16lo(sb.x); acc_b[1] = bf16hi(sb.x); acc_b[2] = bf16lo(sb.y); acc_b[3] = bf16hi(sb.y);
          acc_b[4] = bf16lo(sb.z); acc_b[5] = bf16hi(sb.z); acc_b[6] = bf16lo(sb.w); acc_b[7] = bf16hi(sb.w);
          first = false;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if (rq[u] != -1) {
            fma8(acc_a, gq[u], va[u]);
            fma8(acc_b, gq[u], vb[u]);
          }
        }
      } while (m != 0u);
      if (c0 + 64 < nch) {
        const int na = c0 + 64 + lane, nb = c0 + 96 + lane;
        sa_n = (na < nch) ? shr[na] : make_uint4(0u, 0u, 0u, 0u);
        sb_n = (nb < nch) ? shr[nb] : make_uint4(0u, 0u, 0u, 0u);
      }
      if (oka)
        reinterpret_cast<uint4*>(y + (size_t)t * d)[ca] =
            make_uint4(pack_bf16x2(acc_a[0], acc_a[1]), pack_bf16x2(acc_a[2], acc_a[3]),
                       pack_bf16x2(acc_a[4], acc_a[5]), pack_bf16x2(acc_a[6], acc_a[7]));
      if (okb)
        reinterpret_cast<uint4*>(y + (size_t)t * d)[cb] =
            make_uint4(pack_bf16x2(acc_b[0], acc_b[1]), pack_bf16x2(acc_b[2], acc_b[3]),
                       pack_bf16x2(acc_b[4], acc_b[5]), pack_bf16x2(acc_b[6], acc_b[7]));
    }
    row = rown;
    g = gn;
    t = tn;
  }
}

// Grid choice. A persistent grid (one wave of 256-thread CTAs, each warp looping over
// tokens and prefetching the next token's slots) hides the slot lookups, but its warps take
// fixed shares of the tokens: with few tokens per warp the share with the most sources sets
// the time. Below kCombineTokensPerWarp tokens per resident warp the grid is one token per
// warp in 64-thread CTAs instead, and the block scheduler balances the load.
// (B200, in place, L2 flushed: T = 16384 at the 1.7B shape with K = 8, 73 -> 53 us; at
// T = 131072 the persistent grid stays ahead, 162 against 169-179 us.)
constexpr int kCombineTokensPerWarp = 16;
constexpr int kCombineSmallThreads = 64;

struct CombineGrid {
  int blocks;
  bool persistent;
};

static CombineGrid combine_grid(const moe_dims_t& d) {
  static int per_sm[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  int occ = (dev >= 0 && dev < 64) ? per_sm[dev] : 0;
  if (occ == 0) {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, combine_kernel<false, false, kCombineThreads>,
                                                      kCombineThreads, 0) != cudaSuccess ||
        occ < 1)
      occ = 1;
    if (dev >= 0 && dev < 64) per_sm[dev] = occ;
  }
  const int wpb = kCombineThreads / 32;
  const long long resident_warps = (long long)sm_count() * occ * wpb;
  if ((long long)d.T < kCombineTokensPerWarp * resident_warps) {
    const int swpb = kCombineSmallThreads / 32;
    return {(int)std::max<long long>(1, ((long long)d.T + swpb - 1) / swpb), false};
  }
  return {(int)std::max<long long>(1, resident_warps / wpb), true};
}

int launch_combine(const moe_dims_t& d, const uint16_t* ys, const uint16_t* shared_out,
                   const float* topk_gate, const int32_t* slot_row, const int32_t* topk_idx, const uint16_t* x,
                   const uint16_t* const_vectors, uint16_t* y, cudaStream_t st, void* ws) {
  const CombineGrid g = combine_grid(d);
  // shared_out == y: the shared expert's output is already in y; tokens without a source keep it
  const bool inplace = shared_out == y;
  const int threads = g.persistent ? kCombineThreads : kCombineSmallThreads;
  const long long rcap = (long long)d.T * d.K;
  if (inplace && ws != nullptr) {  // only the tokens the route listed
    const WsLayout L = ws_layout(d);
    auto kern = g.persistent ? combine_kernel<false, true, kCombineThreads, true>
                             : combine_kernel<false, true, kCombineSmallThreads, true>;
    return launch_pdl(kern, dim3(g.blocks), dim3(threads), 0, st, ys, shared_out, topk_gate, slot_row, topk_idx, x,
                      const_vectors, y, d.T, d.d, d.K, rcap, d.N + d.M, d.C, d.V,
                      ws_ptr<uint32_t>(ws, L.hdr), (const int32_t*)ws_ptr<int32_t>(ws, L.srctok),
                      (const int32_t*)ws_ptr<int32_t>(ws, L.hdr + kHdrSrcOffset));
  }
  auto kern = g.persistent ? (inplace ? combine_kernel<false, true, kCombineThreads>
                                      : combine_kernel<false, false, kCombineThreads>)
                           : (inplace ? combine_kernel<false, true, kCombineSmallThreads>
                                      : combine_kernel<false, false, kCombineSmallThreads>);
  return launch_pdl(kern, dim3(g.blocks), dim3(threads), 0, st, ys, shared_out, topk_gate, slot_row, topk_idx, x,
                    const_vectors, y, d.T, d.d, d.K, rcap, d.N + d.M, d.C, d.V, (uint32_t*)nullptr,
                    (const int32_t*)nullptr, (const int32_t*)nullptr);
}

// Input gradient of the backward pass: dx[t] = dx_shared[t] (the shared expert's and the
// router's input gradient) + sum over the token's real slots of dxs[slot_row] + sum over
// its copy-expert slots of g dy[t]; the same gather as the forward combine. In place
// (dx_shared == dx, as moe_backward runs it) tokens without such slots are skipped.
int launch_input_grad(const moe_dims_t& d, const uint16_t* dx_shared, const uint16_t* dxs, const int32_t* slot_row,
                      const int32_t* topk_idx, const float* topk_gate, const uint16_t* dy, uint16_t* dx,
                      uint32_t* status, cudaStream_t st) {
  const CombineGrid g = combine_grid(d);
  // dx_shared == dx (in place): a token with no routed or copy slot already holds its result
  const bool inplace = dx_shared == dx;
  auto kern = g.persistent ? (inplace ? combine_kernel<true, true, kCombineThreads>
                                      : combine_kernel<true, false, kCombineThreads>)
                           : (inplace ? combine_kernel<true, true, kCombineSmallThreads>
                                      : combine_kernel<true, false, kCombineSmallThreads>);
  const int threads = g.persistent ? kCombineThreads : kCombineSmallThreads;
  return launch_pdl(kern, dim3(g.blocks), dim3(threads), 0, st, dxs, dx_shared, topk_gate, slot_row, topk_idx, dy,
                    (const uint16_t*)nullptr, dx, d.T, d.d, d.K, (long long)d.T * d.K, d.N + d.M, d.C, 0, status,
                    (const int32_t*)nullptr, (const int32_t*)nullptr);
}

}  // namespace moe
