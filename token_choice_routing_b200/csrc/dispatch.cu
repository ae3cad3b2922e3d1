// moe_dispatch: the expert-contiguous permutation of the real (token, expert)
// slots, with the row gather of x into xs; and the aux-loss reductions.
//
// Kilian et al., "Improving MoE Compute Efficiency by Composing Weight and Data
// Sparsity" (review page, section 三 / 实现): null indices (>= N) are moved to
// the end of the sorted (token, expert) list and cut off before the grouped
// matmul. Here no sort is run: the route kernel already produced, per block of
// 64 tokens, each slot's rank among the block's tokens that chose the same
// expert, and the per-(expert, block) base row. A slot's row is base + rank,
// which is the stable (expert, token) order. Null slots are skipped before any
// load, so they cost no memory traffic.
//
// Aux (same page, 负载均衡损失 and Z-Loss): L_bal = N * sum_i f_i P_i over the pool
// (reals, null copies, and MoE++ copy/constant experts when present) with f_i =
// count_i / T and P_i = mean_t p_{t,i}; L_z = mean_t lse_t^2. Per-block fp32
// partials from the route kernel are summed in fp64, first over fixed slices of
// blocks (in the scan launch), then over the slices here.
#include "moe_internal.cuh"

namespace moe {

struct AuxPtrs {
  const int32_t* counts;  // [N] real counts (route scan)
  const double* auxp;     // [nparts][(N+1+C+V) + (K+1+C+V) + 1] fp64 partials (scan launch)
  int nparts, N, M, K, T, C, V;
};

// Most doubles the sums of one layer can take (see aux_sums_count).
constexpr int kMaxSums = kMaxN + (kMaxK + 1 + kMaxPP) + kMaxRows + 2;

// sums layout: [counts_real N | hist K+1+C+V (null slots per token, then per copy /
// constant expert) | psum N+1+C+V (per router row) | lsq | T]. The first-level partials
// (at most kAuxParts = 64 of them) are combined one column per warp: lane l adds
// partials l and l+32, then a fixed shuffle tree (deterministic).
__device__ void aux_sums_block(const AuxPtrs& p, double* sums) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
  const int N = p.N, K = p.K, PP = p.C + p.V;
  double* s_cnt = sums;
  double* s_hist = sums + N;
  double* s_psum = s_hist + (K + 1 + PP);
  double* s_lsq = s_psum + (N + 1 + PP);
  const int c1 = N + 1 + PP, c2 = c1 + K + 1 + PP, cols = c2 + 1;
  for (int e = tid; e < N; e += blockDim.x) s_cnt[e] = (double)p.counts[e];
  for (int c = warp; c < cols; c += nwarps) {
    double acc = 0.0;
    if (lane < p.nparts) acc = p.auxp[(size_t)lane * cols + c];
    if (lane + 32 < p.nparts) acc += p.auxp[(size_t)(lane + 32) * cols + c];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) {
      if (c < c1) s_psum[c] = acc;
      else if (c < c2) s_hist[c - c1] = acc;
      else s_lsq[0] = acc;
    }
  }
  if (tid == 0) s_lsq[1] = (double)p.T;
  __syncthreads();
}

__device__ void aux_finalize_block(const double* sums, int N, int M, int K, int PP, int32_t* counts_ext,
                                   float* P, float* losses) {
  const int tid = threadIdx.x;
  const double* s_cnt = sums;
  const double* s_hist = sums + N;
  const double* s_psum = s_hist + (K + 1 + PP);
  const double lsq = s_psum[N + 1 + PP];
  const double Tt = s_psum[N + 1 + PP + 1];
  const double inv = Tt > 0.0 ? 1.0 / Tt : 0.0;
  for (int i = tid; i < N + M + PP; i += blockDim.x) {
    if (i < N) {
      if (counts_ext) counts_ext[i] = (int32_t)s_cnt[i];
      if (P) P[i] = (float)(s_psum[i] * inv);
    } else if (i < N + M) {
      const int j = i - N;  // null copy j is taken by tokens with more than j null slots
      double c = 0.0;
      for (int q = j + 1; q <= K; ++q) c += s_hist[q];
      if (counts_ext) counts_ext[i] = (int32_t)c;
      if (P) P[i] = (float)(s_psum[N] * inv);
    } else {
      const int j = i - N - M;  // copy or constant expert j: its own count and probability
      if (counts_ext) counts_ext[i] = (int32_t)s_hist[K + 1 + j];
      if (P) P[i] = (float)(s_psum[N + 1 + j] * inv);
    }
  }
  if (tid == 0 && losses) {
    double acc = 0.0;
    for (int i = 0; i < N; ++i) acc += s_cnt[i] * s_psum[i];
    double nulls = 0.0;
    for (int q = 1; q <= K; ++q) nulls += (double)q * s_hist[q];
    acc += nulls * s_psum[N];
    for (int j = 0; j < PP; ++j) acc += s_hist[K + 1 + j] * s_psum[N + 1 + j];
    losses[0] = (float)((double)N * acc * inv * inv);
    losses[1] = (float)(lsq * inv);
  }
}

__global__ void __launch_bounds__(256) aux_kernel(AuxPtrs p, double* sums_out, const double* sums_in,
                                                  int32_t* counts_ext, float* P, float* losses, int accumulate) {
  pdl_wait_then_release();
  __shared__ double s_sums[kMaxSums];
  const int n = p.N + (p.K + 1 + p.C + p.V) + (p.N + 1 + p.C + p.V) + 2;
  if (sums_in == nullptr) {
    aux_sums_block(p, s_sums);
    if (sums_out)
      for (int i = threadIdx.x; i < n; i += blockDim.x) sums_out[i] = accumulate ? sums_out[i] + s_sums[i] : s_sums[i];
  } else {
    for (int i = threadIdx.x; i < n; i += blockDim.x) s_sums[i] = sums_in[i];
    __syncthreads();
  }
  if (counts_ext || P || losses) aux_finalize_block(s_sums, p.N, p.M, p.K, p.C + p.V, counts_ext, P, losses);
}

struct DispatchArgs {
  const uint16_t* x;
  const int32_t* topk_idx;
  const int32_t* lrank;
  const int32_t* bases;  // [N][nblk]
  const int32_t* ws_counts;
  const int32_t* ws_offsets;
  int32_t* counts;
  int32_t* offsets;
  int32_t* perm_tok;
  int32_t* slot_row;
  uint16_t* xs;
  uint32_t* status;
  // fused aux (block 0) outputs, or all null
  AuxPtrs aux;
  double* sums;
  int32_t* counts_ext;
  float* P;
  float* losses;
  int fuse_aux;
  int T, d, N, M, K, nblk, blk_tokens;
};

constexpr int kDispatchThreads = 256;

__global__ void __launch_bounds__(kDispatchThreads) dispatch_kernel(DispatchArgs a) {
  pdl_wait_then_release();
  int blk = blockIdx.x;
  if (a.fuse_aux) {
    if (blk == 0) {  // scheduled first, so the reduction overlaps the gather
      __shared__ double s_sums[kMaxSums];
      aux_sums_block(a.aux, s_sums);
      if (a.sums)
        for (int i = threadIdx.x; i < a.N + 2 * (a.aux.C + a.aux.V) + a.K + 1 + a.N + 1 + 2; i += blockDim.x)
          a.sums[i] = s_sums[i];
      aux_finalize_block(s_sums, a.N, a.M, a.K, a.aux.C + a.aux.V, a.counts_ext, a.P, a.losses);
      return;
    }
    --blk;
  }
  const int nblocks = gridDim.x - (a.fuse_aux ? 1 : 0);
  const int tid = threadIdx.x, lane = tid & 31;
  if (blk == 0) {
    for (int i = tid; i <= a.N; i += blockDim.x) {
      a.offsets[i] = a.ws_offsets[i];
      if (i < a.N) a.counts[i] = a.ws_counts[i];
    }
  }
  const int K = a.K, N = a.N, d = a.d;
  const long long rcap = (long long)a.T * K;
  const int nch = d >> 3;  // 16-byte chunks per row
  const int wpb = kDispatchThreads / 32;
  const int stride = nblocks * wpb;
  // lane k < K: the destination row of the token's slot k (-1: null or out of range)
  auto slot_dest = [&](int t) {
    int dest = -1;
    if (t < a.T && lane < K) {
      const int id = __ldg(a.topk_idx + (size_t)t * K + lane);
      if (id >= 0 && id < N) {
        dest = __ldg(a.bases + (size_t)id * a.nblk + t / a.blk_tokens) + __ldg(a.lrank + (size_t)t * K + lane);
        if (dest < 0 || dest >= rcap) {
          atomicOr(a.status, kStatusBounds);
          dest = -1;
        }
      } else if (id < 0 || id >= N + a.M + a.aux.C + a.aux.V) {
        atomicOr(a.status, kStatusBounds);
      }
    }
    return dest;
  };
  int t = blk * wpb + (tid >> 5);
  int dest = slot_dest(t);
  for (; t < a.T; t += stride) {
    const int dest_next = slot_dest(t + stride);  // the next token's rows, looked up meanwhile
    if (lane < K) {
      a.slot_row[(size_t)t * K + lane] = dest;
      if (dest >= 0) a.perm_tok[dest] = t;
    }
    const unsigned real = __ballot_sync(0xffffffffu, dest >= 0);
    if (a.xs != nullptr && real != 0u) {
      // the whole row is loaded (8 x 16 B per lane for d <= 2048) before any copy is stored
      const uint4* src = reinterpret_cast<const uint4*>(a.x + (size_t)t * d);
      for (int c0 = 0; c0 < nch; c0 += 256) {  // warp-uniform trip count
        uint4 v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int c = c0 + j * 32 + lane;
          v[j] = (c < nch) ? __ldg(src + c) : make_uint4(0u, 0u, 0u, 0u);
        }
        for (unsigned m = real; m != 0u; m &= m - 1u) {
          const int k = __ffs(m) - 1;
          const int dk = __shfl_sync(0xffffffffu, dest, k);
          uint4* dst = reinterpret_cast<uint4*>(a.xs + (size_t)dk * d);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int c = c0 + j * 32 + lane;
            if (c < nch) dst[c] = v[j];
          }
        }
      }
    }
    dest = dest_next;
  }
}

static AuxPtrs aux_ptrs(const moe_dims_t& d, const void* ws) {
  const WsLayout L = ws_layout(d);
  AuxPtrs p{};
  p.counts = ws_ptr<int32_t>(ws, L.counts);
  p.auxp = ws_ptr<double>(ws, L.auxp);
  p.nparts = L.nparts;
  p.N = d.N;
  p.M = d.M;
  p.K = d.K;
  p.T = d.T;
  p.C = d.C;
  p.V = d.V;
  return p;
}

int launch_dispatch(const moe_dims_t& d, const uint16_t* x, const int32_t* topk_idx, void* ws,
                    int32_t* counts, int32_t* offsets, int32_t* perm_tok, int32_t* slot_row,
                    uint16_t* xs, int32_t* counts_ext, float* P, float* losses, cudaStream_t st) {
  const WsLayout L = ws_layout(d);
  DispatchArgs a{};
  a.x = x;
  a.topk_idx = topk_idx;
  a.lrank = ws_ptr<int32_t>(ws, L.lrank);
  a.bases = ws_ptr<int32_t>(ws, L.bases);
  a.ws_counts = ws_ptr<int32_t>(ws, L.counts);
  a.ws_offsets = ws_ptr<int32_t>(ws, L.offsets);
  a.counts = counts;
  a.offsets = offsets;
  a.perm_tok = perm_tok;
  a.slot_row = slot_row;
  a.xs = xs;
  a.status = ws_ptr<uint32_t>(ws, L.hdr);
  a.aux = aux_ptrs(d, ws);
  a.sums = ws_ptr<double>(ws, L.sums);
  a.counts_ext = counts_ext;
  a.P = P;
  a.losses = losses;
  a.fuse_aux = 1;
  a.T = d.T;
  a.d = d.d;
  a.N = d.N;
  a.M = d.M;
  a.K = d.K;
  a.nblk = L.nblk;
  a.blk_tokens = L.blk_tokens;
  const int wpb = kDispatchThreads / 32;
  int grid = (d.T + wpb - 1) / wpb;
  const int cap = sm_count() * 8;
  if (grid > cap) grid = cap;
  return launch_pdl(dispatch_kernel, dim3(grid + 1), dim3(kDispatchThreads), 0, st, a);
}

int launch_aux(const moe_dims_t& d, const void* ws, double* sums_out, const double* sums_in,
               int32_t* counts_ext, float* P, float* losses, cudaStream_t st, bool accumulate) {
  return launch_pdl(aux_kernel, dim3(1), dim3(256), 0, st, aux_ptrs(d, ws), sums_out, sums_in, counts_ext, P,
                    losses, accumulate ? 1 : 0);
}

// ---------------------------------------------------------------------------------------
// Test aid: a bounded wait on a barrier that nothing arrives at.
__global__ void selftest_wait_kernel(uint32_t* status, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    (void)mbar_wait_bounded(smem_u32(&bar), 0, limit_ns, &abort_flag, status);
  }
  __syncthreads();
}

int launch_selftest_wait(void* ws, unsigned long long limit_ns, cudaStream_t st) {
  selftest_wait_kernel<<<1, 32, 0, st>>>(reinterpret_cast<uint32_t*>(ws), limit_ns);
  return cuda_status(cudaGetLastError());
}

}  // namespace moe
