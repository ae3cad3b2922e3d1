// moe_route: router GEMM (fp32, CUDA cores) fused with the expanded-pool
// softmax statistics, top-K over the pool, renormalised gates and the
// per-block statistics that dispatch and the aux losses need.
//
// Method (Kilian et al., "Improving MoE Compute Efficiency by Composing Weight
// and Data Sparsity", review page, section 三 技术架构):
//  * Null Expert 机制: N real logits plus one null logit; the null logit is
//    replicated M times before top-K, so the pool is [s_0..s_{N-1}, s_N x M].
//    The pool is never materialised here: a copy is a (value, multiplicity).
//  * 阈值解释: the token keeps the real experts whose logit beats the null
//    logit; so top-K over the pool is K rounds of "best remaining real vs the
//    null logit", the real winning ties (lower index), copies taken in index
//    order N, N+1, ... while any remain.
//  * renormalisation over the selected reals: gates = softmax over their
//    logits; null slots weigh 0.
//  * Z-Loss / 负载均衡损失: lse_t over the N+M pool and p_{t,i} are reduced per
//    block here (fp32 over 32 tokens) and across blocks in fp64 later.
//
// Layout: one CTA = 32 tokens x all N+1 logits (see route_kernel). x (bf16) is
// widened to fp32 once when staged in shared memory; W_r slices arrive by
// cp.async, double-buffered.
#include "moe_internal.cuh"

#include <climits>

namespace moe {

struct RouteArgs {
  const uint16_t* x;
  const float* w;     // [N+1, d]
  const float* bias;  // [N+1] or null
  const float* tnb;   // [T] or null
  float* logits;      // [T, N+1] or null
  int32_t* topk_idx;
  float* topk_gate;
  int32_t* n_real;
  // workspace
  uint32_t* hdr;  // [0] status
  int32_t* tot;   // [N] rows per expert (integer atomics)
  int32_t* counts_blk;
  int32_t* bases;
  float* ppart;
  float* lsq;
  int32_t* hist;
  int32_t* lrank;
  int32_t* counts;
  int32_t* offsets;
  int T, d, N, M, K, nblk;
};

constexpr int kXS = kRouteBK + 4;  // padded fp32 row stride of staged tiles

template <int NPAD>
struct RouteSmem {
  static constexpr int LS = NPAD + 1;  // odd stride: conflict-free per-token rows
  static constexpr size_t main_bytes =
      sizeof(float) * (2 * kRouteTokens * kXS + 2 * (NPAD + 1) * kXS);
  static constexpr size_t off_s = 0;
  static constexpr size_t off_p = off_s + sizeof(float) * kRouteTokens * LS;
  static constexpr size_t off_npart = off_p + sizeof(float) * kRouteTokens * LS;
  static constexpr size_t off_lse2 = off_npart + sizeof(float) * 16 * kRouteTokens;
  static constexpr size_t off_nul = off_lse2 + sizeof(float) * kRouteTokens;
  static constexpr size_t off_mask = align_up(off_nul + sizeof(int) * kRouteTokens, 16);
  static constexpr size_t off_tk = off_mask + sizeof(unsigned long long) * kRouteTokens;
  static constexpr size_t off_tkv = off_tk + sizeof(int) * kRouteTokens * kMaxK;
  static constexpr size_t off_rtab = off_tkv + sizeof(float) * kRouteTokens * kMaxK;
  static constexpr size_t epi_bytes = off_rtab + (size_t)kRouteTokens * NPAD;
  static constexpr size_t bytes = main_bytes > epi_bytes ? main_bytes : epi_bytes;
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// d = a * b + d on two fp32 lanes at once (sm_100 paired FMA).
__device__ __forceinline__ void ffma2(float2& d, float2 a, float2 b) {
  unsigned long long dd = *reinterpret_cast<unsigned long long*>(&d);
  const unsigned long long aa = *reinterpret_cast<const unsigned long long*>(&a);
  const unsigned long long bb = *reinterpret_cast<const unsigned long long*>(&b);
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(dd) : "l"(aa), "l"(bb));
  d = *reinterpret_cast<float2*>(&dd);
}

// (value desc, index asc) order: true if (va, ia) precedes (vb, ib).
__device__ __forceinline__ bool ranks_before(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia < ib);
}

// One CTA: 32 tokens x all N+1 logits. Main loop: 128 threads as 8 token
// groups x 16 logit groups; a thread owns 4 tokens (stride 8) x RPT reals
// (stride 16) and 2 of every 32 d-columns of the null logit. Epilogue: 4
// threads per token (reals i = q, q+4, ...), combined with 4-lane shuffles.
template <int RPT>
__global__ void __launch_bounds__(kRouteThreads) route_kernel(RouteArgs a) {
  constexpr int NPAD = 16 * RPT;
  constexpr int NQ = NPAD / 4;  // reals per epilogue thread
  using SM = RouteSmem<NPAD>;
  constexpr int LS = SM::LS;
  extern __shared__ __align__(16) unsigned char smem[];
  float* xst = reinterpret_cast<float*>(smem);              // [2][32][kXS]
  float* wst = xst + 2 * kRouteTokens * kXS;                // [2][NPAD+1][kXS]

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int tg = lane & 7;                  // token group 0..7
  const int lg = warp * 4 + (lane >> 3);    // logit group 0..15
  const int b = blockIdx.x;
  const int T = a.T, d = a.d, N = a.N, M = a.M, K = a.K;
  const int tok0 = b * kRouteTokens;
  const int nvalid = min(kRouteTokens, T - tok0);
  const int nkt = d / kRouteBK;

  // Paired fp32 FMAs (fma.rn.f32x2): .x accumulates the even d-columns, .y the
  // odd ones; the two partial sums are added once at the end.
  float2 acc[4][RPT];
  float2 accn[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    accn[i] = make_float2(0.f, 0.f);
#pragma unroll
    for (int j = 0; j < RPT; ++j) acc[i][j] = make_float2(0.f, 0.f);
  }

  // x tile: 32 rows x 32 bf16 = 128 16-byte chunks, one per thread
  const int xrow = tid >> 2, xcol8 = (tid & 3) * 8;
  const bool xok = tok0 + xrow < T;
  const uint16_t* xsrc = a.x + (size_t)(tok0 + xrow) * d + xcol8;
  uint4 xr = make_uint4(0u, 0u, 0u, 0u);
  auto load_x = [&](int kt) {
    if (xok) xr = __ldg(reinterpret_cast<const uint4*>(xsrc + (size_t)kt * kRouteBK));
  };
  auto store_x = [&](int buf) {
    float4* dst = reinterpret_cast<float4*>(xst + buf * kRouteTokens * kXS + xrow * kXS + xcol8);
    dst[0] = make_float4(bf16lo(xr.x), bf16hi(xr.x), bf16lo(xr.y), bf16hi(xr.y));
    dst[1] = make_float4(bf16lo(xr.z), bf16hi(xr.z), bf16lo(xr.w), bf16hi(xr.w));
  };
  auto load_w = [&](int kt, int buf) {
    float* wb = wst + buf * (NPAD + 1) * kXS;
    for (int c = tid; c < (NPAD + 1) * 8; c += kRouteThreads) {
      const int r = c >> 3, col4 = (c & 7) * 4;
      const int src_row = (r < N) ? r : (r == NPAD ? N : -1);
      const float* src = a.w + (size_t)(src_row < 0 ? 0 : src_row) * d + (size_t)kt * kRouteBK + col4;
      cp_async16(smem_u32(wb + r * kXS + col4), src, src_row < 0 ? 0 : 16);
    }
    cp_async_commit();
  };

  load_x(0);
  load_w(0, 0);
  for (int kt = 0; kt < nkt; ++kt) {
    const int buf = kt & 1;
    store_x(buf);
    cp_async_wait_all();
    __syncthreads();
    if (kt + 1 < nkt) {
      load_x(kt + 1);
      load_w(kt + 1, buf ^ 1);
    }
    const float* xb = xst + buf * kRouteTokens * kXS;
    const float* wb = wst + buf * (NPAD + 1) * kXS;
#pragma unroll
    for (int kk = 0; kk < kRouteBK / 4; ++kk) {
      float4 xv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) xv[i] = *reinterpret_cast<const float4*>(xb + (tg + 8 * i) * kXS + kk * 4);
#pragma unroll
      for (int jj = 0; jj < RPT; ++jj) {
        const float4 wv = *reinterpret_cast<const float4*>(wb + (lg + 16 * jj) * kXS + kk * 4);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          ffma2(acc[i][jj], make_float2(xv[i].x, xv[i].y), make_float2(wv.x, wv.y));
          ffma2(acc[i][jj], make_float2(xv[i].z, xv[i].w), make_float2(wv.z, wv.w));
        }
      }
    }
    {  // the null logit: this logit group's 2 columns of the d-tile
      const float2 wn = *reinterpret_cast<const float2*>(wb + NPAD * kXS + lg * 2);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 xv = *reinterpret_cast<const float2*>(xb + (tg + 8 * i) * kXS + lg * 2);
        ffma2(accn[i], xv, wn);
      }
    }
  }
  __syncthreads();  // main-loop buffers are reused below

  float* s_l = reinterpret_cast<float*>(smem + SM::off_s);
  float* p_s = reinterpret_cast<float*>(smem + SM::off_p);
  float* npart = reinterpret_cast<float*>(smem + SM::off_npart);
  float* lse2 = reinterpret_cast<float*>(smem + SM::off_lse2);
  int* nul = reinterpret_cast<int*>(smem + SM::off_nul);
  unsigned long long* mask = reinterpret_cast<unsigned long long*>(smem + SM::off_mask);
  int* tk = reinterpret_cast<int*>(smem + SM::off_tk);
  float* tkv = reinterpret_cast<float*>(smem + SM::off_tkv);
  unsigned char* rtab = smem + SM::off_rtab;

#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int t = tg + 8 * i;
#pragma unroll
    for (int jj = 0; jj < RPT; ++jj) {
      const int j = lg + 16 * jj;
      if (j < N) s_l[t * LS + j] = (acc[i][jj].x + acc[i][jj].y) + (a.bias ? __ldg(a.bias + j) : 0.f);
    }
    npart[lg * kRouteTokens + t] = accn[i].x + accn[i].y;
  }
  __syncthreads();

  {
    // ---- per-token routing, 4 lanes per token (all lanes take part in the shuffles)
    const int t = tid >> 2, q = tid & 3;
    const bool valid = t < nvalid;
    const int tok = tok0 + t;
    float sn = 0.f;
#pragma unroll
    for (int l = 0; l < 16; ++l) sn += npart[l * kRouteTokens + t];
    if (a.bias) sn += __ldg(a.bias + N);
    if (a.tnb && valid) sn += __ldg(a.tnb + tok);
    float v[NQ];
#pragma unroll
    for (int u = 0; u < NQ; ++u) {
      const int i = q + 4 * u;
      v[u] = (i < N) ? s_l[t * LS + i] : -INFINITY;
    }
    // softmax statistics over the pool (M copies of the null logit)
    float m = -INFINITY;
#pragma unroll
    for (int u = 0; u < NQ; ++u) m = fmaxf(m, v[u]);
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
    if (M > 0) m = fmaxf(m, sn);
    float z = 0.f;
#pragma unroll
    for (int u = 0; u < NQ; ++u)
      if (q + 4 * u < N) z += expf(v[u] - m);
    z += __shfl_xor_sync(0xffffffffu, z, 1);
    z += __shfl_xor_sync(0xffffffffu, z, 2);
    const float Z = (M > 0) ? z + (float)M * expf(sn - m) : z;
    const float lse = m + logf(Z);
    // p_i = e^{s_i - lse} evaluated as e^{s_i - m} / Z: no cancellation when |m| is large
#pragma unroll
    for (int u = 0; u < NQ; ++u) {
      const int i = q + 4 * u;
      if (i < N) p_s[t * LS + i] = expf(v[u] - m) / Z;
    }
    if (q == 0) {
      p_s[t * LS + NPAD] = (M > 0) ? expf(sn - m) / Z : 0.f;
      lse2[t] = lse * lse;
    }

    // top-K over the pool, in rank order: K rounds of "best remaining real"
    // against the null logit (a real equal to it wins: lower index)
    unsigned sel = 0u;
    int used = 0, r = 0;
    unsigned long long msk = 0ull;
    for (int k = 0; k < K; ++k) {
      float bv = -INFINITY;
      int bi = INT_MAX;
#pragma unroll
      for (int u = 0; u < NQ; ++u) {
        const int i = q + 4 * u;
        if (i < N && !((sel >> u) & 1u) && ranks_before(v[u], i, bv, bi)) {
          bv = v[u];
          bi = i;
        }
      }
#pragma unroll
      for (int off = 1; off <= 2; off <<= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
        if (ranks_before(ov, oi, bv, bi)) {
          bv = ov;
          bi = oi;
        }
      }
      const bool take_null = (used < M) && (bi == INT_MAX || bv < sn);
      int id;
      if (take_null) {
        id = N + used;
        ++used;
      } else {
        id = bi;
        ++r;
        msk |= 1ull << bi;
        if ((bi & 3) == q) sel |= 1u << (bi >> 2);
      }
      if (q == 0) {
        tk[t * kMaxK + k] = id;
        tkv[t * kMaxK + k] = bv;
      }
    }
    __syncwarp();
    if (valid) {
      if (q == 0) {
        // gates: softmax over the selected real logits (rank order: first real is the max)
        float smax = 0.f, gsum = 0.f;
        bool first = true;
        for (int k = 0; k < K; ++k) {
          if (tk[t * kMaxK + k] < N) {
            const float sv = tkv[t * kMaxK + k];
            if (first) {
              smax = sv;
              first = false;
            }
            gsum += expf(sv - smax);
          }
        }
        for (int k = 0; k < K; ++k) {
          const int id = tk[t * kMaxK + k];
          const float g = (id < N) ? expf(tkv[t * kMaxK + k] - smax) / gsum : 0.f;
          a.topk_idx[(size_t)tok * K + k] = id;
          a.topk_gate[(size_t)tok * K + k] = g;
        }
        a.n_real[tok] = r;
        nul[t] = K - r;
        mask[t] = msk;
      }
      if (a.logits) {
        float* lo = a.logits + (size_t)tok * (N + 1);
#pragma unroll
        for (int u = 0; u < NQ; ++u) {
          const int i = q + 4 * u;
          if (i < N) lo[i] = v[u];
        }
        if (q == 0) lo[N] = sn;
      }
    }
  }
  __syncthreads();

  // Per-block ranks and counts (ascending token order inside an expert), P sums.
  if (tid < N) {
    const int e = tid;
    int cnt = 0;
    for (int t = 0; t < nvalid; ++t) {
      if ((mask[t] >> e) & 1ull) rtab[t * NPAD + e] = (unsigned char)(cnt++);
    }
    a.counts_blk[(size_t)e * a.nblk + b] = cnt;
    if (cnt) atomicAdd(a.tot + e, cnt);
  }
  if (tid <= N) {
    const int col = (tid < N) ? tid : NPAD;
    float s = 0.f;
    for (int t = 0; t < nvalid; ++t) s += p_s[t * LS + col];
    a.ppart[(size_t)b * (N + 1) + tid] = s;
  }
  __syncthreads();
  if (tid <= K) {
    int cnt = 0;
    for (int t = 0; t < nvalid; ++t) cnt += (nul[t] == tid);
    a.hist[(size_t)b * (K + 1) + tid] = cnt;
  }
  if (tid == 32) {
    float s = 0.f;
    for (int t = 0; t < nvalid; ++t) s += lse2[t];
    a.lsq[b] = s;
  }
  if (tid < nvalid * 4) {
    // lrank for (token, slot): 4 threads per token, slots k = q, q+4, ...
    const int t = tid >> 2, q = tid & 3;
    const int tok = tok0 + t;
    for (int k = q; k < K; k += 4) {
      const int id = tk[t * kMaxK + k];
      a.lrank[(size_t)tok * K + k] = (id < N) ? (int)rtab[t * NPAD + id] : -1;
    }
  }
}

// Per-expert scan over route blocks: bases[e][b] = offsets[e] + sum_{b' < b}
// counts_blk[e][b'] (ascending token order inside an expert's segment), with
// offsets[e] = sum_{e' < e} tot[e'] from the route blocks' integer atomics.
// Integer sums, so the result does not depend on any execution order.
constexpr int kScanThreads = 256;

struct ScanArgs {
  const int32_t* counts_blk;
  const int32_t* tot;
  int32_t* bases;
  int32_t* counts;
  int32_t* offsets;
  // first-level aux reduction (CTAs N .. N+nparts-1)
  const float* ppart;   // [nblk][N+1]
  const int32_t* hist;  // [nblk][K+1]
  const float* lsq;     // [nblk]
  double* auxp;         // [nparts][cols]
  int N, K, nblk, nparts;
};

__global__ void __launch_bounds__(kScanThreads) scan_kernel(ScanArgs a) {
  __shared__ int s_warp[kScanThreads / 32];
  __shared__ int s_off;
  __shared__ double s_ph[kScanThreads];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int N = a.N, nblk = a.nblk;
  if ((int)blockIdx.x >= N) {
    // fp64 partial sums of the aux statistics over a fixed slice of route blocks
    const int g = blockIdx.x - N;
    const int b0 = (int)((long long)g * nblk / a.nparts), b1 = (int)((long long)(g + 1) * nblk / a.nparts);
    const int c1 = N + 1, c2 = c1 + a.K + 1, cols = c2 + 1;
    const int nph = kScanThreads / cols;
    const int col = tid % cols, ph = tid / cols;
    double acc = 0.0;
    if (ph < nph) {
      for (int b = b0 + ph; b < b1; b += nph) {
        if (col < c1) acc += (double)a.ppart[(size_t)b * c1 + col];
        else if (col < c2) acc += (double)a.hist[(size_t)b * (a.K + 1) + (col - c1)];
        else acc += (double)a.lsq[b];
      }
    }
    s_ph[tid] = acc;
    __syncthreads();
    if (tid < cols) {
      double s = 0.0;
      for (int q = 0; q < nph; ++q) s += s_ph[q * cols + tid];
      a.auxp[(size_t)g * cols + tid] = s;
    }
    return;
  }
  const int e = blockIdx.x;
  if (tid == 0) {
    int o = 0;
    for (int q = 0; q < e; ++q) o += a.tot[q];
    s_off = o;
    if (e == 0) {
      int run = 0;
      for (int q = 0; q < N; ++q) {
        a.offsets[q] = run;
        a.counts[q] = a.tot[q];
        run += a.tot[q];
      }
      a.offsets[N] = run;
    }
  }
  const int per = (nblk + kScanThreads - 1) / kScanThreads;
  const int b0 = tid * per;
  const int32_t* c = a.counts_blk + (size_t)e * nblk;
  int loc = 0;
  for (int q = 0; q < per; ++q) {
    const int b = b0 + q;
    if (b < nblk) loc += c[b];
  }
  int inc = loc;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += u;
  }
  if (lane == 31) s_warp[warp] = inc;
  __syncthreads();
  int wpre = 0;
  for (int w = 0; w < warp; ++w) wpre += s_warp[w];
  int run = s_off + wpre + inc - loc;
  for (int q = 0; q < per; ++q) {
    const int b = b0 + q;
    if (b < nblk) {
      a.bases[(size_t)e * nblk + b] = run;
      run += c[b];
    }
  }
}

template <int RPT>
static int launch_route_t(const RouteArgs& a, cudaStream_t st) {
  using SM = RouteSmem<16 * RPT>;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(route_kernel<RPT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SM::bytes);
    if (e != cudaSuccess) return cuda_status(e);
    attr_set[dev] = true;
  }
  route_kernel<RPT><<<a.nblk, kRouteThreads, SM::bytes, st>>>(a);
  return cuda_status(cudaGetLastError());
}

int launch_route(const moe_dims_t& d, const uint16_t* x, const float* w_router, const float* bias,
                 const float* tok_null_bias, float* logits_out, int32_t* topk_idx, float* topk_gate,
                 int32_t* n_real, void* ws, cudaStream_t st) {
  const WsLayout L = ws_layout(d);
  RouteArgs a{};
  a.x = x;
  a.w = w_router;
  a.bias = bias;
  a.tnb = tok_null_bias;
  a.logits = logits_out;
  a.topk_idx = topk_idx;
  a.topk_gate = topk_gate;
  a.n_real = n_real;
  a.hdr = ws_ptr<uint32_t>(ws, L.hdr);
  a.tot = ws_ptr<int32_t>(ws, L.hdr + kHdrTotOffset);
  a.counts_blk = ws_ptr<int32_t>(ws, L.counts_blk);
  a.bases = ws_ptr<int32_t>(ws, L.bases);
  a.ppart = ws_ptr<float>(ws, L.ppart);
  a.lsq = ws_ptr<float>(ws, L.lsq);
  a.hist = ws_ptr<int32_t>(ws, L.hist);
  a.lrank = ws_ptr<int32_t>(ws, L.lrank);
  a.counts = ws_ptr<int32_t>(ws, L.counts);
  a.offsets = ws_ptr<int32_t>(ws, L.offsets);
  a.T = d.T;
  a.d = d.d;
  a.N = d.N;
  a.M = d.M;
  a.K = d.K;
  a.nblk = L.nblk;
  // the status word and the per-expert totals start at zero for every layer call
  cudaError_t e = cudaMemsetAsync(a.hdr, 0, kHdrTotOffset + sizeof(int32_t) * d.N, st);
  if (e != cudaSuccess) return cuda_status(e);
  int r;
  if (d.N <= 16) r = launch_route_t<1>(a, st);
  else if (d.N <= 32) r = launch_route_t<2>(a, st);
  else r = launch_route_t<4>(a, st);
  if (r != MOE_OK) return r;
  ScanArgs sa{};
  sa.counts_blk = a.counts_blk;
  sa.tot = a.tot;
  sa.bases = a.bases;
  sa.counts = a.counts;
  sa.offsets = a.offsets;
  sa.ppart = a.ppart;
  sa.hist = a.hist;
  sa.lsq = a.lsq;
  sa.auxp = ws_ptr<double>(ws, L.auxp);
  sa.N = d.N;
  sa.K = d.K;
  sa.nblk = L.nblk;
  sa.nparts = L.nparts;
  scan_kernel<<<d.N + L.nparts, kScanThreads, 0, st>>>(sa);
  return cuda_status(cudaGetLastError());
}

}  // namespace moe
