// moe_route, fp32 CUDA-core variant (selected with MOE_FLAG_ROUTER_FP32_CORES):
// the router product as an fp32 FMA GEMM on the CUDA cores, fused with the
// expanded-pool softmax statistics, top-K over the pool, renormalised gates
// and the per-block statistics that dispatch and the aux losses need. Same
// outputs and workspace contents as the tensor-core route, over 64-token blocks.
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
//    block here (fp32 over 64 tokens) and across blocks in fp64 later.
//
// Layout: one CTA = 64 tokens x all N+1 logits (see route_kernel). x (bf16) is
// widened to fp32 once when staged in shared memory; W_r slices arrive by
// cp.async from a transposed copy made once per call.
#include "moe_internal.cuh"

#include <climits>

namespace moe {
namespace fp32route {

// Tiling of this variant (64-token route blocks).
constexpr int kRouteTokens = kFp32RouteTokens;
constexpr int kRouteBK = 32;        // d-slice per pipeline stage
constexpr int kRouteThreads = 256;  // 8 token groups x logit groups x d-slices


struct RouteArgs {
  const uint16_t* x;
  const float* w;     // [N+1, d]
  const float* wt;    // [d][NPAD+4] W^T of this call (workspace)
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
  int32_t* srctok;  // [T] tokens with a source, appended per block
  int32_t* nsrc;    // their count (zero at the start of every call)
  int T, d, N, M, K, nblk;
};


// Thread tile of the router product: 8 tokens x 8 reals. Shared memory, not
// the FMA pipe, bounds an fp32 CUDA-core GEMM: an a x b register tile loads
// (a + b) / (a b) floats per FMA, and 8 x 8 keeps that at 1/4, the balance
// point of an SM. Staged tiles are stored k-major (x^T and W^T) so a thread
// fetches its 8 tokens and 8 reals at one d-column with four 16-byte loads.
// To keep enough warps, the d-columns of each staged tile are split over S
// thread slices whose partial sums are added once at the end.
constexpr int kTileT = 8;  // tokens per thread
constexpr int kTileR = 8;  // reals per thread
constexpr int kXT = kRouteTokens + 4;  // row stride of the staged x^T tile

template <int LG>
struct RouteGeo {
  static constexpr int NPAD = kTileR * LG;            // padded real count
  static constexpr int TG = kRouteTokens / kTileT;    // token groups (8)
  static constexpr int S = kRouteThreads / (TG * LG); // d-slices per staged tile
  static constexpr int KS = kRouteBK / S;             // d-columns per slice per tile (= LG)
  static_assert(S * KS == kRouteBK, "slices must tile the staged d-range");
  static constexpr int WT = NPAD + 4;                 // row stride of W^T (null at column NPAD)
  static constexpr int WCH = kRouteBK * WT / 4;       // 16-byte chunks of a staged W^T tile
  static constexpr int WPT = (WCH + kRouteThreads - 1) / kRouteThreads;  // chunks per thread
  static constexpr int LS = NPAD + 1;                 // odd row stride
  // x^T: 2 stages; W^T: 3 stages (loaded two tiles ahead); x landing: 2 slots of 16 B per thread
  static constexpr size_t main_bytes =
      sizeof(float) * (2 * kRouteBK * kXT + 3 * kRouteBK * WT + 2 * (size_t)kRouteThreads * 4);
  // slice partial sums [S][64][NPAD+1] alias the main-loop buffers
  static constexpr size_t red_bytes = sizeof(float) * S * kRouteTokens * (NPAD + 1);
  static constexpr size_t regionB = align_up(main_bytes > red_bytes ? main_bytes : red_bytes, 16);
  // region C (after B): null partials and the logits
  static constexpr int NNP = kRouteThreads / kRouteTokens;  // null partial sums per token (4)
  static constexpr size_t off_npart = regionB;
  static constexpr size_t off_s = off_npart + sizeof(float) * NNP * kRouteTokens;
  static constexpr size_t endC = off_s + sizeof(float) * kRouteTokens * LS;
  // per-token scratch reuses region B once the partial sums are folded
  static constexpr size_t off_p = 0;
  static constexpr size_t off_lse2 = off_p + sizeof(float) * kRouteTokens * LS;
  static constexpr size_t off_nul = off_lse2 + sizeof(float) * kRouteTokens;
  static constexpr size_t off_mask = align_up(off_nul + sizeof(int) * kRouteTokens, 16);
  static constexpr size_t off_tk = off_mask + sizeof(unsigned long long) * kRouteTokens;
  static constexpr size_t off_tkv = off_tk + sizeof(int) * kRouteTokens * kMaxK;
  static constexpr size_t off_tokbits = off_tkv + sizeof(float) * kRouteTokens * kMaxK;
  static constexpr size_t endB = off_tokbits + sizeof(unsigned) * 2 * kMaxN;
  static_assert(endB <= regionB, "per-token scratch must fit in region B");
  static constexpr size_t bytes = endC;
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_group1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

// (value desc, index asc) order: true if (va, ia) precedes (vb, ib).
__device__ __forceinline__ bool ranks_before(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia < ib);
}

// W^T for one call: wt[k][j] = W_r[j][k] for real j < N, wt[k][NPAD] = W_r[N][k]
// (the null row), zero for the padding columns; row stride NPAD + 4. One CTA
// per 32 d-columns, through a shared tile so both sides are coalesced.
template <int LG>
__global__ void __launch_bounds__(256) router_transpose_kernel(const float* __restrict__ w, float* __restrict__ wt,
                                                               int N, int d) {
  pdl_wait_then_release();
  using G = RouteGeo<LG>;
  constexpr int NPAD = G::NPAD, WT = G::WT;
  __shared__ float tile[NPAD + 1][33];
  const int k0 = blockIdx.x * 32;
  for (int i = threadIdx.x; i < (NPAD + 1) * 32; i += blockDim.x) {
    const int r = i >> 5, kk = i & 31;
    const int src = (r < N) ? r : (r == NPAD ? N : -1);
    tile[r][kk] = (src >= 0) ? w[(size_t)src * d + k0 + kk] : 0.f;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < 32 * WT; i += blockDim.x) {
    const int kk = i / WT, j = i - kk * WT;
    wt[(size_t)(k0 + kk) * WT + j] = (j <= NPAD) ? tile[j][kk] : 0.f;
  }
}

// One CTA: 64 tokens x all N+1 logits, 256 threads. Main loop: thread
// (s, lg, tg) owns tokens {4tg..4tg+3, 32+4tg..32+4tg+3} and reals
// {4lg..4lg+3, 4LG+4lg..4LG+4lg+3} over the d-columns [s*KS, (s+1)*KS) of
// every staged tile; the null logit of token tid & 63 over the 8 d-columns it stages.
// Epilogue: 4 threads per token.
template <int LG>
__global__ void __launch_bounds__(kRouteThreads, 2) route_kernel(RouteArgs a) {
  pdl_wait_then_release();
  using G = RouteGeo<LG>;
  constexpr int NPAD = G::NPAD, S = G::S, KS = G::KS, LS = G::LS, WT = G::WT;
  constexpr int NQ = NPAD / 4;  // reals per epilogue thread
  extern __shared__ __align__(16) unsigned char smem[];
  float* xsT = reinterpret_cast<float*>(smem);       // [2][BK][kXT]

  const int tid = threadIdx.x;
  const int tg = tid % G::TG;
  const int lg = (tid / G::TG) % LG;
  const int sl = tid / (G::TG * LG);
  const int b = blockIdx.x;
  const int T = a.T, d = a.d, N = a.N, M = a.M, K = a.K;
  const int tok0 = b * kRouteTokens;
  const int nvalid = min(kRouteTokens, T - tok0);
  const int nkt = d / kRouteBK;

  float acc[kTileT][kTileR];
#pragma unroll
  for (int i = 0; i < kTileT; ++i)
#pragma unroll
    for (int j = 0; j < kTileR; ++j) acc[i][j] = 0.f;

  // Staging, two tiles ahead. W^T tile kt+2 is copied by cp.async straight
  // into its slot of a 3-deep ring (rows of NPAD+4 floats, already transposed
  // by router_transpose_kernel). x: thread copies token tid & 63, 8 d-columns
  // from (tid >> 6) * 8, into its own landing slot; after its own wait it
  // widens them into the x^T stage of tile kt+1 and adds their share of the
  // null logit (null weights from global, cached). No registers are held
  // across the multiply.
  float* wsT = xsT + 2 * kRouteBK * kXT;                       // [3][BK][WT]
  float* land0 = wsT + 3 * kRouteBK * WT;                      // [2][256][4]
  const int xrow = tid & 63, xkc = (tid >> 6) * 8;
  const bool xok = tok0 + xrow < T;
  const uint16_t* xsrc = a.x + (size_t)(tok0 + (xok ? xrow : 0)) * d + xkc;
  const float* wnull = a.w + (size_t)N * d + xkc;
  float accn = 0.f;  // null logit of token xrow over its staged columns
  auto load_tiles = [&](int kt) {
    if (kt < nkt) {
      cp_async16(smem_u32(land0 + ((kt & 1) * kRouteThreads + tid) * 4), xsrc + (size_t)kt * kRouteBK, xok ? 16 : 0);
      float* wb = wsT + (kt % 3) * kRouteBK * WT;
      const float* src = a.wt + (size_t)kt * kRouteBK * WT;
#pragma unroll
      for (int q = 0; q < G::WPT; ++q) {
        const int c = tid + kRouteThreads * q;
        if (c < G::WCH) cp_async16(smem_u32(wb + 4 * c), src + 4 * c, 16);
      }
    }
    cp_async_commit();  // one group per call, possibly empty
  };
  auto store_x = [&](int kt) {
    const uint4 xr = *reinterpret_cast<const uint4*>(land0 + ((kt & 1) * kRouteThreads + tid) * 4);
    float* xb = xsT + (kt & 1) * kRouteBK * kXT;
    const float xv[8] = {bf16lo(xr.x), bf16hi(xr.x), bf16lo(xr.y), bf16hi(xr.y),
                         bf16lo(xr.z), bf16hi(xr.z), bf16lo(xr.w), bf16hi(xr.w)};
#pragma unroll
    for (int u = 0; u < 8; ++u) xb[(xkc + u) * kXT + xrow] = xv[u];
    const float4 w0 = __ldg(reinterpret_cast<const float4*>(wnull + (size_t)kt * kRouteBK));
    const float4 w1 = __ldg(reinterpret_cast<const float4*>(wnull + (size_t)kt * kRouteBK + 4));
    const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
    for (int u = 0; u < 8; ++u) accn = fmaf(xv[u], wv[u], accn);
  };

  load_tiles(0);
  load_tiles(1);
  cp_async_wait_group1();  // this thread's copies of tile 0
  store_x(0);
  for (int kt = 0; kt < nkt; ++kt) {
    __syncthreads();
    load_tiles(kt + 2);  // its W^T slot was last read at iteration kt-1; its x slot was written out
    const float* xb = xsT + (kt & 1) * kRouteBK * kXT + (sl * KS) * kXT;
    const float* wb = wsT + (kt % 3) * kRouteBK * WT + (sl * KS) * WT;
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
      const float4 xa = *reinterpret_cast<const float4*>(xb + kk * kXT + 4 * tg);
      const float4 xc = *reinterpret_cast<const float4*>(xb + kk * kXT + 32 + 4 * tg);
      const float4 wa = *reinterpret_cast<const float4*>(wb + kk * WT + 4 * lg);
      const float4 wc = *reinterpret_cast<const float4*>(wb + kk * WT + 4 * LG + 4 * lg);
      const float xv[8] = {xa.x, xa.y, xa.z, xa.w, xc.x, xc.y, xc.z, xc.w};
      const float wv[8] = {wa.x, wa.y, wa.z, wa.w, wc.x, wc.y, wc.z, wc.w};
#pragma unroll
      for (int i = 0; i < kTileT; ++i)
#pragma unroll
        for (int jj = 0; jj < kTileR; ++jj) acc[i][jj] = fmaf(xv[i], wv[jj], acc[i][jj]);
    }
    if (kt + 1 < nkt) {
      cp_async_wait_group1();  // this thread's copies of tile kt+1 (tile kt+2 may be in flight)
      store_x(kt + 1);         // x^T stage (kt+1)&1 was last read before this iteration's barrier
    }
  }
  cp_async_wait_all();
  __syncthreads();  // main-loop buffers are reused below

  float* red = reinterpret_cast<float*>(smem);  // [S][64][NPAD+1]
  float* npart = reinterpret_cast<float*>(smem + G::off_npart);
  float* s_l = reinterpret_cast<float*>(smem + G::off_s);
#pragma unroll
  for (int i = 0; i < kTileT; ++i) {
    const int t = 4 * tg + (i & 3) + 32 * (i >> 2);
#pragma unroll
    for (int jj = 0; jj < kTileR; ++jj) {
      const int r = 4 * lg + (jj & 3) + 4 * LG * (jj >> 2);
      red[(sl * kRouteTokens + t) * (NPAD + 1) + r] = acc[i][jj];
    }
  }
  npart[(tid >> 6) * kRouteTokens + (tid & 63)] = accn;
  __syncthreads();
  for (int o = tid; o < kRouteTokens * NPAD; o += kRouteThreads) {
    const int t = o / NPAD, j = o - t * NPAD;
    if (j < N) {
      float v = 0.f;
#pragma unroll
      for (int q = 0; q < S; ++q) v += red[(q * kRouteTokens + t) * (NPAD + 1) + j];
      s_l[t * LS + j] = v + (a.bias ? __ldg(a.bias + j) : 0.f);
    }
  }
  __syncthreads();  // region B is free from here on

  float* p_s = reinterpret_cast<float*>(smem + G::off_p);
  float* lse2 = reinterpret_cast<float*>(smem + G::off_lse2);
  int* nul = reinterpret_cast<int*>(smem + G::off_nul);
  unsigned long long* mask = reinterpret_cast<unsigned long long*>(smem + G::off_mask);
  int* tk = reinterpret_cast<int*>(smem + G::off_tk);
  float* tkv = reinterpret_cast<float*>(smem + G::off_tkv);
  unsigned* tokbits = reinterpret_cast<unsigned*>(smem + G::off_tokbits);  // [2][kMaxN]

  {
    // ---- per-token routing, 4 lanes per token (all lanes take part in the shuffles)
    const int t = tid >> 2, q = tid & 3;
    const bool valid = t < nvalid;
    const int tok = tok0 + t;
    float sn = 0.f;
#pragma unroll
    for (int l = 0; l < G::NNP; ++l) sn += npart[l * kRouteTokens + t];
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

  // Per-block ranks and counts (ascending token order inside an expert): for
  // each expert e, warps 0 and 1 ballot bit e of their 32 tokens' selection
  // masks, giving the block's tokens that chose e as a 64-bit set; a slot's
  // rank is the number of earlier tokens in that set.
  const int lane = tid & 31, warp = tid >> 5;
  if (warp < 2) {
    const int t = 32 * warp + lane;
    const unsigned long long m = (t < nvalid) ? mask[t] : 0ull;
    for (int e = 0; e < N; ++e) {
      const unsigned bits = __ballot_sync(0xffffffffu, (m >> e) & 1ull);
      if (lane == 0) tokbits[warp * kMaxN + e] = bits;
    }
  }
  if (tid >= 64 && tid <= 64 + N) {  // probability sums of the block, one column per thread
    const int i = tid - 64;
    const int col = (i < N) ? i : NPAD;
    float s = 0.f;
    for (int t = 0; t < nvalid; ++t) s += p_s[t * LS + col];
    a.ppart[(size_t)b * (N + 1) + i] = s;
  }
  if (tid >= 160 && tid <= 160 + K) {
    const int c = tid - 160;
    int cnt = 0;
    for (int t = 0; t < nvalid; ++t) cnt += (nul[t] == c);
    a.hist[(size_t)b * (K + 1) + c] = cnt;
  }
  if (tid == 192) {
    float s = 0.f;
    for (int t = 0; t < nvalid; ++t) s += lse2[t];
    a.lsq[b] = s;
  }
  __syncthreads();
  if (tid < N) {
    const int cnt = __popc(tokbits[tid]) + __popc(tokbits[kMaxN + tid]);
    a.counts_blk[(size_t)tid * a.nblk + b] = cnt;
    if (cnt) atomicAdd(a.tot + tid, cnt);
  }
  if (tid < nvalid * 4) {
    // lrank for (token, slot): 4 threads per token, slots k = q, q+4, ...
    const int t = tid >> 2, q = tid & 3;
    const int tok = tok0 + t;
    const int w = t >> 5;
    const unsigned below = (1u << (t & 31)) - 1u;
    for (int k = q; k < K; k += 4) {
      const int id = tk[t * kMaxK + k];
      int rank = -1;
      if (id < N) rank = __popc(tokbits[w * kMaxN + id] & below) + (w ? __popc(tokbits[id]) : 0);
      a.lrank[(size_t)tok * K + k] = rank;
    }
  }
  // the block's tokens with a source (a real expert: this route has no copy or constant
  // experts), appended to the token list with one atomic
  if (tid >= 224) {
    const int lane = tid & 31;
    const bool s0 = lane < nvalid && mask[lane] != 0ull;
    const bool s1 = 32 + lane < nvalid && mask[32 + lane] != 0ull;
    const unsigned w0 = __ballot_sync(0xffffffffu, s0), w1 = __ballot_sync(0xffffffffu, s1);
    const int c0 = __popc(w0), n = c0 + __popc(w1);
    if (n > 0) {
      int at = 0;
      if (lane == 0) at = atomicAdd(a.nsrc, n);
      at = __shfl_sync(0xffffffffu, at, 0);
      const unsigned below = (1u << lane) - 1u;
      if (at >= 0 && at + n <= T) {
        if (s0) a.srctok[at + __popc(w0 & below)] = tok0 + lane;
        if (s1) a.srctok[at + c0 + __popc(w1 & below)] = tok0 + 32 + lane;
      } else if (lane == 0) {
        atomicOr(a.hdr, kStatusBounds);  // more tokens than T: the count was not cleared
      }
    }
  }
}

template <int LG>
static int launch_route_t(const RouteArgs& a, cudaStream_t st) {
  using SM = RouteGeo<LG>;
  const int rt = launch_pdl(router_transpose_kernel<LG>, dim3(a.d / 32), dim3(256), 0, st, a.w,
                            const_cast<float*>(a.wt), a.N, a.d);
  if (rt != MOE_OK) return rt;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(route_kernel<LG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SM::bytes);
    if (e != cudaSuccess) return cuda_status(e);
    attr_set[dev] = true;
  }
  return launch_pdl(route_kernel<LG>, dim3(a.nblk), dim3(kRouteThreads), SM::bytes, st, a);
}

}  // namespace fp32route

int launch_route_fp32(const moe_dims_t& d, const uint16_t* x, const float* w_router, const float* bias,
                      const float* tok_null_bias, float* logits_out, int32_t* topk_idx, float* topk_gate,
                      int32_t* n_real, void* ws, cudaStream_t st) {
  using namespace fp32route;
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
  a.wt = ws_ptr<float>(ws, L.wprep);
  a.tot = ws_ptr<int32_t>(ws, L.hdr + kHdrTotOffset);
  a.counts_blk = ws_ptr<int32_t>(ws, L.counts_blk);
  a.bases = ws_ptr<int32_t>(ws, L.bases);
  a.ppart = ws_ptr<float>(ws, L.ppart);
  a.lsq = ws_ptr<float>(ws, L.lsq);
  a.hist = ws_ptr<int32_t>(ws, L.hist);
  a.lrank = ws_ptr<int32_t>(ws, L.lrank);
  a.counts = ws_ptr<int32_t>(ws, L.counts);
  a.offsets = ws_ptr<int32_t>(ws, L.offsets);
  a.srctok = ws_ptr<int32_t>(ws, L.srctok);
  a.nsrc = ws_ptr<int32_t>(ws, L.hdr + kHdrSrcOffset);
  a.T = d.T;
  a.d = d.d;
  a.N = d.N;
  a.M = d.M;
  a.K = d.K;
  a.nblk = L.nblk;
  // the status word, the per-expert totals and the down GEMM's counters start at zero for
  // every layer call
  cudaError_t e = cudaMemsetAsync(a.hdr, 0, kHdrClearBytes, st);
  if (e != cudaSuccess) return cuda_status(e);
  int r;
  if (d.N <= 8) r = launch_route_t<1>(a, st);
  else if (d.N <= 16) r = launch_route_t<2>(a, st);
  else if (d.N <= 32) r = launch_route_t<4>(a, st);
  else r = launch_route_t<8>(a, st);
  if (r != MOE_OK) return r;
  return launch_route_scan(d, ws, st);
}

}  // namespace moe
