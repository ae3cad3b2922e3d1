// moe_route: router product on the tensor cores, fused with the expanded-pool
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
//    block here (fp32 over 128 tokens) and across blocks in fp64 later.
//
// The router is an fp32 linear layer over bf16 tokens. Its product runs on the
// tcgen05 tensor cores at fp32 accuracy: every fp32 weight w is the exact sum
// of three bf16 numbers hi + mid + lo (each term takes the next 8 significant
// bits), a bf16 x bf16 product is exact, and the MMA accumulates in fp32. So
// s_j = sum_c x_c (hi_jc + mid_jc + lo_jc) is evaluated as three fp32
// accumulations (one MMA with the three terms side by side in N) added in
// fp32: the same error bound as an fp32 dot product of length d, with two
// more roundings.
//
// Layout: a persistent CTA per SM takes tiles of 128 tokens x all N+1 logits (one
// M=128 MMA tile each) in turn. Warp 0 issues TMA loads of the x tile (128 x 64
// bf16) and the split weight tile (3*NPW x 64 bf16) into a 3-stage ring, running
// ahead across tiles; warp 1 issues the MMAs (M=128, N=3*NPW, K=16) from one
// thread into one of two TMEM accumulators; warps 2-17 add the three terms per
// logit into shared memory (which frees the accumulator for the tile after next),
// then route the 128 tokens with 4 lanes per token while the next tile's product
// is already running.
#include "moe_internal.cuh"

#include <climits>

namespace moe {

struct RouteArgs {
  int32_t* tot;       // [N] rows per expert (integer atomics; zero at the start of every call)
  const float* bias;  // [N+1] or null
  const float* tnb;   // [T] or null
  float* logits;      // [T, N+1] or null
  int32_t* topk_idx;
  float* topk_gate;
  int32_t* n_real;
  // workspace
  uint32_t* hdr;  // [0] status
  int32_t* counts_blk;
  int32_t* bases;
  float* ppart;
  float* lsq;
  int32_t* hist;
  int32_t* lrank;
  int32_t* counts;
  int32_t* offsets;
  int32_t* srctok;  // [T] tokens with a source, appended per tile
  int32_t* nsrc;    // their count (zero at the start of every call)
  unsigned long long limit_ns;
  int T, d, N, M, K, nblk;
  int ncols;  // router rows N + 1 + C + V (MoE++ copy and constant experts after the null logit)
};

// ---------------------------------------------------------------------------------------
// W_r (fp32 [rows][d], rows = N+1+C+V) -> three bf16 terms, rows t*NPW + j (t = 0 hi,
// 1 mid, 2 lo), zero rows for rows <= j < NPW. With w = m 2^e (24-bit m): hi = RN8(w) leaves a
// remainder of at most 16 significant bits, mid = RN8(remainder) leaves at most
// 8, and lo holds those exactly; both subtractions are exact in fp32.
__device__ __forceinline__ void split3(float w, uint16_t& h, uint16_t& m, uint16_t& l) {
  const __nv_bfloat16 bh = __float2bfloat16_rn(w);
  const float r1 = w - __bfloat162float(bh);
  const __nv_bfloat16 bm = __float2bfloat16_rn(r1);
  const float r2 = r1 - __bfloat162float(bm);
  const __nv_bfloat16 bl = __float2bfloat16_rn(r2);
  h = __bfloat16_as_ushort(bh);
  m = __bfloat16_as_ushort(bm);
  l = __bfloat16_as_ushort(bl);
}

// One thread per 8 d-columns of one padded row. With hdr set, block 0 also clears the
// first `nclear` words of the workspace header (status word, per-expert totals and the
// counters of the down GEMM with the combine folded in), which must start at zero for
// every layer call; with npw = 0 that is all it does (the weight was split beforehand).
__global__ void __launch_bounds__(256) router_split_kernel(const float* __restrict__ w, uint16_t* __restrict__ w3,
                                                           int rows, int npw, int d, uint32_t* hdr, int nclear) {
  pdl_wait_then_release();
  if (hdr != nullptr && blockIdx.x == 0)
    for (int i = threadIdx.x; i < nclear; i += blockDim.x) hdr[i] = 0u;
  const int nch = d >> 3;
  const long long total = (long long)npw * nch;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int j = (int)(i / nch), c = (int)(i - (long long)j * nch);
    uint16_t hv[8], mv[8], lv[8];
    if (j < rows) {
      const float4* src = reinterpret_cast<const float4*>(w + (size_t)j * d + (size_t)c * 8);
      const float4 p0 = __ldg(src), p1 = __ldg(src + 1);
      const float v[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
      for (int e = 0; e < 8; ++e) split3(v[e], hv[e], mv[e], lv[e]);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) hv[e] = mv[e] = lv[e] = 0;
    }
    auto pack = [](const uint16_t (&u)[8]) {
      return make_uint4(u[0] | ((uint32_t)u[1] << 16), u[2] | ((uint32_t)u[3] << 16),
                        u[4] | ((uint32_t)u[5] << 16), u[6] | ((uint32_t)u[7] << 16));
    };
    const size_t col = (size_t)c * 8;
    *reinterpret_cast<uint4*>(w3 + (size_t)j * d + col) = pack(hv);
    *reinterpret_cast<uint4*>(w3 + (size_t)(npw + j) * d + col) = pack(mv);
    *reinterpret_cast<uint4*>(w3 + (size_t)(2 * npw + j) * d + col) = pack(lv);
  }
}

// ---------------------------------------------------------------------------------------
// Shared memory of the route kernel: a 3-stage ring of x and split-weight tiles, and the
// routing scratch of the epilogue beside it (not aliased: the epilogue of one tile runs
// while the ring already fills for the next).
template <int NPW, bool PAIR>
struct RouteSmem {
  static constexpr int STAGES = PAIR ? 4 : 3;
  static constexpr int BROWS = 3 * NPW;                   // rows of the split weight (the MMA's N)
  static constexpr int BROWS_CTA = PAIR ? BROWS / 2 : BROWS;  // rows this CTA loads
  static constexpr int A_BYTES = kRouteTokens * kRouteBK * 2;
  static constexpr int B_BYTES = BROWS_CTA * kRouteBK * 2;
  static constexpr size_t off_a = 0;
  static constexpr size_t off_b = off_a + (size_t)STAGES * A_BYTES;
  static constexpr size_t ring_end = off_b + (size_t)STAGES * B_BYTES;
  // routing scratch
  static constexpr int LS = NPW + 1;  // odd row stride of the logit rows
  static constexpr size_t off_s = ring_end;  // float [128][LS]: logits, then p in place
  static constexpr size_t off_pn = off_s + sizeof(float) * kRouteTokens * LS;  // float [128] null p
  static constexpr size_t off_lse2 = off_pn + sizeof(float) * kRouteTokens;    // float [128]
  static constexpr size_t off_mask = align_up(off_lse2 + sizeof(float) * kRouteTokens, 16);  // u64 [128]
  static constexpr size_t off_tk = off_mask + sizeof(unsigned long long) * kRouteTokens;  // int [128][kMaxK]
  static constexpr size_t off_tkv = off_tk + sizeof(int) * kRouteTokens * kMaxK;          // float [128][kMaxK]
  static constexpr size_t off_tokbits = off_tkv + sizeof(float) * kRouteTokens * kMaxK;  // u32 [4][kMaxN]
  static constexpr int HIST = kMaxK + 1 + kMaxPP;  // null histogram + copy/constant counts
  static constexpr size_t off_hist = off_tokbits + sizeof(unsigned) * 4 * kMaxN;         // int [HIST]
  static constexpr size_t off_srcw = off_hist + sizeof(int) * HIST;  // u32 [4]: tokens with a source
  static constexpr size_t scratch_end = off_srcw + sizeof(unsigned) * 4;
  // full[STAGES], empty[STAGES], tfull[2], tempty[2], drain
  static constexpr size_t off_bar = align_up(scratch_end, 8);
  static constexpr size_t off_misc = off_bar + 8 * (2 * STAGES + 5);  // [0] TMEM base, [1] abort
  static constexpr size_t bytes = off_misc + 16 + 1024;  // + slack for 1024-byte alignment
  static_assert(bytes <= 227 * 1024, "route kernel shared memory");
};

// (value desc, index asc) order: true if (va, ia) precedes (vb, ib).
__device__ __forceinline__ bool ranks_before(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia < ib);
}

// ---------------------------------------------------------------------------------------
// Persistent: one CTA per SM (at most), 576 threads, taking 128-token tiles in turn
// (tokens [128 b, 128 b + 128) x all router rows each). Two TMEM accumulators: the MMA of
// tile i+1 runs while the epilogue routes tile i.
// PAIR: the two CTAs of a cluster share one MMA of M = 256 (tcgen05 cta_group::2) over a
// unit of two consecutive tiles: each CTA loads its own 128 tokens and half of the split
// weight's rows, so the weight, which every tile reads whole, crosses from L2 once per 256
// tokens instead of once per 128. Each CTA's TMEM then holds its own tokens x all logits,
// and the epilogue is unchanged. Without PAIR a unit is one tile.
// NQ: logit columns per lane (4 lanes per token): NPW / 4, or 16 when NPW = 80 and
// there are no copy/constant experts (the candidates are then the reals, columns < 64).
template <int NPW, int NQ, bool PAIR>
__global__ void __launch_bounds__(kRouteThreads, 1)
    route_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                 const RouteArgs a) {
  pdl_wait_then_release();
  using SM = RouteSmem<NPW, PAIR>;
  constexpr int STAGES = SM::STAGES;
  constexpr int LS = SM::LS;
  constexpr uint32_t ACOLS = SM::BROWS <= 64 ? 64u : SM::BROWS <= 128 ? 128u : 256u;  // per accumulator
  constexpr uint32_t TCOLS = 2 * ACOLS;
  constexpr uint32_t IDESC = idesc_bf16_f32(PAIR ? 2 * kRouteTokens : kRouteTokens, SM::BROWS);
  constexpr uint32_t TX = (PAIR ? 2 : 1) * (SM::A_BYTES + SM::B_BYTES);  // one stage, both CTAs

  extern __shared__ unsigned char smem_raw[];
  unsigned char* base =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sA = base + SM::off_a;
  unsigned char* sB = base + SM::off_b;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + SM::off_bar);
  volatile int* misc = reinterpret_cast<volatile int*>(base + SM::off_misc);
  auto full_bar = [&](int s) { return smem_u32(bars + s); };
  auto empty_bar = [&](int s) { return smem_u32(bars + STAGES + s); };
  auto tfull_bar = [&](int s) { return smem_u32(bars + 2 * STAGES + s); };
  auto tempty_bar = [&](int s) { return smem_u32(bars + 2 * STAGES + 2 + s); };
  const uint32_t drain_bar = smem_u32(bars + 2 * STAGES + 4);
  volatile int* abort_flag = misc + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = a.T, N = a.N, M = a.M, K = a.K;
  const int nkb = a.d / kRouteBK;
  const uint32_t crank = PAIR ? cluster_rank() : 0u;
  const bool leader = crank == 0u;
  // units (a tile, or two tiles for a pair) u = unit0, unit0 + ustep, ...; this CTA's tile of
  // unit u is tile_of(u) (with an odd tile count the last pair's second CTA has none: its
  // tokens are past T, loaded as zeros and never written)
  const int unit0 = PAIR ? (int)cluster_id_x() : (int)blockIdx.x;
  const int ustep = PAIR ? (int)cluster_count_x() : (int)gridDim.x;
  const int nunit = PAIR ? (a.nblk + 1) / 2 : a.nblk;
  auto tile_of = [&](int u) { return PAIR ? 2 * u + (int)crank : u; };

  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmX);
    prefetch_tmap(&tmW);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(tfull_bar(s), 1);
      mbar_init(tempty_bar(s), (PAIR ? 2 : 1) * (kRouteEpiThreads / 32));  // one arrival per epilogue warp
    }
    mbar_init(drain_bar, 1);
    misc[1] = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc_pair(smem_u32(const_cast<int*>(misc)), TCOLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(const_cast<int*>(misc)), TCOLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  if constexpr (PAIR) cluster_sync_all();  // both CTAs' barriers initialised, TMEM allocated
  else __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = (uint32_t)misc[0];

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------ TMA producer (runs ahead across tiles)
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_par = 0;
      bool ok = true;
      for (int u = unit0; u < nunit && ok; u += ustep) {
        const int b = tile_of(u);
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait_bounded(empty_bar(stage), phase ^ 1u, a.limit_ns, abort_flag, a.hdr)) {
            ok = false;
            break;
          }
          if constexpr (PAIR) {
            // both CTAs' copies of a stage complete on the leader's barrier
            const uint32_t fb = map_to_rank(full_bar(stage), 0);
            if (leader) mbar_arrive_expect_tx(full_bar(stage), TX);
            tma_load_2d_pair(smem_u32(sA + stage * SM::A_BYTES), &tmX, fb, kb * kRouteBK, b * kRouteTokens);
            tma_load_2d_pair(smem_u32(sB + stage * SM::B_BYTES), &tmW, fb, kb * kRouteBK,
                             (int)crank * SM::BROWS_CTA);
          } else {
            mbar_arrive_expect_tx(full_bar(stage), TX);
            tma_load_2d(smem_u32(sA + stage * SM::A_BYTES), &tmX, full_bar(stage), kb * kRouteBK,
                        b * kRouteTokens);
            tma_load_2d(smem_u32(sB + stage * SM::B_BYTES), &tmW, full_bar(stage), kb * kRouteBK, 0);
          }
          armed |= 1u << stage;
          armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (*abort_flag && leader) {
        // let every issued copy land before the CTA can exit (a pair's copies all count on
        // the leader's barriers)
        for (int s = 0; s < STAGES; ++s)
          if (armed & (1u << s))
            (void)mbar_wait_bounded(full_bar(s), (armed_par >> s) & 1u, a.limit_ns, nullptr, a.hdr);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ------------------------------ MMA issuer (single thread; the leader's, for a pair)
      int stage = 0;
      uint32_t phase = 0;
      int li = 0;
      bool ok = true;
      for (int u = unit0; u < nunit && ok; u += ustep, ++li) {
        const int acc = li & 1;
        const uint32_t ap = (uint32_t)(li >> 1) & 1u;
        if (!mbar_wait_bounded(tempty_bar(acc), ap ^ 1u, a.limit_ns, abort_flag, a.hdr)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)acc * ACOLS;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait_bounded(full_bar(stage), phase, a.limit_ns, abort_flag, a.hdr)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t adesc = smem_desc_sw128(smem_u32(sA + stage * SM::A_BYTES));
          const uint64_t bdesc = smem_desc_sw128(smem_u32(sB + stage * SM::B_BYTES));
#pragma unroll
          for (int k = 0; k < kRouteBK / 16; ++k) {
            if constexpr (PAIR)
              tc_mma_pair(d_tmem, adesc + (uint64_t)(2 * k), bdesc + (uint64_t)(2 * k), IDESC,
                          (kb | k) != 0 ? 1u : 0u);
            else
              tc_mma_f16(d_tmem, adesc + (uint64_t)(2 * k), bdesc + (uint64_t)(2 * k), IDESC,
                         (kb | k) != 0 ? 1u : 0u);
          }
          if constexpr (PAIR) {  // free this stage in both CTAs
            tc_commit_pair(empty_bar(stage));
            tc_commit_pair(map_to_rank(empty_bar(stage), 1));
          } else {
            tc_commit(empty_bar(stage));
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) {
          if constexpr (PAIR) {
            tc_commit_pair(tfull_bar(acc));
            tc_commit_pair(map_to_rank(tfull_bar(acc), 1));
          } else {
            tc_commit(tfull_bar(acc));
          }
        }
      }
      // fires once every MMA issued above has completed (also after an abort)
      if constexpr (PAIR) tc_commit_pair(drain_bar);
      else tc_commit(drain_bar);
      (void)mbar_wait_bounded(drain_bar, 0, a.limit_ns, nullptr, a.hdr);
    }
  } else {
    // ------------------------------ epilogue warps 2..17, one tile after another
    const int etid = threadIdx.x - 64;  // 0..511
    const int ew = warp - 2;            // 0..15
    float* s_l = reinterpret_cast<float*>(base + SM::off_s);
    float* pn = reinterpret_cast<float*>(base + SM::off_pn);
    float* lse2 = reinterpret_cast<float*>(base + SM::off_lse2);
    unsigned long long* mask = reinterpret_cast<unsigned long long*>(base + SM::off_mask);
    int* tk = reinterpret_cast<int*>(base + SM::off_tk);
    float* tkv = reinterpret_cast<float*>(base + SM::off_tkv);
    unsigned* tokbits = reinterpret_cast<unsigned*>(base + SM::off_tokbits);  // [4][kMaxN]
    int* s_hist = reinterpret_cast<int*>(base + SM::off_hist);                // [kMaxK+1]
    unsigned* srcw = reinterpret_cast<unsigned*>(base + SM::off_srcw);        // [4]: bit per token
    int li = 0;
    for (int u = unit0; u < nunit; u += ustep, ++li) {
    const int b = tile_of(u);
    const bool live = b < a.nblk;  // false: the empty second tile of an odd tile count
    const int acc = li & 1;
    const uint32_t ap = (uint32_t)(li >> 1) & 1u;
    const int tok0 = b * kRouteTokens;
    const int nvalid = max(0, min(kRouteTokens, T - tok0));
    const bool ok = mbar_wait_bounded(tfull_bar(acc), ap, a.limit_ns, abort_flag, a.hdr) && *abort_flag == 0;
    if (!named_bar_and(1, kRouteEpiThreads, ok)) break;
    {
      // ---- logits from TMEM: warp reads lane quarter q (tokens 32q..32q+31) and
      // every fourth 8-column chunk; s_j = (hi_j + mid_j) + lo_j (+ bias)
      tc_fence_after();
      const int q = warp & 3, part = ew >> 2;
      const int t = q * 32 + lane;
      const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)acc * ACOLS;
      const float tn = (a.tnb != nullptr && t < nvalid) ? __ldg(a.tnb + tok0 + t) : 0.f;
      if (etid < SM::HIST) s_hist[etid] = 0;
      if (etid < 4) srcw[etid] = 0u;
#pragma unroll 1
      for (int c0 = part * 8; c0 < NPW; c0 += 32) {
        uint32_t rh[8], rm[8], rl[8];
        tmem_ld8(tb + (uint32_t)c0, rh);
        tmem_ld8(tb + (uint32_t)(NPW + c0), rm);
        tmem_ld8(tb + (uint32_t)(2 * NPW + c0), rl);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int col = c0 + j;
          if (col < a.ncols) {
            float s = (__uint_as_float(rh[j]) + __uint_as_float(rm[j])) + __uint_as_float(rl[j]);
            if (a.bias) s += __ldg(a.bias + col);
            if (col == N) s += tn;
            s_l[t * LS + col] = s;
          }
        }
      }
      // the accumulator is free for the tile after next (for a pair, once both CTAs say so)
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if constexpr (PAIR) mbar_arrive_cluster(map_to_rank(tempty_bar(acc), 0));
        else mbar_arrive(tempty_bar(acc));
      }
    }
    named_bar_sync(1, kRouteEpiThreads);
    {
      // ---- per-token routing, 4 lanes per token. Lane q holds the distinct candidates
      // in logit columns i = q, q+4, ...: reals (i < N, pool index i) and MoE++ copy and
      // constant experts (N < i < ncols, pool index i - 1 + M); column N is the null logit.
      const int t = etid >> 2, q = etid & 3;
      const bool valid = t < nvalid;
      const int tok = tok0 + t;
      const int ncols = a.ncols;
      auto is_cand = [&](int i) { return i < ncols && i != N; };
      auto pool_of = [&](int i) { return i < N ? i : i - 1 + M; };
      float* row = s_l + t * LS;
      const float sn = row[N];
      float v[NQ];
#pragma unroll
      for (int u = 0; u < NQ; ++u) {
        const int i = q + 4 * u;
        v[u] = is_cand(i) ? row[i] : -INFINITY;
      }
      // softmax statistics over the pool (M copies of the null logit)
      float m = -INFINITY;
#pragma unroll
      for (int u = 0; u < NQ; ++u) m = fmaxf(m, v[u]);
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
      if (M > 0) m = fmaxf(m, sn);
      // (these feed only the aux statistics P and L_z, kept to ~1e-6 relative: the
      // fast exponential and one reciprocal are within that)
      float e[NQ];
      float z = 0.f;
#pragma unroll
      for (int u = 0; u < NQ; ++u) {
        e[u] = is_cand(q + 4 * u) ? __expf(v[u] - m) : 0.f;
        z += e[u];
      }
      z += __shfl_xor_sync(0xffffffffu, z, 1);
      z += __shfl_xor_sync(0xffffffffu, z, 2);
      const float en = (M > 0) ? __expf(sn - m) : 0.f;
      const float Z = (M > 0) ? z + (float)M * en : z;
      const float lse = m + logf(Z);
      const float rz = 1.f / Z;
      // p_i = e^{s_i - lse} evaluated as e^{s_i - m} / Z (no cancellation when |m| is
      // large), written over this lane's own logits
#pragma unroll
      for (int u = 0; u < NQ; ++u) {
        const int i = q + 4 * u;
        if (is_cand(i)) row[i] = e[u] * rz;
      }
      if (q == 0) {
        pn[t] = (M > 0) ? en * rz : 0.f;
        lse2[t] = lse * lse;
      }

      // top-K over the pool, in rank order: K rounds of "best remaining candidate"
      // against the next null copy, compared by (value desc, pool index asc): a real
      // equal to the null logit wins, a copy or constant expert equal to it loses.
      // Taking a null copy leaves the best remaining candidate as it was, and the null
      // keeps beating it while copies remain (a real's index is below every copy's, a
      // copy or constant expert's above), so the candidates are scanned again only after
      // one of them was taken: about r + 1 scans instead of K. The four lanes of a token
      // take the same decisions; the shuffles run within them (tokens diverge).
      const unsigned gmask = 0xFu << (lane & ~3);
      unsigned sel = 0u;
      int used = 0, r = 0, rpp = 0;
      unsigned long long msk = 0ull;
      float smax = 0.f;  // the first non-null slot taken holds the largest gated logit
      float bv = -INFINITY;
      int bi = INT_MAX;
      bool have_best = false;
      for (int k = 0; k < K; ++k) {
        if (!have_best) {
          bv = -INFINITY;
          bi = INT_MAX;
#pragma unroll
          for (int u = 0; u < NQ; ++u) {
            const int i = q + 4 * u;
            if (is_cand(i) && !((sel >> u) & 1u) && ranks_before(v[u], pool_of(i), bv, bi)) {
              bv = v[u];
              bi = pool_of(i);
            }
          }
#pragma unroll
          for (int off = 1; off <= 2; off <<= 1) {
            const float ov = __shfl_xor_sync(gmask, bv, off);
            const int oi = __shfl_xor_sync(gmask, bi, off);
            if (ranks_before(ov, oi, bv, bi)) {
              bv = ov;
              bi = oi;
            }
          }
          have_best = true;
        }
        const bool take_null = (used < M) && (bi == INT_MAX || ranks_before(sn, N + used, bv, bi));
        int id;
        float idv;
        if (take_null) {
          id = N + used;
          idv = sn;
          ++used;
        } else {
          id = bi;
          idv = bv;
          have_best = false;  // taken: the next round scans the remaining candidates
          if (r + rpp == 0) smax = bv;
          if (bi < N) {
            ++r;
            msk |= 1ull << bi;
          } else {
            ++rpp;
          }
          const int ci = (bi < N) ? bi : bi - M + 1;  // logit column of the candidate taken
          if ((ci & 3) == q) sel |= 1u << (ci >> 2);
        }
        if ((k & 3) == q) {  // slot k belongs to lane k mod 4 from here on
          tk[t * kMaxK + k] = id;
          tkv[t * kMaxK + k] = idv;
        }
      }
      // gates: softmax over the selected slots that are not null copies; each lane takes
      // slots q, q+4, ... and the four partial sums are added in a fixed order
      auto gated = [&](int id) { return id < N || id >= N + M; };
      float gsum = 0.f;
      for (int k = q; k < K; k += 4)
        if (gated(tk[t * kMaxK + k])) gsum += expf(tkv[t * kMaxK + k] - smax);
      gsum += __shfl_xor_sync(0xffffffffu, gsum, 1);
      gsum += __shfl_xor_sync(0xffffffffu, gsum, 2);
      if (valid) {
        for (int k = q; k < K; k += 4) {
          const int id = tk[t * kMaxK + k];
          const float g = gated(id) ? expf(tkv[t * kMaxK + k] - smax) / gsum : 0.f;
          a.topk_idx[(size_t)tok * K + k] = id;
          a.topk_gate[(size_t)tok * K + k] = g;
          if (id >= N + M) atomicAdd(s_hist + (K + 1) + (id - N - M), 1);  // copy/constant counts
        }
        if (q == 0) {
          a.n_real[tok] = r;
          atomicAdd(s_hist + (K - r - rpp), 1);  // null slots; integer: order does not matter
          if (r + rpp > 0) atomicOr(srcw + (t >> 5), 1u << (t & 31));  // a source to combine
        }
        mask[t] = msk;  // identical on the token's four lanes
        if (a.logits) {
          float* lo = a.logits + (size_t)tok * ncols;
#pragma unroll
          for (int u = 0; u < NQ; ++u) {
            const int i = q + 4 * u;
            if (is_cand(i)) lo[i] = v[u];
          }
          if (q == 0) lo[N] = sn;
        }
      }
    }
    named_bar_sync(1, kRouteEpiThreads);

    {
      // ---- block statistics. Ballots: warp ew takes the 32 tokens of group ew & 3
      // and experts [16 (ew >> 2), +16); bit e of the selection masks gives the
      // block's tokens that chose e as a 128-bit set (a slot's rank is the number
      // of earlier tokens in it). Column sums of p and the sum of lse^2: lane l
      // adds tokens l, l+32, l+64, l+96 in that order, then a butterfly over the
      // warp (every lane ends with the same, order-fixed total).
      {
        const int g = ew & 3;
        const int tt = 32 * g + lane;
        const unsigned long long mk = (tt < nvalid) ? mask[tt] : 0ull;
        const int e1 = min(N, 16 * (ew >> 2) + 16);
        for (int e = 16 * (ew >> 2); e < e1; ++e) {
          const unsigned bits = __ballot_sync(0xffffffffu, (mk >> e) & 1ull);
          if (lane == 0) tokbits[g * kMaxN + e] = bits;
        }
      }
      const int ncols = a.ncols;
      for (int c = ew; c <= ncols; c += 16) {
        // c < ncols: probability of logit column c (real, the null logit for c == N, copy
        // or constant expert); c == ncols: lse^2
        const float* col = (c == N) ? pn : (c < ncols) ? s_l + c : lse2;
        const int stride = (c == N || c == ncols) ? 1 : LS;
        float sum = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int tt = lane + 32 * i;
          if (tt < nvalid) sum += col[tt * stride];
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        if (lane == 0 && live) {
          if (c < ncols) a.ppart[(size_t)b * ncols + c] = sum;
          else a.lsq[b] = sum;
        }
      }
    }
    named_bar_sync(1, kRouteEpiThreads);

    {
      const int hc = K + 1 + (a.ncols - N - 1);  // null histogram, then copy/constant counts
      if (live && etid < hc) a.hist[(size_t)b * hc + etid] = s_hist[etid];
      if (live && etid < N) {
        int cnt = 0;
#pragma unroll
        for (int w = 0; w < 4; ++w) cnt += __popc(tokbits[w * kMaxN + etid]);
        a.counts_blk[(size_t)etid * a.nblk + b] = cnt;
        if (cnt) atomicAdd(a.tot + etid, cnt);
      }
      // lrank for (token, slot): 4 threads per token, slots k = q, q+4, ...
      const int t = etid >> 2, q = etid & 3;
      if (t < nvalid) {
        const int w = t >> 5;
        const unsigned below = (1u << (t & 31)) - 1u;
        for (int k = q; k < K; k += 4) {
          const int id = tk[t * kMaxK + k];
          int rank = -1;
          if (id < N) {
            rank = __popc(tokbits[w * kMaxN + id] & below);
            for (int w2 = 0; w2 < w; ++w2) rank += __popc(tokbits[w2 * kMaxN + id]);
          }
          a.lrank[(size_t)(tok0 + t) * K + k] = rank;
        }
      }
      // the tile's tokens with a source, appended to the token list with one atomic (the
      // list's order depends on the tiles' timing; the combine's sums do not)
      if (live && ew == 15) {
        const unsigned w0 = srcw[0], w1 = srcw[1], w2 = srcw[2], w3 = srcw[3];
        const int c0 = __popc(w0), c1 = __popc(w1), c2 = __popc(w2);
        const int n = c0 + c1 + c2 + __popc(w3);
        if (n > 0) {
          int at = 0;
          if (lane == 0) at = atomicAdd(a.nsrc, n);
          at = __shfl_sync(0xffffffffu, at, 0);
          const unsigned below = (1u << lane) - 1u;
          if (at >= 0 && at + n <= T) {
            if ((w0 >> lane) & 1u) a.srctok[at + __popc(w0 & below)] = tok0 + lane;
            if ((w1 >> lane) & 1u) a.srctok[at + c0 + __popc(w1 & below)] = tok0 + 32 + lane;
            if ((w2 >> lane) & 1u) a.srctok[at + c0 + c1 + __popc(w2 & below)] = tok0 + 64 + lane;
            if ((w3 >> lane) & 1u) a.srctok[at + c0 + c1 + c2 + __popc(w3 & below)] = tok0 + 96 + lane;
          } else if (lane == 0) {
            atomicOr(a.hdr, kStatusBounds);  // more tokens than T: the count was not cleared
          }
        }
      }
    }
    named_bar_sync(1, kRouteEpiThreads);  // scratch free for the next tile
    }
  }

  tc_fence_before();
  if constexpr (PAIR) cluster_sync_all();  // the leader's MMAs read both CTAs' shared memory
  else __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    if constexpr (PAIR) tmem_dealloc_pair(tmem_base, TCOLS);
    else tmem_dealloc(tmem_base, TCOLS);
  }
}

// ---------------------------------------------------------------------------------------
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
  const float* ppart;   // [nblk][ncols]
  const int32_t* hist;  // [nblk][hcols]
  const float* lsq;     // [nblk]
  double* auxp;         // [nparts][ncols + hcols + 1]
  int N, K, nblk, nparts;
  int ncols, hcols;     // router rows; null histogram + copy/constant expert counts
};

__global__ void __launch_bounds__(kScanThreads) scan_kernel(ScanArgs a) {
  pdl_wait_then_release();
  __shared__ int s_warp[kScanThreads / 32];
  __shared__ int s_off;
  __shared__ double s_ph[kScanThreads];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int N = a.N, nblk = a.nblk;
  if ((int)blockIdx.x >= N) {
    // fp64 partial sums of the aux statistics over a fixed slice of route blocks
    const int g = blockIdx.x - N;
    const int b0 = (int)((long long)g * nblk / a.nparts), b1 = (int)((long long)(g + 1) * nblk / a.nparts);
    const int c1 = a.ncols, c2 = c1 + a.hcols, cols = c2 + 1;
    const int nph = kScanThreads / cols;
    const int col = tid % cols, ph = tid / cols;
    double acc = 0.0;
    if (ph < nph) {
      for (int b = b0 + ph; b < b1; b += nph) {
        if (col < c1) acc += (double)a.ppart[(size_t)b * c1 + col];
        else if (col < c2) acc += (double)a.hist[(size_t)b * a.hcols + (col - c1)];
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
  if (warp == 0) {
    // exclusive prefix of the per-expert totals (N <= 64: two per lane), by shuffles
    const int t0 = (lane < N) ? a.tot[lane] : 0;
    const int t1 = (lane + 32 < N) ? a.tot[lane + 32] : 0;
    int i0 = t0, i1 = t1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u0 = __shfl_up_sync(0xffffffffu, i0, o);
      const int u1 = __shfl_up_sync(0xffffffffu, i1, o);
      if (lane >= o) {
        i0 += u0;
        i1 += u1;
      }
    }
    const int low_total = __shfl_sync(0xffffffffu, i0, 31);
    const int ex0 = i0 - t0, ex1 = low_total + i1 - t1;  // exclusive prefixes of experts lane, lane + 32
    if (lane == (e & 31)) s_off = (e < 32) ? ex0 : ex1;
    if (e == 0) {
      if (lane < N) {
        a.offsets[lane] = ex0;
        a.counts[lane] = t0;
      }
      if (lane + 32 < N) {
        a.offsets[lane + 32] = ex1;
        a.counts[lane + 32] = t1;
      }
      if (lane == 31) a.offsets[N] = low_total + i1;
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

template <int NPW, int NQ, bool PAIR>
static int launch_route_t(const CUtensorMap& tx, const CUtensorMap& tw, const RouteArgs& a, cudaStream_t st) {
  using SM = RouteSmem<NPW, PAIR>;
  auto kern = route_kernel<NPW, NQ, PAIR>;
  static int max_units[64] = {0};  // resident CTAs (or pairs) per device
  int dev = 0;
  cudaGetDevice(&dev);
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = PAIR ? 2 : 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // see launch_pdl
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.blockDim = dim3(kRouteThreads, 1, 1);
  cfg.dynamicSmemBytes = SM::bytes;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (dev >= 0 && dev < 64 && max_units[dev] == 0) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SM::bytes);
    if (e != cudaSuccess) return cuda_status(e);
    int n = PAIR ? sm_count() / 2 : sm_count();
    if (PAIR) {
      int c = 0;
      cfg.gridDim = dim3(2 * (sm_count() / 2), 1, 1);
      if (cudaOccupancyMaxActiveClusters(&c, kern, &cfg) == cudaSuccess && c >= 1) n = c;
    }
    max_units[dev] = n;
  }
  // persistent: at most one CTA per SM (the shared memory allows no second), units round robin
  const int units = PAIR ? (a.nblk + 1) / 2 : a.nblk;
  int grid_units = (dev >= 0 && dev < 64) ? max_units[dev] : (PAIR ? sm_count() / 2 : sm_count());
  if (units < grid_units) grid_units = units;
  if (grid_units < 1) grid_units = 1;
  cfg.gridDim = dim3((unsigned)((PAIR ? 2 : 1) * grid_units), 1, 1);
  cfg.attrs = PAIR ? attr : attr + 1;
  cfg.numAttrs = PAIR ? 2 : 1;
  return cuda_status(cudaLaunchKernelEx(&cfg, kern, tx, tw, a));
}

// CTA pairs when the tiles outnumber the SMs (each CTA then takes several tiles and the
// weight's L2 stream is what the pair halves); with one wave of tiles or less the single-CTA
// kernel starts every tile at once and measured slightly faster.
static bool route_pairs(int nblk) { return nblk > sm_count(); }

template <int NPW, int NQ>
static int launch_route_np(const CUtensorMap& tx, const CUtensorMap& tw, const RouteArgs& a, cudaStream_t st) {
  return route_pairs(a.nblk) ? launch_route_t<NPW, NQ, true>(tx, tw, a, st)
                             : launch_route_t<NPW, NQ, false>(tx, tw, a, st);
}

int launch_route_scan(const moe_dims_t& d, void* ws, cudaStream_t st) {
  const WsLayout L = ws_layout(d);
  ScanArgs sa{};
  sa.counts_blk = ws_ptr<int32_t>(ws, L.counts_blk);
  sa.tot = ws_ptr<int32_t>(ws, L.hdr + kHdrTotOffset);
  sa.bases = ws_ptr<int32_t>(ws, L.bases);
  sa.counts = ws_ptr<int32_t>(ws, L.counts);
  sa.offsets = ws_ptr<int32_t>(ws, L.offsets);
  sa.ppart = ws_ptr<float>(ws, L.ppart);
  sa.hist = ws_ptr<int32_t>(ws, L.hist);
  sa.lsq = ws_ptr<float>(ws, L.lsq);
  sa.auxp = ws_ptr<double>(ws, L.auxp);
  sa.N = d.N;
  sa.K = d.K;
  sa.nblk = L.nblk;
  sa.nparts = L.nparts;
  sa.ncols = router_rows(d);
  sa.hcols = hist_cols(d);
  return launch_pdl(scan_kernel, dim3(d.N + L.nparts), dim3(kScanThreads), 0, st, sa);
}

int launch_router_split(const moe_dims_t& d, const float* w_router, uint16_t* w3, cudaStream_t st, void* ws) {
  const int npw = (w3 != nullptr) ? route_npw(d) : 0;  // no weight: only the header is cleared
  const long long work = (long long)npw * (d.d / 8);
  long long grid = (work + 255) / 256;
  if (grid > (long long)sm_count() * 8) grid = (long long)sm_count() * 8;
  if (grid < 1) grid = 1;
  uint32_t* hdr = (ws != nullptr) ? ws_ptr<uint32_t>(ws, ws_layout(d).hdr) : nullptr;
  const int nclear = (int)(kHdrClearBytes / sizeof(uint32_t));
  return launch_pdl(router_split_kernel, dim3((unsigned)grid), dim3(256), 0, st, w_router, w3, router_rows(d), npw,
                    d.d, hdr, nclear);
}

int launch_route(const moe_dims_t& d, const uint16_t* x, const float* w_router, const float* bias,
                 const float* tok_null_bias, float* logits_out, int32_t* topk_idx, float* topk_gate,
                 int32_t* n_real, void* ws, cudaStream_t st, const uint16_t* w_split) {
  if (route_fp32_cores(d))
    return launch_route_fp32(d, x, w_router, bias, tok_null_bias, logits_out, topk_idx, topk_gate, n_real,
                             ws, st);
  const WsLayout L = ws_layout(d);
  RouteArgs a{};
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
  a.srctok = ws_ptr<int32_t>(ws, L.srctok);
  a.nsrc = ws_ptr<int32_t>(ws, L.hdr + kHdrSrcOffset);
  a.limit_ns = kWaitLimitNs;
  a.T = d.T;
  a.d = d.d;
  a.N = d.N;
  a.M = d.M;
  a.K = d.K;
  a.nblk = L.nblk;
  a.ncols = router_rows(d);
  // the split router weight: prepared once by the caller (moe_prepare_router), or split
  // here into the workspace for this call; the same launch clears the workspace header (with
  // a prepared weight that is all it does, in one block); then tensor maps over x and it
  const int npw = route_npw(d);
  const uint16_t* w3 = w_split;
  {
    uint16_t* w3c = (w3 == nullptr) ? ws_ptr<uint16_t>(ws, L.wprep) : nullptr;
    const int r = launch_router_split(d, w_router, w3c, st, ws);
    if (r != MOE_OK) return r;
    if (w3 == nullptr) w3 = w3c;
  }
  // the weight's box: all 3 npw rows, or half of them for each CTA of a pair
  const uint32_t wbox = (uint32_t)(route_pairs(L.nblk) ? 3 * npw / 2 : 3 * npw);
  CUtensorMap tx, tw;
  if (!make_tmap_bf16(&tx, x, (uint64_t)d.T, (uint64_t)d.d, kRouteTokens) ||
      !make_tmap_bf16(&tw, w3, (uint64_t)3 * npw, (uint64_t)d.d, wbox))
    return MOE_ERR_CUDA;
  int r;
  switch (npw) {
    case 16: r = launch_route_np<16, 4>(tx, tw, a, st); break;
    case 32: r = launch_route_np<32, 8>(tx, tw, a, st); break;
    case 48: r = launch_route_np<48, 12>(tx, tw, a, st); break;
    case 64: r = launch_route_np<64, 16>(tx, tw, a, st); break;
    default:  // 80 rows: without copy/constant experts the candidates are the reals, columns < 64
      r = (pp_experts(d) == 0) ? launch_route_np<80, 16>(tx, tw, a, st) : launch_route_np<80, 20>(tx, tw, a, st);
      break;
  }
  if (r != MOE_OK) return r;
  return launch_route_scan(d, ws, st);
}

}  // namespace moe
