// moe_expert_ffn: the routed experts and the shared expert as two persistent
// grouped GEMMs on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// Kilian et al., "Improving MoE Compute Efficiency by Composing Weight and Data
// Sparsity" (review page, section 三 / 实现): after null slots are cut from the
// expert-sorted list, the same grouped matmul runs on the real rows only; the
// layer is y = E_shared(x) + sum g_i E_i(x) (核心公式). Each expert is SwiGLU:
//   GEMM 1: h  = bf16(silu(A W_g^T) * (A W_u^T))   (gate and up in one tile)
//   GEMM 2: ys = bf16(h W_d^T)
// Group e < N covers rows [offsets[e], offsets[e+1]) of xs/h/ys, read on the
// device (no host synchronisation on the data-dependent row counts); group N
// is the shared expert over all T rows of x.
//
// Kernel: one CTA per SM, 6 warps. Warp 0 issues TMA loads (128B-swizzled
// K-major tiles of 128 x 64 for A and BN x 64 for B) into a 4-stage mbarrier
// ring; warp 1 owns TMEM (2 x BN fp32 columns, double-buffered accumulators)
// and issues tcgen05.mma (M=128, N=BN, K=16) from a single thread, releasing
// smem stages with tcgen05.commit; warps 2-5 drain TMEM with tcgen05.ld, apply
// the epilogue, stage bf16 rows in shared memory and store them with
// coalesced, row-masked 16-byte stores (a tile may run past its expert's last
// row; those rows are computed but never stored). Tiles are handed out
// round-robin (all tiles of a GEMM have the same cost). Every wait is bounded.
//
// Combine folded into the down GEMM (COMBINE): the shared expert's tiles come after every
// routed tile in the tile order, so their epilogue can finish the layer: y[t] =
// bf16(shared[t]) + sum over the token's slots, in rank order, of g * ys[slot_row] (fp32,
// one rounding; the same arithmetic as moe_combine, so y is bit-identical). Each routed
// tile's epilogue publishes its stored rows with a release increment of a counter in the
// workspace; before its first shared tile a CTA's epilogue waits (bounded) until the
// counter holds every routed tile. The grid is persistent (one CTA per SM, at most one
// per SM) and each CTA takes its tiles in increasing order, so the CTA that owns a routed
// tile never waits before finishing it: the wait cannot deadlock while the grid is
// resident. The last CTA to exit resets the counters for the next launch.
//
// Row gather (gate/up with a token permutation): instead of reading routed rows
// from a gathered copy xs, the producer warp copies them from x with 16-byte
// cp.async loads (4 rows per pass, 8 lanes per row) straight into the
// 128B-swizzled tile a 2-D TMA load would write; each lane's copies signal the
// stage's full barrier on completion (cp.async.mbarrier.arrive.noinc) and the
// MMA thread fences them into the async proxy before issuing. Rows past the
// expert's end read token 0 and are never stored. Dispatch then writes no row
// copies at all.
#include "moe_internal.cuh"

#include <cudaTypedefs.h>
#include <mutex>

namespace moe {

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kStages = 4;
constexpr int kGemmThreads = 192;
constexpr int kStgRow = 64 * 2 + 16;  // staging row: 64 bf16 + 16 B pad

struct GemmArgs {
  const int32_t* offsets;  // [N+1]
  const int32_t* perm;     // token of each routed row, or null (routed A read from xs)
  const uint16_t* x;       // [T, ld_x]: the rows perm refers to
  int ld_x;
  int N, T;
  int kb_r, kb_s;          // 64-wide k-blocks per tile: routed, shared
  int nt_r, nt_s;          // n-tiles per group: routed, shared
  int brows_r;             // B rows per routed expert
  long long rows_cap;      // rows of the routed A/out buffers
  uint16_t* out_r;
  int ld_r;
  uint16_t* out_s;
  int ld_s;
  uint32_t* status;
  unsigned long long limit_ns;
  int has_shared;
  uint16_t* zout_r;        // SAVEZ: gate/up pre-activations [rows_cap, 2F] (packed column order)
  int ldz_r;
  uint16_t* zout_s;        // SAVEZ: the shared expert's [T, 2F_shared]
  int ldz_s;
  // COMBINE: the shared tiles' epilogue writes y from the shared expert's output and the
  // token's slots (source of slot k: slot_row >= 0 a row of out_r = ys; else, with MoE++
  // experts, topk_idx tells a copy expert (row of cx) or constant expert j (row j of cv))
  const int32_t* slot_row;  // [T, K]
  const float* gate;        // [T, K]
  const int32_t* topk_idx;  // [T, K] (read only when C + V > 0)
  const uint16_t* cx;       // [T, d] the layer input (copy experts)
  const uint16_t* cv;       // [V, d] constant experts' vectors
  uint16_t* y;              // [T, d]
  int K, NM, C, V;
  uint32_t* tiles_done;     // routed tiles whose rows are stored (workspace header)
  uint32_t* cta_exits;      // CTAs that have exited (the last resets both counters)
};

template <int BN>
struct GemmSmem {
  static constexpr int A_BYTES = kBM * kBK * 2;
  static constexpr int B_BYTES = BN * kBK * 2;
  static constexpr size_t off_a = 0;
  static constexpr size_t off_b = off_a + (size_t)kStages * A_BYTES;
  static constexpr size_t off_stg = off_b + (size_t)kStages * B_BYTES;
  static constexpr size_t off_bar = off_stg + (size_t)kBM * kStgRow;
  static constexpr int n_bar = 2 * kStages + 5;  // full, empty, tfull[2], tempty[2], drain
  static constexpr size_t off_misc = off_bar + 8 * n_bar;
  static constexpr size_t off_tab = off_misc + 16;
  static constexpr size_t off_perm = off_tab + sizeof(int) * 3 * (kMaxN + 2);  // int [128]: tokens of a tile
  static constexpr size_t end = off_perm + sizeof(int) * kBM;
  static constexpr size_t bytes = end + 1024;  // slack for 1024-byte alignment
};

struct TileInfo {
  int g, arow, mvalid, brow, nkb, col0;
};

__device__ __forceinline__ void fma8(float (&acc)[8], float g, const uint4& v) {
  acc[0] = fmaf(g, bf16lo(v.x), acc[0]); acc[1] = fmaf(g, bf16hi(v.x), acc[1]);
  acc[2] = fmaf(g, bf16lo(v.y), acc[2]); acc[3] = fmaf(g, bf16hi(v.y), acc[3]);
  acc[4] = fmaf(g, bf16lo(v.z), acc[4]); acc[5] = fmaf(g, bf16hi(v.z), acc[5]);
  acc[6] = fmaf(g, bf16lo(v.w), acc[6]); acc[7] = fmaf(g, bf16hi(v.w), acc[7]);
}

// Combine in a shared tile (COMBINE), one thread per tile row (its TMEM lane), the token
// t = arow + row. combine_sources: the token's slots in rank order, compacted to the ones
// with an output (a row of ys, written by this launch's routed tiles; x for a copy expert;
// a constant vector), coded as in moe_combine (>= 0 ys row, -2 x row, -3 - j constant j),
// into this thread's own entries of src/gw. combine_chunk: 64 columns of the row: the
// shared expert's bf16 values plus the sources' in rank order, fp32, one rounding.
__device__ __forceinline__ int combine_sources(const GemmArgs& a, int t, int* src, float* gw) {
  const int K = a.K;
  int n = 0;
  for (int k = 0; k < K; ++k) {
    int r = __ldg(a.slot_row + (size_t)t * K + k);
    const float g = __ldg(a.gate + (size_t)t * K + k);
    if (r >= a.rows_cap) {
      atomicOr(a.status, kStatusBounds);
      r = -1;
    }
    if (r < 0 && a.C + a.V > 0) {
      const int id = __ldg(a.topk_idx + (size_t)t * K + k) - a.NM;  // among copy/constant experts
      if (id >= 0 && id < a.C) r = -2;
      else if (id >= a.C && id < a.C + a.V) r = -3 - (id - a.C);
    }
    if (r != -1) {
      src[n] = r;
      gw[n] = g;
      ++n;
    }
  }
  return n;
}

__device__ __forceinline__ const uint4* combine_src_ptr(const GemmArgs& a, int code, int t, int col) {
  const uint16_t* p = (code >= 0) ? a.out_r + (size_t)code * a.ld_r
                      : (code == -2) ? a.cx + (size_t)t * a.ld_s
                                     : a.cv + (size_t)(-3 - code) * a.ld_s;
  return reinterpret_cast<const uint4*>(p + col);
}

__device__ __forceinline__ void combine_chunk(const GemmArgs& a, const uint32_t (&sh)[64], int t, int col, int n,
                                              const int* src, const float* gw) {
  float acc[64];
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const uint32_t p = pack_bf16x2(__uint_as_float(sh[2 * j]), __uint_as_float(sh[2 * j + 1]));
    acc[2 * j] = bf16lo(p);
    acc[2 * j + 1] = bf16hi(p);
  }
  // two sources per pass: all their 16-byte pieces are loaded before either is added
#pragma unroll 1
  for (int i = 0; i < n; i += 2) {
    const bool two = i + 1 < n;
    uint4 v0[8], v1[8];
    const uint4* p0 = combine_src_ptr(a, src[i], t, col);
#pragma unroll
    for (int j = 0; j < 8; ++j) v0[j] = __ldcg(p0 + j);
    if (two) {
      const uint4* p1 = combine_src_ptr(a, src[i + 1], t, col);
#pragma unroll
      for (int j = 0; j < 8; ++j) v1[j] = __ldcg(p1 + j);
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      float (&c8)[8] = *reinterpret_cast<float(*)[8]>(acc + 8 * j);
      fma8(c8, gw[i], v0[j]);
    }
    if (two) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float (&c8)[8] = *reinterpret_cast<float(*)[8]>(acc + 8 * j);
        fma8(c8, gw[i + 1], v1[j]);
      }
    }
  }
  uint4* dst = reinterpret_cast<uint4*>(a.y + (size_t)t * a.ld_s + col);
#pragma unroll
  for (int j = 0; j < 8; ++j)
    dst[j] = make_uint4(pack_bf16x2(acc[8 * j + 0], acc[8 * j + 1]), pack_bf16x2(acc[8 * j + 2], acc[8 * j + 3]),
                        pack_bf16x2(acc[8 * j + 4], acc[8 * j + 5]), pack_bf16x2(acc[8 * j + 6], acc[8 * j + 7]));
}

template <int BN, bool SWIGLU, bool GATHER, bool SAVEZ = false, bool COMBINE = false>
__global__ void __launch_bounds__(kGemmThreads, 1)
grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA_r, const __grid_constant__ CUtensorMap tmB_r,
                    const __grid_constant__ CUtensorMap tmA_s, const __grid_constant__ CUtensorMap tmB_s,
                    const GemmArgs a) {
  pdl_wait_then_release();
  using SM = GemmSmem<BN>;
  constexpr int OUTC = SWIGLU ? BN / 2 : BN;  // output columns per tile
  constexpr int NCHUNK = OUTC / 64;
  constexpr uint32_t TMEM_COLS = 2 * BN;
  constexpr uint32_t IDESC = idesc_bf16_f32(kBM, BN);
  constexpr uint32_t TX_BYTES = SM::A_BYTES + SM::B_BYTES;

  extern __shared__ unsigned char smem_raw[];
  unsigned char* base =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sA = base + SM::off_a;
  unsigned char* sB = base + SM::off_b;
  unsigned char* stg = base + SM::off_stg;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + SM::off_bar);
  volatile int* misc = reinterpret_cast<volatile int*>(base + SM::off_misc);  // [0] tmem, [1] abort
  int* s_tstart = reinterpret_cast<int*>(base + SM::off_tab);  // [N+2]
  int* s_row0 = s_tstart + (kMaxN + 2);                       // [N+1]
  int* s_m = s_row0 + (kMaxN + 2);                            // [N+1]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int N = a.N;
  auto full_bar = [&](int s) { return smem_u32(bars + s); };
  auto empty_bar = [&](int s) { return smem_u32(bars + kStages + s); };
  auto tfull_bar = [&](int s) { return smem_u32(bars + 2 * kStages + s); };
  auto tempty_bar = [&](int s) { return smem_u32(bars + 2 * kStages + 2 + s); };
  const uint32_t drain_bar = smem_u32(bars + 2 * kStages + 4);
  volatile int* abort_flag = misc + 1;

  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA_r);
    prefetch_tmap(&tmB_r);
    if (a.has_shared) {
      prefetch_tmap(&tmA_s);
      prefetch_tmap(&tmB_s);
    }
    for (int s = 0; s < kStages; ++s) {
      // producer lane 0's expect_tx arrival (+ with row gathers, 32 copy-completion arrivals)
      mbar_init(full_bar(s), GATHER ? 1 + 32 : 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(tfull_bar(s), 1);
      mbar_init(tempty_bar(s), 128);
    }
    mbar_init(drain_bar, 1);
    misc[1] = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(const_cast<int*>(misc)), TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 2 && lane == 0) {
    // Per-group tile table from the device-resident offsets.
    int acc = 0;
    int prev = 0;
    bool bad = false;
    for (int g = 0; g <= N; ++g) {
      int m, row0, nt;
      if (g < N) {
        const int o0 = a.offsets[g], o1 = a.offsets[g + 1];
        if (o0 != prev || o1 < o0 || (long long)o1 > a.rows_cap) bad = true;
        prev = o1;
        m = bad ? 0 : o1 - o0;
        row0 = o0;
        nt = a.nt_r;
      } else {
        m = a.has_shared ? a.T : 0;
        row0 = 0;
        nt = a.nt_s;
      }
      s_tstart[g] = acc;
      s_row0[g] = row0;
      s_m[g] = m;
      acc += ((m + kBM - 1) / kBM) * nt;
    }
    s_tstart[N + 1] = acc;
    if (bad) atomicOr(a.status, kStatusBounds);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = (uint32_t)misc[0];
  const int total = s_tstart[N + 1];

  auto decode = [&](int tile) {
    TileInfo ti;
    int lo = 0, hi = N;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_tstart[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    ti.g = lo;
    const int nt = (lo < N) ? a.nt_r : a.nt_s;
    const int local = tile - s_tstart[lo];
    const int mt = local / nt;
    const int ntile = local - mt * nt;
    ti.arow = s_row0[lo] + mt * kBM;
    ti.mvalid = min(kBM, s_m[lo] - mt * kBM);
    ti.brow = (lo < N ? lo * a.brows_r : 0) + ntile * BN;
    ti.nkb = (lo < N) ? a.kb_r : a.kb_s;
    ti.col0 = ntile * OUTC;
    return ti;
  };

  if (warp == 0 && !GATHER) {
    if (lane == 0) {
      // ------------------------------ TMA producer
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_par = 0;
      for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
        const TileInfo ti = decode(tile);
        const void* ta = (ti.g < N) ? (const void*)&tmA_r : (const void*)&tmA_s;
        const void* tb = (ti.g < N) ? (const void*)&tmB_r : (const void*)&tmB_s;
        bool ok = true;
        for (int kb = 0; kb < ti.nkb; ++kb) {
          if (!mbar_wait_bounded(empty_bar(stage), phase ^ 1u, a.limit_ns, abort_flag, a.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(full_bar(stage), TX_BYTES);
          tma_load_2d(smem_u32(sA + stage * SM::A_BYTES), ta, full_bar(stage), kb * kBK, ti.arow);
          tma_load_2d(smem_u32(sB + stage * SM::B_BYTES), tb, full_bar(stage), kb * kBK, ti.brow);
          armed |= 1u << stage;
          armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
      }
      if (*abort_flag) {
        // let every issued copy land before the CTA can exit
        for (int s = 0; s < kStages; ++s)
          if (armed & (1u << s))
            (void)mbar_wait_bounded(full_bar(s), (armed_par >> s) & 1u, a.limit_ns, nullptr, a.status);
      }
    }
  } else if (warp == 0) {
    // ------------------------------ producer warp with row gathers: TMA loads (lane 0),
    // routed A rows by cp.async (all lanes)
    int* s_perm = reinterpret_cast<int*>(base + SM::off_perm);
    int stage = 0;
    uint32_t phase = 0;
    uint32_t armed = 0, armed_par = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
      const TileInfo ti = decode(tile);
      const void* ta = (ti.g < N) ? (const void*)&tmA_r : (const void*)&tmA_s;
      const void* tb = (ti.g < N) ? (const void*)&tmB_r : (const void*)&tmB_s;
      const bool gather = ti.g < N;
      if (gather) {
        // the token of each tile row; rows past the expert's end read token 0 (never stored)
        __syncwarp();  // the previous tile's copies have all been issued
#pragma unroll
        for (int j = 0; j < kBM / 32; ++j) {
          const int i = j * 32 + lane;
          s_perm[i] = (i < ti.mvalid) ? __ldg(a.perm + ti.arow + i) : 0;
        }
        __syncwarp();
      }
      bool ok = true;
      for (int kb = 0; kb < ti.nkb; ++kb) {
        int w = 1;
        if (lane == 0) w = mbar_wait_bounded(empty_bar(stage), phase ^ 1u, a.limit_ns, abort_flag, a.status);
        if (!__shfl_sync(0xffffffffu, w, 0)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          mbar_arrive_expect_tx(full_bar(stage), gather ? (uint32_t)SM::B_BYTES : TX_BYTES);
          if (!gather) tma_load_2d(smem_u32(sA + stage * SM::A_BYTES), ta, full_bar(stage), kb * kBK, ti.arow);
          tma_load_2d(smem_u32(sB + stage * SM::B_BYTES), tb, full_bar(stage), kb * kBK, ti.brow);
        }
        if (gather) {
          // 128 rows x 128 B: 4 rows per pass, 8 lanes per row, 16 B per lane, into the
          // 128B-swizzled layout a 2-D TMA load would write (chunk c of row r at c ^ (r & 7))
          const int chunk = lane & 7;
          const uint32_t dst0 = smem_u32(sA + stage * SM::A_BYTES);
          const uint16_t* src0 = a.x + (size_t)kb * kBK + chunk * 8;
#pragma unroll 8
          for (int p = 0; p < kBM / 4; ++p) {
            const int r = p * 4 + (lane >> 3);
            const int tok = s_perm[r];
            cp_async_16(dst0 + (uint32_t)(r * 128 + ((chunk ^ (r & 7)) << 4)), src0 + (size_t)tok * a.ld_x);
          }
        }
        cp_async_mbar_arrive_noinc(full_bar(stage));  // fires when this lane's copies so far have landed
        armed |= 1u << stage;
        armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
    }
    cp_async_wait_all_copies();
    if (lane == 0 && *abort_flag) {
      // let every issued copy land before the CTA can exit
      for (int s = 0; s < kStages; ++s)
        if (armed & (1u << s))
          (void)mbar_wait_bounded(full_bar(s), (armed_par >> s) & 1u, a.limit_ns, nullptr, a.status);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------ MMA issuer (single thread)
      int stage = 0;
      uint32_t phase = 0;
      int li = 0;
      for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++li) {
        const TileInfo ti = decode(tile);
        const int acc = li & 1;
        const uint32_t ap = (uint32_t)(li >> 1) & 1u;
        if (!mbar_wait_bounded(tempty_bar(acc), ap ^ 1u, a.limit_ns, abort_flag, a.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        bool ok = true;
        for (int kb = 0; kb < ti.nkb; ++kb) {
          if (!mbar_wait_bounded(full_bar(stage), phase, a.limit_ns, abort_flag, a.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if constexpr (GATHER) fence_proxy_async_shared();  // gathered rows -> async proxy (tensor cores)
          const uint64_t adesc = smem_desc_sw128(smem_u32(sA + stage * SM::A_BYTES));
          const uint64_t bdesc = smem_desc_sw128(smem_u32(sB + stage * SM::B_BYTES));
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k) {
            // +32 bytes along K inside the 128-byte swizzle atom = +2 in the address field
            tc_mma_f16(d_tmem, adesc + (uint64_t)(2 * k), bdesc + (uint64_t)(2 * k), IDESC,
                       (kb | k) != 0 ? 1u : 0u);
          }
          tc_commit(empty_bar(stage));
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(tfull_bar(acc));
      }
      // all MMAs issued by this thread have completed once the drain barrier fires
      tc_commit(drain_bar);
      (void)mbar_wait_bounded(drain_bar, 0, a.limit_ns, nullptr, a.status);
    }
  } else {
    // ------------------------------ epilogue warpgroup (warps 2..5)
    const int q = warp & 3;             // TMEM lane quarter this warp may access
    const int row = q * 32 + lane;      // tile row held by this thread
    const int etid = (warp - 2) * 32 + lane;
    bool routed_done = false;
    int li = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++li) {
      const TileInfo ti = decode(tile);
      const int acc = li & 1;
      const uint32_t ap = (uint32_t)(li >> 1) & 1u;
      if (!mbar_wait_bounded(tfull_bar(acc), ap, a.limit_ns, abort_flag, a.status)) break;
      const bool comb = COMBINE && ti.g == N;
      if constexpr (COMBINE) {
        if (comb && !routed_done) {
          // every routed tile's ys rows must be stored before a shared tile combines them
          int ok = 1;
          if (etid == 0)
            ok = counter_wait_bounded(a.tiles_done, (uint32_t)s_tstart[N], a.limit_ns, abort_flag, a.status);
          if (!named_bar_and(1, 128, ok != 0)) break;
          routed_done = true;
        }
      }
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
      if constexpr (COMBINE && !SWIGLU) {
        if (comb) {
          // thread-per-row combine: no staging; the staging rows hold each thread's own
          // compacted slot list instead (16 sources x 8 B per row fits in a 144-byte row)
          int* src = reinterpret_cast<int*>(stg + row * kStgRow);
          float* gw = reinterpret_cast<float*>(stg + row * kStgRow + 64);
          const int t = ti.arow + row;
          const bool live = row < ti.mvalid;
          const int n = live ? combine_sources(a, t, src, gw) : 0;
#pragma unroll 1
          for (int c = 0; c < NCHUNK; ++c) {
            uint32_t r[64];
#pragma unroll
            for (int g16 = 0; g16 < 4; ++g16) {
              uint32_t (&r16)[16] = *reinterpret_cast<uint32_t(*)[16]>(r + 16 * g16);
              tmem_ld16(tb + (uint32_t)(c * 64 + g16 * 16), r16);
            }
            tmem_ld_wait();
            if (c == NCHUNK - 1) {
              tc_fence_before();
              mbar_arrive(tempty_bar(acc));  // TMEM buffer free for the next-but-one tile
            }
            if (live) combine_chunk(a, r, t, ti.col0 + c * 64, n, src, gw);
          }
          continue;
        }
      }
      uint16_t* out = (ti.g < N) ? a.out_r : a.out_s;
      const int ld = (ti.g < N) ? a.ld_r : a.ld_s;
#pragma unroll 1
      for (int c = 0; c < NCHUNK; ++c) {
#pragma unroll
        for (int g16 = 0; g16 < 4; ++g16) {
          uint32_t packed[8];
          if constexpr (SWIGLU) {
            uint32_t gr[16], ur[16];
            tmem_ld16(tb + (uint32_t)(c * 128 + g16 * 16), gr);
            tmem_ld16(tb + (uint32_t)(c * 128 + 64 + g16 * 16), ur);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float g0 = __uint_as_float(gr[2 * j]), g1 = __uint_as_float(gr[2 * j + 1]);
              const float u0 = __uint_as_float(ur[2 * j]), u1 = __uint_as_float(ur[2 * j + 1]);
              const float h0 = __fdividef(g0, 1.f + __expf(-g0)) * u0;
              const float h1 = __fdividef(g1, 1.f + __expf(-g1)) * u1;
              packed[j] = pack_bf16x2(h0, h1);
            }
            if constexpr (SAVEZ) {
              // training: keep the pre-activations (bf16, packed order) for the backward pass
              if (row < ti.mvalid) {
                uint16_t* zo = (ti.g < N) ? a.zout_r : a.zout_s;
                const int ldz = (ti.g < N) ? a.ldz_r : a.ldz_s;
                uint16_t* zrow = zo + (size_t)(ti.arow + row) * ldz + 2 * ti.col0 + c * 128 + g16 * 16;
                uint4* zg = reinterpret_cast<uint4*>(zrow);
                uint4* zu = reinterpret_cast<uint4*>(zrow + 64);
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                  zg[q] = make_uint4(pack_bf16x2(__uint_as_float(gr[8 * q + 0]), __uint_as_float(gr[8 * q + 1])),
                                     pack_bf16x2(__uint_as_float(gr[8 * q + 2]), __uint_as_float(gr[8 * q + 3])),
                                     pack_bf16x2(__uint_as_float(gr[8 * q + 4]), __uint_as_float(gr[8 * q + 5])),
                                     pack_bf16x2(__uint_as_float(gr[8 * q + 6]), __uint_as_float(gr[8 * q + 7])));
                  zu[q] = make_uint4(pack_bf16x2(__uint_as_float(ur[8 * q + 0]), __uint_as_float(ur[8 * q + 1])),
                                     pack_bf16x2(__uint_as_float(ur[8 * q + 2]), __uint_as_float(ur[8 * q + 3])),
                                     pack_bf16x2(__uint_as_float(ur[8 * q + 4]), __uint_as_float(ur[8 * q + 5])),
                                     pack_bf16x2(__uint_as_float(ur[8 * q + 6]), __uint_as_float(ur[8 * q + 7])));
                }
              }
            }
          } else {
            uint32_t r[16];
            tmem_ld16(tb + (uint32_t)(c * 64 + g16 * 16), r);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 8; ++j)
              packed[j] = pack_bf16x2(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1]));
          }
          uint4* dst = reinterpret_cast<uint4*>(stg + row * kStgRow + g16 * 32);
          dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
          dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
        }
        if (c == NCHUNK - 1) {
          tc_fence_before();
          mbar_arrive(tempty_bar(acc));  // TMEM buffer free for the next-but-one tile
        }
        named_bar_sync(1, 128);
#pragma unroll
        for (int it = 0; it < 8; ++it) {
          const int idx = it * 128 + etid;
          const int r = idx >> 3, ch = idx & 7;
          if (r < ti.mvalid) {
            const uint4 v = *reinterpret_cast<const uint4*>(stg + r * kStgRow + ch * 16);
            *reinterpret_cast<uint4*>(out + (size_t)(ti.arow + r) * ld + ti.col0 + c * 64 + ch * 8) = v;
          }
        }
        if (COMBINE && c == NCHUNK - 1) __threadfence();  // this routed tile's rows, before the release
        named_bar_sync(1, 128);
      }
      if (COMBINE && etid == 0) red_add_release_gpu(a.tiles_done, 1u);
    }
  }

  if constexpr (COMBINE) {
    // the last CTA out resets the counters for the next launch (every CTA has passed its
    // waits by the time it exits)
    __syncthreads();
    if (threadIdx.x == 0) {
      __threadfence();
      if (atomicAdd(a.cta_exits, 1u) == gridDim.x - 1) {
        atomicExch(a.tiles_done, 0u);
        atomicExch(a.cta_exits, 0u);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------------------
// Gate/up packing: 64-row panels, gate panel then the matching up panel.
__global__ void pack_gate_up_kernel(const uint16_t* __restrict__ wg, const uint16_t* __restrict__ wu,
                                    uint16_t* __restrict__ out, int groups, int F, int d) {
  pdl_wait_then_release();
  const int lane = threadIdx.x & 31;
  const long long rows = (long long)groups * 2 * F;
  const int nch = d >> 3;
  for (long long pr = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); pr < rows;
       pr += (long long)gridDim.x * (blockDim.x >> 5)) {
    const long long e = pr / (2 * F);
    const int r = (int)(pr - e * 2 * F);
    const int pair = r >> 7, within = r & 127;
    const uint16_t* src = (within < 64 ? wg : wu) + ((size_t)e * F + pair * 64 + (within & 63)) * d;
    uint4* dst = reinterpret_cast<uint4*>(out + (size_t)pr * d);
    for (int c = lane; c < nch; c += 32) dst[c] = __ldg(reinterpret_cast<const uint4*>(src) + c);
  }
}

int launch_pack_gate_up(const moe_dims_t& d, const uint16_t* w_gate, const uint16_t* w_up,
                        const uint16_t* ws_gate, const uint16_t* ws_up, uint16_t* gate_up,
                        uint16_t* sgate_up, cudaStream_t st) {
  const int grid = sm_count() * 8;
  if (gate_up) {
    int r = launch_pdl(pack_gate_up_kernel, dim3(grid), dim3(256), 0, st, w_gate, w_up, gate_up, d.N, d.F, d.d);
    if (r != MOE_OK) return r;
  }
  if (sgate_up) {
    int r = launch_pdl(pack_gate_up_kernel, dim3(grid), dim3(256), 0, st, ws_gate, ws_up, sgate_up, 1, d.F_shared,
                       d.d);
    if (r != MOE_OK) return r;
  }
  return MOE_OK;
}

// ---------------------------------------------------------------------------------------
// Host side: tensor maps and launches.
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D bf16 tensor [rows, cols] (cols contiguous), box = box_rows x 64 cols, 128B swizzle.
bool make_tmap_bf16(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int BN, bool SWIGLU, bool GATHER, bool SAVEZ = false, bool COMBINE = false>
static int launch_gemm(const CUtensorMap& ar, const CUtensorMap& br, const CUtensorMap& as_,
                       const CUtensorMap& bs, const GemmArgs& a, long long max_tiles, cudaStream_t st) {
  using SM = GemmSmem<BN>;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(grouped_gemm_kernel<BN, SWIGLU, GATHER, SAVEZ, COMBINE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SM::bytes);
    if (e != cudaSuccess) return cuda_status(e);
    attr_set[dev] = true;
  }
  // persistent: at most one CTA per SM (the shared memory allows no second), so with COMBINE
  // every CTA is resident at once and the shared tiles' wait on the routed tiles cannot stall
  long long grid = sm_count();
  if (max_tiles < grid) grid = max_tiles;
  if (grid < 1) grid = 1;
  return launch_pdl(grouped_gemm_kernel<BN, SWIGLU, GATHER, SAVEZ, COMBINE>, dim3((unsigned)grid),
                    dim3(kGemmThreads), SM::bytes, st, ar, br, as_, bs, a);
}

struct FfnPlan {
  int BN1, BN2;
  long long max1, max2;
  GemmArgs g1, g2;
};

// rows_cap: rows of the routed A/output buffers; by default the layer's R_cap = T K (the
// expert-parallel calls pass the rows a rank received instead)
static FfnPlan plan_ffn(const moe_dims_t& d, const int32_t* offsets, void* ws, long long rows_cap = -1) {
  const WsLayout L = ws_layout(d);
  FfnPlan p{};
  const long long rcap = rows_cap >= 0 ? rows_cap : (long long)d.T * d.K;
  p.BN1 = (d.F % 128 == 0 && d.F_shared % 128 == 0) ? 256 : 128;
  p.BN2 = (d.d % 256 == 0) ? 256 : 128;
  const long long mtiles_r = rcap / kBM + d.N;  // sum_e ceil(m_e/128) <= R/128 + N
  const long long mtiles_s = (d.T + kBM - 1) / kBM;
  GemmArgs& g1 = p.g1;
  g1.offsets = offsets;
  g1.N = d.N;
  g1.T = d.T;
  g1.kb_r = d.d / kBK;
  g1.kb_s = d.d / kBK;
  g1.nt_r = 2 * d.F / p.BN1;
  g1.nt_s = 2 * d.F_shared / p.BN1;
  g1.brows_r = 2 * d.F;
  g1.rows_cap = rcap;
  g1.ld_r = d.F;
  g1.ld_s = d.F_shared;
  g1.status = ws_ptr<uint32_t>(ws, L.hdr);
  g1.limit_ns = kWaitLimitNs;
  g1.has_shared = 1;
  p.max1 = mtiles_r * g1.nt_r + mtiles_s * g1.nt_s;
  GemmArgs& g2 = p.g2;
  g2 = g1;
  g2.kb_r = d.F / kBK;
  g2.kb_s = d.F_shared / kBK;
  g2.nt_r = d.d / p.BN2;
  g2.nt_s = d.d / p.BN2;
  g2.brows_r = d.d;
  g2.ld_r = d.d;
  g2.ld_s = d.d;
  p.max2 = mtiles_r * g2.nt_r + mtiles_s * g2.nt_s;
  return p;
}

int launch_gate_up(const moe_dims_t& d, const uint16_t* xs, const uint16_t* x, const int32_t* offsets,
                   const uint16_t* gate_up, const uint16_t* sgate_up, uint16_t* h, uint16_t* h_shared,
                   void* ws, cudaStream_t st) {
  return launch_gate_up_perm(d, xs, x, offsets, nullptr, gate_up, sgate_up, h, h_shared, ws, st);
}

int launch_gate_up_perm(const moe_dims_t& d, const uint16_t* xs, const uint16_t* x, const int32_t* offsets,
                        const int32_t* perm, const uint16_t* gate_up, const uint16_t* sgate_up, uint16_t* h,
                        uint16_t* h_shared, void* ws, cudaStream_t st) {
  if (perm == nullptr && ffn_pair_gate_up_ok(d))
    return launch_gate_up_pair(d, xs, x, offsets, gate_up, sgate_up, h, h_shared, ws, st);
  FfnPlan p = plan_ffn(d, offsets, ws);
  const long long rcap = (long long)d.T * d.K;
  CUtensorMap ar, br, as_, bs;
  // routed A: the gathered copy xs (128-row boxes), or x itself for row gathers (1-row boxes)
  // (with perm the routed rows are gathered by cp.async and the map is not used)
  const bool ok_a = make_tmap_bf16(&ar, perm ? x : xs, perm ? (uint64_t)d.T : (uint64_t)rcap, d.d, kBM);
  if (!(ok_a &&
        make_tmap_bf16(&br, gate_up, (uint64_t)d.N * 2 * d.F, d.d, p.BN1) &&
        make_tmap_bf16(&as_, x, d.T, d.d, kBM) &&
        make_tmap_bf16(&bs, sgate_up, (uint64_t)2 * d.F_shared, d.d, p.BN1)))
    return MOE_ERR_CUDA;
  p.g1.out_r = h;
  p.g1.out_s = h_shared;
  p.g1.perm = perm;
  p.g1.x = x;
  p.g1.ld_x = d.d;
  if (perm)
    return (p.BN1 == 256) ? launch_gemm<256, true, true>(ar, br, as_, bs, p.g1, p.max1, st)
                          : launch_gemm<128, true, true>(ar, br, as_, bs, p.g1, p.max1, st);
  return (p.BN1 == 256) ? launch_gemm<256, true, false>(ar, br, as_, bs, p.g1, p.max1, st)
                        : launch_gemm<128, true, false>(ar, br, as_, bs, p.g1, p.max1, st);
}

// gate/up with the pre-activations also written (training): z [rows_cap, 2F] and zs [T, 2F_shared]
// in the packed column order, bf16. Copy path (xs) only.
int launch_gate_up_save(const moe_dims_t& d, const uint16_t* xs, const uint16_t* x, const int32_t* offsets,
                        const uint16_t* gate_up, const uint16_t* sgate_up, uint16_t* h, uint16_t* h_shared,
                        uint16_t* z, uint16_t* zs, void* ws, cudaStream_t st) {
  FfnPlan p = plan_ffn(d, offsets, ws);
  const long long rcap = (long long)d.T * d.K;
  CUtensorMap ar, br, as_, bs;
  if (!(make_tmap_bf16(&ar, xs, (uint64_t)rcap, d.d, kBM) &&
        make_tmap_bf16(&br, gate_up, (uint64_t)d.N * 2 * d.F, d.d, p.BN1) &&
        make_tmap_bf16(&as_, x, d.T, d.d, kBM) &&
        make_tmap_bf16(&bs, sgate_up, (uint64_t)2 * d.F_shared, d.d, p.BN1)))
    return MOE_ERR_CUDA;
  p.g1.out_r = h;
  p.g1.out_s = h_shared;
  p.g1.x = x;
  p.g1.ld_x = d.d;
  p.g1.zout_r = z;
  p.g1.ldz_r = 2 * d.F;
  p.g1.zout_s = zs;
  p.g1.ldz_s = 2 * d.F_shared;
  return (p.BN1 == 256) ? launch_gemm<256, true, false, true>(ar, br, as_, bs, p.g1, p.max1, st)
                        : launch_gemm<128, true, false, true>(ar, br, as_, bs, p.g1, p.max1, st);
}

int launch_down(const moe_dims_t& d, const int32_t* offsets, const uint16_t* h, const uint16_t* h_shared,
                const uint16_t* w_down, const uint16_t* sdown, uint16_t* ys, uint16_t* shared_out, void* ws,
                cudaStream_t st) {
  if (ffn_pair_down_ok(d)) return launch_down_pair(d, offsets, h, h_shared, w_down, sdown, ys, shared_out, ws, st);
  FfnPlan p = plan_ffn(d, offsets, ws);
  const long long rcap = (long long)d.T * d.K;
  CUtensorMap ar, br, as_, bs;
  if (!(make_tmap_bf16(&ar, h, rcap, d.F, kBM) &&
        make_tmap_bf16(&br, w_down, (uint64_t)d.N * d.d, d.F, p.BN2) &&
        make_tmap_bf16(&as_, h_shared, d.T, d.F_shared, kBM) &&
        make_tmap_bf16(&bs, sdown, d.d, d.F_shared, p.BN2)))
    return MOE_ERR_CUDA;
  p.g2.out_r = ys;
  p.g2.out_s = shared_out;
  return (p.BN2 == 256) ? launch_gemm<256, false, false>(ar, br, as_, bs, p.g2, p.max2, st)
                        : launch_gemm<128, false, false>(ar, br, as_, bs, p.g2, p.max2, st);
}

// The down GEMM with the combine folded into its shared-expert tiles: ys for the routed
// rows, and y = bf16(shared) + sum_k g ys (and the MoE++ copy / constant terms) for every
// token; shared_out is not written. Single-CTA tiles (the CTA-pair flag does not apply).
int launch_down_combine(const moe_dims_t& d, const int32_t* offsets, const uint16_t* h, const uint16_t* h_shared,
                        const uint16_t* w_down, const uint16_t* sdown, uint16_t* ys, const float* topk_gate,
                        const int32_t* slot_row, const int32_t* topk_idx, const uint16_t* x,
                        const uint16_t* const_vectors, uint16_t* y, void* ws, cudaStream_t st) {
  FfnPlan p = plan_ffn(d, offsets, ws);
  const long long rcap = (long long)d.T * d.K;
  CUtensorMap ar, br, as_, bs;
  if (!(make_tmap_bf16(&ar, h, rcap, d.F, kBM) &&
        make_tmap_bf16(&br, w_down, (uint64_t)d.N * d.d, d.F, p.BN2) &&
        make_tmap_bf16(&as_, h_shared, d.T, d.F_shared, kBM) &&
        make_tmap_bf16(&bs, sdown, d.d, d.F_shared, p.BN2)))
    return MOE_ERR_CUDA;
  const WsLayout L = ws_layout(d);
  GemmArgs& g = p.g2;
  g.out_r = ys;
  g.out_s = nullptr;
  g.slot_row = slot_row;
  g.gate = topk_gate;
  g.topk_idx = topk_idx;
  g.cx = x;
  g.cv = const_vectors;
  g.y = y;
  g.K = d.K;
  g.NM = d.N + d.M;
  g.C = d.C;
  g.V = d.V;
  g.tiles_done = ws_ptr<uint32_t>(ws, L.hdr + kHdrCombineOffset);
  g.cta_exits = g.tiles_done + 1;
  return (p.BN2 == 256) ? launch_gemm<256, false, false, false, true>(ar, br, as_, bs, g, p.max2, st)
                        : launch_gemm<128, false, false, false, true>(ar, br, as_, bs, g, p.max2, st);
}

// Expert parallelism: the grouped GEMMs of one rank's expert shard over the rows it
// received (rows_cap of them at most, expert-contiguous by offsets[0..N]), with the shared
// expert over this rank's own T tokens. Single-CTA tiles.
int launch_gate_up_rows(const moe_dims_t& d, long long rows_cap, const uint16_t* xs, const uint16_t* x,
                        const int32_t* offsets, const uint16_t* gate_up, const uint16_t* sgate_up, uint16_t* h,
                        uint16_t* h_shared, void* ws, cudaStream_t st) {
  FfnPlan p = plan_ffn(d, offsets, ws, rows_cap);
  CUtensorMap ar, br, as_, bs;
  if (!(make_tmap_bf16(&ar, xs, (uint64_t)rows_cap, d.d, kBM) &&
        make_tmap_bf16(&br, gate_up, (uint64_t)d.N * 2 * d.F, d.d, p.BN1)))
    return MOE_ERR_CUDA;
  if (d.T == 0) {  // a rank without tokens of its own: routed rows only (the shared maps go unused)
    p.g1.has_shared = 0;
    as_ = ar;
    bs = br;
  } else if (!(make_tmap_bf16(&as_, x, d.T, d.d, kBM) &&
               make_tmap_bf16(&bs, sgate_up, (uint64_t)2 * d.F_shared, d.d, p.BN1))) {
    return MOE_ERR_CUDA;
  }
  p.g1.out_r = h;
  p.g1.out_s = h_shared;
  p.g1.x = x;
  p.g1.ld_x = d.d;
  return (p.BN1 == 256) ? launch_gemm<256, true, false>(ar, br, as_, bs, p.g1, p.max1, st)
                        : launch_gemm<128, true, false>(ar, br, as_, bs, p.g1, p.max1, st);
}

int launch_down_rows(const moe_dims_t& d, long long rows_cap, const int32_t* offsets, const uint16_t* h,
                     const uint16_t* h_shared, const uint16_t* w_down, const uint16_t* sdown, uint16_t* ys,
                     uint16_t* shared_out, void* ws, cudaStream_t st) {
  FfnPlan p = plan_ffn(d, offsets, ws, rows_cap);
  CUtensorMap ar, br, as_, bs;
  if (!(make_tmap_bf16(&ar, h, (uint64_t)rows_cap, d.F, kBM) &&
        make_tmap_bf16(&br, w_down, (uint64_t)d.N * d.d, d.F, p.BN2)))
    return MOE_ERR_CUDA;
  if (d.T == 0) {
    p.g2.has_shared = 0;
    as_ = ar;
    bs = br;
  } else if (!(make_tmap_bf16(&as_, h_shared, d.T, d.F_shared, kBM) &&
               make_tmap_bf16(&bs, sdown, d.d, d.F_shared, p.BN2))) {
    return MOE_ERR_CUDA;
  }
  p.g2.out_r = ys;
  p.g2.out_s = shared_out;
  return (p.BN2 == 256) ? launch_gemm<256, false, false>(ar, br, as_, bs, p.g2, p.max2, st)
                        : launch_gemm<128, false, false>(ar, br, as_, bs, p.g2, p.max2, st);
}

int launch_expert_ffn(const moe_dims_t& d, const uint16_t* xs, const uint16_t* x, const int32_t* offsets,
                      const uint16_t* gate_up, const uint16_t* w_down, const uint16_t* sgate_up,
                      const uint16_t* sdown, uint16_t* h, uint16_t* h_shared, uint16_t* ys,
                      uint16_t* shared_out, void* ws, cudaStream_t st) {
  const int r = launch_gate_up(d, xs, x, offsets, gate_up, sgate_up, h, h_shared, ws, st);
  if (r != MOE_OK) return r;
  return launch_down(d, offsets, h, h_shared, w_down, sdown, ys, shared_out, ws, st);
}

}  // namespace moe
