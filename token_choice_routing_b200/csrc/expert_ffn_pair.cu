// moe_expert_ffn on CTA pairs: the two grouped GEMMs of expert_ffn.cu with one
// tcgen05 MMA shared by the two CTAs of a cluster.
//
// Kilian et al., "Improving MoE Compute Efficiency by Composing Weight and Data
// Sparsity" (review page, section 三 / 实现): after null slots are cut from the
// expert-sorted list, the same grouped matmul runs on the real rows only. Each
// expert is SwiGLU:
//   GEMM 1: h  = bf16(silu(A W_g^T) * (A W_u^T))   (gate and up in one tile)
//   GEMM 2: ys = bf16(h W_d^T)
//
// A pair tile is 256 token rows x 256 output columns. Each CTA loads its own
// 128 token rows and half (128) of the 256 weight rows per k-block: 32 KB, where
// a 1-CTA 128 x 256 tile loads 48 KB for the same MMA work. The operand stream
// out of L2 is what limits the 1-CTA kernel (extra L2 traffic slows it down in
// proportion), so a third less of it per flop is the point of the pair. The
// leader CTA issues tcgen05.mma.cta_group::2 (M=256, N=256, K=16); each CTA's
// TMEM then holds its own 128 token rows x all 256 columns, the same
// accumulator layout as the 1-CTA kernel, and the epilogue is the same: SwiGLU
// or a plain conversion, bf16 rows staged in shared memory, coalesced stores
// masked at the expert's last row (rows past it are computed, never stored).
//
// Selected with MOE_FLAG_FFN_CTA_PAIR. Measured on the 16K-token workloads it
// is not faster than the 1-CTA kernel: both are held by the L2 output rate,
// which the 1-CTA kernel's concurrent reads of the same tiles already share,
// and pair tiles round each expert up to 256 rows.
//
// Roles (192 threads per CTA, both CTAs): warp 0 lane 0 issues TMA loads into
// its own CTA's 6-stage ring and counts them on the leader's full barrier;
// warp 1 allocates TMEM (cta_group::2, 2 x 256 columns) and, in the leader only,
// one thread issues the MMAs and commits to both CTAs' barriers; warps 2-5 of
// each CTA drain their TMEM. Every wait is bounded.
#include "moe_internal.cuh"

namespace moe {

constexpr int kQM = 128;             // token rows per CTA (256 per pair)
constexpr int kQN = 256;             // output columns per tile (128 weight rows from each CTA)
constexpr int kQK = 64;              // k per stage (one 128-byte swizzle row of bf16)
constexpr int kQStages = 6;
constexpr int kQThreads = 192;
constexpr int kQStgRow = 64 * 2 + 16;  // staging row: 64 bf16 + 16 B pad

struct PairArgs {
  const int32_t* offsets;  // [N+1]
  int N, T;
  int kb_r, kb_s;          // k-blocks per tile: routed, shared
  int nt_r, nt_s;          // 256-column tiles per group: routed, shared
  int brows_r;             // weight rows per routed expert
  long long rows_cap;      // rows of the routed A/out buffers
  uint16_t* out_r;
  int ld_r;
  uint16_t* out_s;
  int ld_s;
  uint32_t* status;
  unsigned long long limit_ns;
  int has_shared;
};

struct PairSmem {
  static constexpr int A_BYTES = kQM * kQK * 2;        // 16 KB: this CTA's 128 token rows
  static constexpr int B_BYTES = (kQN / 2) * kQK * 2;  // 16 KB: this CTA's 128 weight rows
  static constexpr size_t off_a = 0;
  static constexpr size_t off_b = off_a + (size_t)kQStages * A_BYTES;
  static constexpr size_t off_stg = off_b + (size_t)kQStages * B_BYTES;
  static constexpr size_t off_bar = off_stg + (size_t)kQM * kQStgRow;
  static constexpr int n_bar = 2 * kQStages + 5;  // full, empty, tfull[2], tempty[2], drain
  static constexpr size_t off_misc = off_bar + 8 * n_bar;
  static constexpr size_t off_tab = off_misc + 16;
  static constexpr size_t end = off_tab + sizeof(int) * 3 * (kMaxN + 2);
  static constexpr size_t bytes = end + 1024;  // slack for 1024-byte alignment
};

struct PairTile {
  int g, arow, mvalid, brow, nkb, col0;
};

template <bool SWIGLU>
__global__ void __launch_bounds__(kQThreads, 1)
    grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA_r, const __grid_constant__ CUtensorMap tmB_r,
                             const __grid_constant__ CUtensorMap tmA_s, const __grid_constant__ CUtensorMap tmB_s,
                             const PairArgs a) {
  pdl_wait_then_release();
  using SM = PairSmem;
  constexpr int OUTC = SWIGLU ? kQN / 2 : kQN;  // output columns per tile
  constexpr int NCHUNK = OUTC / 64;
  constexpr uint32_t TMEM_COLS = 2 * kQN;                  // two 256-column accumulators
  constexpr uint32_t IDESC = idesc_bf16_f32(2 * kQM, kQN);  // M = 256 over the pair
  constexpr uint32_t TX_BYTES = 2 * (SM::A_BYTES + SM::B_BYTES);  // both CTAs' loads of one stage

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
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  auto full_bar = [&](int s) { return smem_u32(bars + s); };
  auto empty_bar = [&](int s) { return smem_u32(bars + kQStages + s); };
  auto tfull_bar = [&](int s) { return smem_u32(bars + 2 * kQStages + s); };
  auto tempty_bar = [&](int s) { return smem_u32(bars + 2 * kQStages + 2 + s); };
  const uint32_t drain_bar = smem_u32(bars + 2 * kQStages + 4);
  volatile int* abort_flag = misc + 1;

  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA_r);
    prefetch_tmap(&tmB_r);
    if (a.has_shared) {
      prefetch_tmap(&tmA_s);
      prefetch_tmap(&tmB_s);
    }
    for (int s = 0; s < kQStages; ++s) {
      mbar_init(full_bar(s), 1);   // leader: its own expect_tx arrival, plus both CTAs' bytes
      mbar_init(empty_bar(s), 1);  // one commit from the leader's MMA thread
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(tfull_bar(s), 1);
      mbar_init(tempty_bar(s), 2 * 128);  // leader: every epilogue thread of both CTAs
    }
    mbar_init(drain_bar, 1);
    misc[1] = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(const_cast<int*>(misc)), TMEM_COLS);
    tmem_relinquish_pair();
  }
  if (warp == 2 && lane == 0) {
    // Per-group tile table from the device-resident offsets (both CTAs build the same one).
    int acc = 0, prev = 0;
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
      acc += ((m + 2 * kQM - 1) / (2 * kQM)) * nt;
    }
    s_tstart[N + 1] = acc;
    if (bad && leader) atomicOr(a.status, kStatusBounds);
  }
  tc_fence_before();
  cluster_sync_all();  // barriers of both CTAs initialised, TMEM allocated, tables built
  tc_fence_after();
  const uint32_t tmem_base = (uint32_t)misc[0];
  const int total = s_tstart[N + 1];
  const int pair = (int)cluster_id_x(), npairs = (int)cluster_count_x();

  auto decode = [&](int tile) {
    PairTile ti;
    int lo = 0, hi = N;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_tstart[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    ti.g = lo;
    const int nt = (lo < N) ? a.nt_r : a.nt_s;
    const int local = tile - s_tstart[lo];
    const int pmt = local / nt;
    const int ntile = local - pmt * nt;
    ti.arow = s_row0[lo] + pmt * 2 * kQM + (int)rank * kQM;
    ti.mvalid = min(kQM, s_m[lo] - pmt * 2 * kQM - (int)rank * kQM);  // <= 0: no row of this CTA
    ti.brow = (lo < N ? lo * a.brows_r : 0) + ntile * kQN + (int)rank * (kQN / 2);
    ti.nkb = (lo < N) ? a.kb_r : a.kb_s;
    ti.col0 = ntile * OUTC;
    return ti;
  };

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------ TMA producer (both CTAs)
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_par = 0;
      for (int tile = pair; tile < total; tile += npairs) {
        const PairTile ti = decode(tile);
        const void* ta = (ti.g < N) ? (const void*)&tmA_r : (const void*)&tmA_s;
        const void* tb = (ti.g < N) ? (const void*)&tmB_r : (const void*)&tmB_s;
        bool ok = true;
        for (int kb = 0; kb < ti.nkb; ++kb) {
          if (!mbar_wait_bounded(empty_bar(stage), phase ^ 1u, a.limit_ns, abort_flag, a.status)) {
            ok = false;
            break;
          }
          const uint32_t fb = map_to_rank(full_bar(stage), 0);
          if (leader) mbar_arrive_expect_tx(full_bar(stage), TX_BYTES);
          tma_load_2d_pair(smem_u32(sA + stage * SM::A_BYTES), ta, fb, kb * kQK, ti.arow);
          tma_load_2d_pair(smem_u32(sB + stage * SM::B_BYTES), tb, fb, kb * kQK, ti.brow);
          armed |= 1u << stage;
          armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
          if (++stage == kQStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
      }
      if (*abort_flag && leader) {
        // the leader's full barriers count both CTAs' copies: let armed stages land
        for (int s = 0; s < kQStages; ++s)
          if (armed & (1u << s))
            (void)mbar_wait_bounded(full_bar(s), (armed_par >> s) & 1u, a.limit_ns, nullptr, a.status);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ------------------------------ MMA issuer (leader CTA, one thread)
      int stage = 0;
      uint32_t phase = 0;
      int li = 0;
      for (int tile = pair; tile < total; tile += npairs, ++li) {
        const PairTile ti = decode(tile);
        const int acc = li & 1;
        const uint32_t ap = (uint32_t)(li >> 1) & 1u;
        if (!mbar_wait_bounded(tempty_bar(acc), ap ^ 1u, a.limit_ns, abort_flag, a.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * kQN);
        bool ok = true;
        for (int kb = 0; kb < ti.nkb; ++kb) {
          if (!mbar_wait_bounded(full_bar(stage), phase, a.limit_ns, abort_flag, a.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t adesc = smem_desc_sw128(smem_u32(sA + stage * SM::A_BYTES));
          const uint64_t bdesc = smem_desc_sw128(smem_u32(sB + stage * SM::B_BYTES));
#pragma unroll
          for (int k = 0; k < kQK / 16; ++k) {
            // +32 bytes along K inside the 128-byte swizzle atom = +2 in the address field
            tc_mma_pair(d_tmem, adesc + (uint64_t)(2 * k), bdesc + (uint64_t)(2 * k), IDESC,
                        (kb | k) != 0 ? 1u : 0u);
          }
          // free this stage in both CTAs
          tc_commit_pair(empty_bar(stage));
          tc_commit_pair(map_to_rank(empty_bar(stage), 1));
          if (++stage == kQStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit_pair(tfull_bar(acc));
        tc_commit_pair(map_to_rank(tfull_bar(acc), 1));
      }
      // all MMAs issued by this thread have completed once the drain barrier fires
      tc_commit_pair(drain_bar);
      (void)mbar_wait_bounded(drain_bar, 0, a.limit_ns, nullptr, a.status);
    }
  } else {
    // ------------------------------ epilogue warpgroup (warps 2..5 of each CTA)
    const int q = warp & 3;         // TMEM lane quarter this warp may access
    const int row = q * 32 + lane;  // tile row held by this thread
    const int etid = (warp - 2) * 32 + lane;
    const uint32_t tempty_leader = map_to_rank(tempty_bar(0), 0);
    int li = 0;
    for (int tile = pair; tile < total; tile += npairs, ++li) {
      const PairTile ti = decode(tile);
      const int acc = li & 1;
      const uint32_t ap = (uint32_t)(li >> 1) & 1u;
      if (!mbar_wait_bounded(tfull_bar(acc), ap, a.limit_ns, abort_flag, a.status)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * kQN);
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
          } else {
            uint32_t r[16];
            tmem_ld16(tb + (uint32_t)(c * 64 + g16 * 16), r);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 8; ++j)
              packed[j] = pack_bf16x2(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1]));
          }
          uint4* dst = reinterpret_cast<uint4*>(stg + row * kQStgRow + g16 * 32);
          dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
          dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
        }
        if (c == NCHUNK - 1) {
          // this CTA's half of the accumulator is drained: let the leader reuse it
          tc_fence_before();
          mbar_arrive_cluster(tempty_leader + 8u * (uint32_t)acc);
        }
        named_bar_sync(1, 128);
#pragma unroll
        for (int it = 0; it < 8; ++it) {
          const int idx = it * 128 + etid;
          const int r = idx >> 3, ch = idx & 7;
          if (r < ti.mvalid) {
            const uint4 v = *reinterpret_cast<const uint4*>(stg + r * kQStgRow + ch * 16);
            *reinterpret_cast<uint4*>(out + (size_t)(ti.arow + r) * ld + ti.col0 + c * 64 + ch * 8) = v;
          }
        }
        named_bar_sync(1, 128);
      }
    }
  }

  tc_fence_before();
  cluster_sync_all();  // the leader's MMAs read both CTAs' shared memory: nobody leaves early
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------------------
// Host side.
template <bool SWIGLU>
static int launch_pair(const CUtensorMap& ar, const CUtensorMap& br, const CUtensorMap& as_, const CUtensorMap& bs,
                       const PairArgs& a, long long max_tiles, cudaStream_t st) {
  static int clusters[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  auto kern = grouped_gemm_pair_kernel<SWIGLU>;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // see launch_pdl
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.blockDim = dim3(kQThreads, 1, 1);
  cfg.dynamicSmemBytes = PairSmem::bytes;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;  // the occupancy query below sees the cluster shape only
  if (dev >= 0 && dev < 64 && clusters[dev] == 0) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)PairSmem::bytes);
    if (e != cudaSuccess) return cuda_status(e);
    int n = 0;
    cfg.gridDim = dim3(2 * (sm_count() / 2), 1, 1);
    e = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
    if (e != cudaSuccess || n < 1) n = sm_count() / 2;
    clusters[dev] = n;
  }
  long long np = (dev >= 0 && dev < 64) ? clusters[dev] : sm_count() / 2;
  if (max_tiles < np) np = max_tiles;
  if (np < 1) np = 1;
  cfg.gridDim = dim3((unsigned)(2 * np), 1, 1);
  cfg.numAttrs = 2;
  return cuda_status(cudaLaunchKernelEx(&cfg, kern, ar, br, as_, bs, a));
}

static PairArgs pair_common(const moe_dims_t& d, const int32_t* offsets, void* ws) {
  const WsLayout L = ws_layout(d);
  PairArgs a{};
  a.offsets = offsets;
  a.N = d.N;
  a.T = d.T;
  a.rows_cap = (long long)d.T * d.K;
  a.status = ws_ptr<uint32_t>(ws, L.hdr);
  a.limit_ns = kWaitLimitNs;
  a.has_shared = 1;
  return a;
}

bool ffn_pair_gate_up_ok(const moe_dims_t& d) {
  return (d.flags & MOE_FLAG_FFN_CTA_PAIR) && d.F % 128 == 0 && d.F_shared % 128 == 0;
}
bool ffn_pair_down_ok(const moe_dims_t& d) { return (d.flags & MOE_FLAG_FFN_CTA_PAIR) && d.d % 256 == 0; }

int launch_gate_up_pair(const moe_dims_t& d, const uint16_t* xs, const uint16_t* x, const int32_t* offsets,
                        const uint16_t* gate_up, const uint16_t* sgate_up, uint16_t* h, uint16_t* h_shared,
                        void* ws, cudaStream_t st) {
  const long long rcap = (long long)d.T * d.K;
  CUtensorMap ar, br, as_, bs;
  if (!(make_tmap_bf16(&ar, xs, rcap, d.d, kQM) &&
        make_tmap_bf16(&br, gate_up, (uint64_t)d.N * 2 * d.F, d.d, kQN / 2) &&
        make_tmap_bf16(&as_, x, d.T, d.d, kQM) &&
        make_tmap_bf16(&bs, sgate_up, (uint64_t)2 * d.F_shared, d.d, kQN / 2)))
    return MOE_ERR_CUDA;
  PairArgs a = pair_common(d, offsets, ws);
  a.kb_r = a.kb_s = d.d / kQK;
  a.nt_r = 2 * d.F / kQN;
  a.nt_s = 2 * d.F_shared / kQN;
  a.brows_r = 2 * d.F;
  a.out_r = h;
  a.ld_r = d.F;
  a.out_s = h_shared;
  a.ld_s = d.F_shared;
  // sum_e ceil(m_e / 256) <= R_cap / 256 + N pair row-tiles for the routed experts
  const long long max_tiles = (rcap / (2 * kQM) + d.N) * a.nt_r + ((d.T + 2 * kQM - 1) / (2 * kQM)) * a.nt_s;
  return launch_pair<true>(ar, br, as_, bs, a, max_tiles, st);
}

int launch_down_pair(const moe_dims_t& d, const int32_t* offsets, const uint16_t* h, const uint16_t* h_shared,
                     const uint16_t* w_down, const uint16_t* sdown, uint16_t* ys, uint16_t* shared_out, void* ws,
                     cudaStream_t st) {
  const long long rcap = (long long)d.T * d.K;
  CUtensorMap ar, br, as_, bs;
  if (!(make_tmap_bf16(&ar, h, rcap, d.F, kQM) &&
        make_tmap_bf16(&br, w_down, (uint64_t)d.N * d.d, d.F, kQN / 2) &&
        make_tmap_bf16(&as_, h_shared, d.T, d.F_shared, kQM) &&
        make_tmap_bf16(&bs, sdown, d.d, d.F_shared, kQN / 2)))
    return MOE_ERR_CUDA;
  PairArgs a = pair_common(d, offsets, ws);
  a.kb_r = d.F / kQK;
  a.kb_s = d.F_shared / kQK;
  a.nt_r = a.nt_s = d.d / kQN;
  a.brows_r = d.d;
  a.out_r = ys;
  a.ld_r = d.d;
  a.out_s = shared_out;
  a.ld_s = d.d;
  const long long max_tiles = (rcap / (2 * kQM) + d.N) * a.nt_r + ((d.T + 2 * kQM - 1) / (2 * kQM)) * a.nt_s;
  return launch_pair<false>(ar, br, as_, bs, a, max_tiles, st);
}

}  // namespace moe
