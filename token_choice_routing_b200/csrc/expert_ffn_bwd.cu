// Backward pass of the expert FFNs: data and weight gradients of the routed experts and
// the shared expert as persistent grouped GEMMs on the 5th-generation tensor cores.
//
// Kilian et al., "Improving MoE Compute Efficiency by Composing Weight and Data Sparsity"
// (review page, section 四 实验结果 / 训练配置: the layer is trained end to end; section
// 三 / 实现: the grouped matmul runs on the real rows only). With the SwiGLU expert
// E(x) = W_d (silu(W_g x) * (W_u x)), its gate/up pre-activations [a | b] = x W_gu^T
// (recomputed from the forward's rows) and h = silu(a) * b, the gradients of one expert's
// rows xs are
//   dh    = dys W_d                     (dgrad of the down projection)
//   dz    = [da | db] from dh, a, b     (SwiGLU backward, in the recomputing GEMM's epilogue)
//   dW_d  = dys^T h                     (wgrad, K = the expert's rows)
//   dxs   = dz W_gu                     (dgrad of gate/up)
//   dW_gu = dz^T xs                     (wgrad, K = the expert's rows)
// so, as in the forward, nothing is computed for null slots.
//
// One kernel template serves the three GEMM shapes:
//   kDgradPlain: C[row, n] = sum_k A[row, k] B[k, n]. A (activation rows, K contiguous) is
//     K-major; B is the weight in its natural layout [K, n] (n contiguous) and is read
//     MN-major: 64 x 64 TMA boxes, one per 64 output columns.
//   kPreactSwiglu: the forward's gate/up product z = A W_gu^T (both K-major) recomputed
//     into TMEM in fp32; its epilogue reads the matching tile of dh (TMA) and writes the
//     SwiGLU derivative dz = [da | db] in the packed column order, with 8 epilogue warps.
//   kWgrad: C[m, n] = sum_r A[r, m] B[r, n] over the rows r of one expert: both operands are
//     activation rows read MN-major. The last k-block of an expert reads rows of the next
//     expert (or unwritten rows); those rows are zeroed in shared memory before the MMA.
// The MN-major tiles are what a 64 x 64 TMA box with the 128-byte swizzle writes: 64
// k-rows of 128 bytes, so the matrix descriptor has 8-row groups 1024 B apart (SBO) and
// 64-element strips one box (8 KB) apart (LBO), and the instruction descriptor marks the
// operand as transposed (MN-major). Warp roles and the pipeline follow the forward kernel:
// warp 0 TMA producer, warp 1 TMEM owner and single-thread MMA issuer, warps 2-5 epilogue.
// The shared expert's weight gradients have K = T rows: they are split into chunks
// written as fp32 partials and summed in a fixed order by a second kernel.
#include "moe_internal.cuh"

namespace moe {

namespace bwd {

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kStages = 4;
constexpr int kStgRow = 64 * 2 + 16;
constexpr int kBox = 64 * 64 * 2;  // one 64 x 64 bf16 box (8 KB)

enum Mode { kDgradPlain = 0, kPreactSwiglu = 1, kWgrad = 2 };

template <int MODE>
struct Threads {
  static constexpr int epi = (MODE == kPreactSwiglu) ? 256 : 128;  // epilogue threads
  static constexpr int total = 64 + epi;
};

struct Args {
  const int32_t* offsets;  // [N+1]
  int N, T;
  int kb_r, kb_s;          // dgrad: k-blocks per tile (routed, shared)
  int nt_r, nt_s;          // n-tiles per group
  int mt_r, mt_s;          // wgrad: m-tiles per group (output rows / 128)
  int kdim_r;              // dgrad: B rows per routed expert (its K)
  int nsplit, chunk_kb;    // wgrad: shared-expert K chunks and k-blocks per chunk
  long long rows_cap;
  uint16_t* out_r;         // dgrad: [rows_cap, ld_r]; wgrad: [N, Mout, ld_r] (or the gate half)
  int ld_r;
  uint16_t* out_s;         // dgrad: [T, ld_s]; wgrad: [Mout_s, ld_s] (or the gate half)
  int ld_s;
  uint16_t* out_r2;        // wgrad of packed gate/up: destination of the up rows (else null)
  uint16_t* out_s2;
  float* part_s;           // wgrad, nsplit > 1: fp32 partials [nsplit, Mout_s, ld_s]
  int part_only;           // wgrad: the shared group always writes fp32 partials
  int kb_x, xrp;           // dgrad: extra k-blocks of the shared group (router term), term width
  uint32_t* status;
  unsigned long long limit_ns;
  int has_shared;
};

template <int BN, int MODE>
struct Smem {
  static constexpr int A_BYTES = kBM * kBK * 2;
  static constexpr int B_BYTES = BN * kBK * 2;
  static constexpr int Z_BYTES = (MODE == kPreactSwiglu) ? kBM * BN : 0;  // dh tile: 128 x BN/2 bf16
  static constexpr int STG_BYTES = (MODE == kPreactSwiglu) ? 0 : kBM * kStgRow;
  static constexpr size_t off_a = 0;
  static constexpr size_t off_b = off_a + (size_t)kStages * A_BYTES;
  static constexpr size_t off_z = off_b + (size_t)kStages * B_BYTES;
  static constexpr size_t off_stg = off_z + Z_BYTES;
  static constexpr size_t off_bar = off_stg + STG_BYTES;
  static constexpr int n_bar = 2 * kStages + 6;  // full, empty, tfull[2], tempty[2], drain, z
  static constexpr size_t off_misc = off_bar + 8 * n_bar;
  static constexpr size_t off_tab = off_misc + 16;
  static constexpr size_t end = off_tab + sizeof(int) * 3 * (kMaxN + 2);
  static constexpr size_t bytes = end + 1024;
  static_assert(bytes <= 232448, "shared memory per CTA");
};

struct Tile {
  int g;      // group (expert, N = shared)
  int row0;   // dgrad: first row of the tile; wgrad: first K row of the expert/chunk
  int mvalid; // dgrad: valid rows of the tile
  int krows;  // wgrad: K rows of the expert/chunk
  int nkb;    // k-blocks
  int mt, nt; // m-tile (wgrad) and n-tile
  int chunk;  // wgrad shared: K chunk
  int brow;   // dgrad: first B row of the group (e * kdim)
};

// MN-major tile descriptor: 64-element strips lbo bytes apart, 8-row k groups 1024 B apart.
__device__ __forceinline__ uint64_t desc_mn_sw128(uint32_t saddr, uint32_t lbo_bytes) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)(lbo_bytes >> 4) << 16) | ((uint64_t)64 << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor with the transpose (MN-major) bits of A (bit 15) and B (bit 16).
__host__ __device__ constexpr uint32_t idesc_t(int M, int N, bool a_mn, bool b_mn) {
  return idesc_bf16_f32(M, N) | (a_mn ? (1u << 15) : 0u) | (b_mn ? (1u << 16) : 0u);
}

template <int BN, int MODE>
__global__ void __launch_bounds__(Threads<MODE>::total, 1)
bwd_gemm_kernel(const __grid_constant__ CUtensorMap tmA_r, const __grid_constant__ CUtensorMap tmB_r,
                const __grid_constant__ CUtensorMap tmA_s, const __grid_constant__ CUtensorMap tmB_s,
                const __grid_constant__ CUtensorMap tmZ_r, const __grid_constant__ CUtensorMap tmZ_s,
                const Args a) {
  pdl_wait_then_release();
  using SM = Smem<BN, MODE>;
  constexpr bool WG = (MODE == kWgrad);
  constexpr bool PRE = (MODE == kPreactSwiglu);
  constexpr int EPI = Threads<MODE>::epi;
  constexpr uint32_t TMEM_COLS = 2 * BN < 32 ? 32 : 2 * BN;
  constexpr uint32_t IDESC = idesc_t(kBM, BN, WG, !PRE);
  constexpr uint32_t TX_BYTES = SM::A_BYTES + SM::B_BYTES;
  constexpr int NBOX_B = BN / 64;

  extern __shared__ unsigned char smem_raw[];
  unsigned char* base =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sA = base + SM::off_a;
  unsigned char* sB = base + SM::off_b;
  unsigned char* sZ = base + SM::off_z;
  unsigned char* stg = base + SM::off_stg;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + SM::off_bar);
  volatile int* misc = reinterpret_cast<volatile int*>(base + SM::off_misc);  // [0] tmem, [1] abort
  int* s_tstart = reinterpret_cast<int*>(base + SM::off_tab);
  int* s_row0 = s_tstart + (kMaxN + 2);
  int* s_m = s_row0 + (kMaxN + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int N = a.N;
  auto full_bar = [&](int s) { return smem_u32(bars + s); };
  auto empty_bar = [&](int s) { return smem_u32(bars + kStages + s); };
  auto tfull_bar = [&](int s) { return smem_u32(bars + 2 * kStages + s); };
  auto tempty_bar = [&](int s) { return smem_u32(bars + 2 * kStages + 2 + s); };
  const uint32_t drain_bar = smem_u32(bars + 2 * kStages + 4);
  const uint32_t z_bar = smem_u32(bars + 2 * kStages + 5);
  volatile int* abort_flag = misc + 1;

  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA_r);
    prefetch_tmap(&tmB_r);
    if (a.has_shared) {
      prefetch_tmap(&tmA_s);
      prefetch_tmap(&tmB_s);
    }
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(tfull_bar(s), 1);
      mbar_init(tempty_bar(s), EPI);
    }
    mbar_init(drain_bar, 1);
    mbar_init(z_bar, 1);
    misc[1] = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(const_cast<int*>(misc)), TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 2 && lane == 0) {
    // Per-group tile table from the device-resident offsets.
    int acc = 0, prev = 0;
    bool bad = false;
    if (WG && a.has_shared) {  // shared expert first: its K chunks are the longest tiles
      s_tstart[N] = 0;
      acc = a.nsplit * a.mt_s * a.nt_s;
    }
    for (int g = 0; g <= N; ++g) {
      int m, row0;
      if (g < N) {
        const int o0 = a.offsets[g], o1 = a.offsets[g + 1];
        if (o0 != prev || o1 < o0 || (long long)o1 > a.rows_cap) bad = true;
        prev = o1;
        m = bad ? 0 : o1 - o0;
        row0 = o0;
      } else {
        m = a.has_shared ? a.T : 0;
        row0 = 0;
      }
      s_row0[g] = row0;
      s_m[g] = m;
      if (WG) {
        if (g < N) {
          s_tstart[g] = acc;
          acc += a.mt_r * a.nt_r;
        }
      } else {
        s_tstart[g] = acc;
        acc += ((m + kBM - 1) / kBM) * (g < N ? a.nt_r : a.nt_s);
      }
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
    Tile ti;
    if constexpr (WG) {
      const int nsh = a.has_shared ? a.nsplit * a.mt_s * a.nt_s : 0;
      if (tile < nsh) {
        const int per = a.mt_s * a.nt_s;
        ti.g = N;
        ti.chunk = tile / per;
        const int local = tile - ti.chunk * per;
        ti.mt = local / a.nt_s;
        ti.nt = local - ti.mt * a.nt_s;
        ti.row0 = ti.chunk * a.chunk_kb * kBK;
        ti.krows = max(0, min(a.chunk_kb * kBK, s_m[N] - ti.row0));
      } else {
        const int per = a.mt_r * a.nt_r;
        const int e = (tile - nsh) / per;
        const int local = tile - nsh - e * per;
        ti.g = e;
        ti.chunk = 0;
        ti.mt = local / a.nt_r;
        ti.nt = local - ti.mt * a.nt_r;
        ti.row0 = s_row0[e];
        ti.krows = s_m[e];
      }
      ti.nkb = (ti.krows + kBK - 1) / kBK;
      ti.mvalid = kBM;
      ti.brow = 0;
    } else {
      int lo = 0, hi = N;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_tstart[mid] <= tile) lo = mid; else hi = mid - 1;
      }
      ti.g = lo;
      const int nt = (lo < N) ? a.nt_r : a.nt_s;
      const int local = tile - s_tstart[lo];
      const int mt = local / nt;
      ti.nt = local - mt * nt;
      ti.mt = mt;
      ti.row0 = s_row0[lo] + mt * kBM;
      ti.mvalid = min(kBM, s_m[lo] - mt * kBM);
      ti.krows = 0;
      ti.chunk = 0;
      ti.nkb = (lo < N) ? a.kb_r : a.kb_s + a.kb_x;
      ti.brow = (lo < N) ? lo * a.kdim_r : 0;
    }
    return ti;
  };

  // This CTA's r-th tile: round-robin, so neighbouring CTAs work on neighbouring tiles (the
  // same expert's operands) at the same time. (Dealing weight-gradient tiles largest expert
  // first in snake order measured 40-45% slower: it breaks that L2 sharing.)
  auto tile_at = [&](int r) { return r * (int)gridDim.x + (int)blockIdx.x; };

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------ TMA producer
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_par = 0;
      for (int r = 0;; ++r) {
        const int tile = tile_at(r);
        if (tile >= total) break;
        const Tile ti = decode(tile);
        const void* ta = (ti.g < N) ? (const void*)&tmA_r : (const void*)&tmA_s;
        const void* tb = (ti.g < N) ? (const void*)&tmB_r : (const void*)&tmB_s;
        bool ok = true;
        for (int kb = 0; kb < ti.nkb; ++kb) {
          if (!mbar_wait_bounded(empty_bar(stage), phase ^ 1u, a.limit_ns, abort_flag, a.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(full_bar(stage), TX_BYTES);
          const uint32_t dA = smem_u32(sA + stage * SM::A_BYTES);
          const uint32_t dB = smem_u32(sB + stage * SM::B_BYTES);
          if constexpr (WG) {
            const int kr = ti.row0 + kb * kBK;
            tma_load_2d(dA, ta, full_bar(stage), ti.mt * kBM, kr);
            tma_load_2d(dA + kBox, ta, full_bar(stage), ti.mt * kBM + 64, kr);
#pragma unroll
            for (int j = 0; j < NBOX_B; ++j)
              tma_load_2d(dB + j * kBox, tb, full_bar(stage), ti.nt * BN + 64 * j, kr);
          } else if (PRE) {
            // K-major A and B (the packed gate/up rows of this n-tile), as in the forward
            tma_load_2d(dA, ta, full_bar(stage), kb * kBK, ti.row0);
            tma_load_2d(dB, tb, full_bar(stage), kb * kBK, ti.brow + ti.nt * BN);
          } else if (ti.g == N && kb >= a.kb_s) {
            // router term of the shared group: ds W_r = ds_hi W_hi + ds_hi W_lo + ds_lo W_hi, the
            // two-term splits read from the maps in the pre-activation slots
            const int e = kb - a.kb_s;
            const int njb = a.xrp / kBK;
            const int p = e / njb, jb = e - p * njb;
            const int at = (p == 2) ? 1 : 0, bt = (p == 1) ? 1 : 0;
            tma_load_2d(dA, &tmZ_r, full_bar(stage), at * a.xrp + jb * kBK, ti.row0);
#pragma unroll
            for (int j = 0; j < NBOX_B; ++j)
              tma_load_2d(dB + j * kBox, &tmZ_s, full_bar(stage), ti.nt * BN + 64 * j, bt * a.xrp + jb * kBK);
          } else {
            tma_load_2d(dA, ta, full_bar(stage), kb * kBK, ti.row0);
#pragma unroll
            for (int j = 0; j < NBOX_B; ++j)
              tma_load_2d(dB + j * kBox, tb, full_bar(stage), ti.nt * BN + 64 * j, ti.brow + kb * kBK);
          }
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
        for (int s = 0; s < kStages; ++s)
          if (armed & (1u << s))
            (void)mbar_wait_bounded(full_bar(s), (armed_par >> s) & 1u, a.limit_ns, nullptr, a.status);
      }
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer (lane 0); the whole warp zeroes k-tails (wgrad)
    int stage = 0;
    uint32_t phase = 0;
    int li = 0;
    for (;; ++li) {
      const int tile = tile_at(li);
      if (tile >= total) break;
      const Tile ti = decode(tile);
      const int acc = li & 1;
      const uint32_t ap = (uint32_t)(li >> 1) & 1u;
      int w = 1;
      if (lane == 0) w = mbar_wait_bounded(tempty_bar(acc), ap ^ 1u, a.limit_ns, abort_flag, a.status);
      if (!__shfl_sync(0xffffffffu, w, 0)) break;
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
      bool ok = true;
      for (int kb = 0; kb < ti.nkb; ++kb) {
        int f = 1;
        if (lane == 0) f = mbar_wait_bounded(full_bar(stage), phase, a.limit_ns, abort_flag, a.status);
        if (!__shfl_sync(0xffffffffu, f, 0)) {
          ok = false;
          break;
        }
        int nk16 = kBK / 16;
        if constexpr (WG) {
          const int rem = ti.krows - kb * kBK;
          if (rem < kBK) {
            // rows [rem, 16 * ceil(rem / 16)) of every box belong to another expert (or were
            // never written): zero them in both operands; later 16-row steps are skipped
            nk16 = (rem + 15) >> 4;
            const int z0 = rem, z1 = nk16 * 16;
            const int nrows = z1 - z0;
            const int nbox = 2 + NBOX_B;
            for (int i = lane; i < nbox * nrows * 8; i += 32) {
              const int box = i / (nrows * 8);
              const int rr = (i / 8) % nrows + z0;
              const int ch = i & 7;
              unsigned char* p = (box < 2) ? sA + stage * SM::A_BYTES + box * kBox
                                           : sB + stage * SM::B_BYTES + (box - 2) * kBox;
              *reinterpret_cast<uint4*>(p + rr * 128 + ch * 16) = make_uint4(0u, 0u, 0u, 0u);
            }
            fence_proxy_async_shared();
            __syncwarp();
          }
        }
        if (lane == 0) {
          tc_fence_after();
          const uint32_t aS = smem_u32(sA + stage * SM::A_BYTES);
          const uint32_t bS = smem_u32(sB + stage * SM::B_BYTES);
          for (int k = 0; k < nk16; ++k) {
            uint64_t adesc, bdesc;
            if constexpr (WG) {
              adesc = desc_mn_sw128(aS + (uint32_t)(k * 2048), kBox);
            } else {
              // K-major A: +32 bytes along K inside the 128-byte swizzle atom
              adesc = smem_desc_sw128(aS) + (uint64_t)(2 * k);
            }
            if constexpr (PRE)
              bdesc = smem_desc_sw128(bS) + (uint64_t)(2 * k);
            else
              bdesc = desc_mn_sw128(bS + (uint32_t)(k * 2048), kBox);
            tc_mma_f16(d_tmem, adesc, bdesc, IDESC, (kb | k) != 0 ? 1u : 0u);
          }
          tc_commit(empty_bar(stage));
        }
        __syncwarp();
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      if (lane == 0) tc_commit(tfull_bar(acc));
      __syncwarp();
    }
    if (lane == 0) {
      tc_commit(drain_bar);
      (void)mbar_wait_bounded(drain_bar, 0, a.limit_ns, nullptr, a.status);
    }
    __syncwarp();
  } else {
    // ------------------------------ epilogue warps (2..5, or 2..9 for kPreactSwiglu)
    const int q = warp & 3;              // TMEM lane quarter this warp may access
    const int row = q * 32 + lane;
    const int etid = (warp - 2) * 32 + lane;
    const int ehalf = (warp - 2) >> 2;   // kPreactSwiglu: which half of the tile's columns
    int li = 0;
    int z_inflight = -1;  // (etid 0) tile counter of a dh-tile load not yet waited for
    // dh tile of a tile: rows row0.., dh columns [nt BN/2, (nt+1) BN/2) in 64-column boxes
    auto load_dh = [&](const Tile& t, uint32_t bar) {
      const void* tz = (t.g < N) ? (const void*)&tmZ_r : (const void*)&tmZ_s;
      mbar_arrive_expect_tx(bar, SM::Z_BYTES);
#pragma unroll
      for (int b = 0; b < BN / 128; ++b)
        tma_load_2d(smem_u32(sZ + b * (kBM * 128)), tz, bar, t.nt * (BN / 2) + 64 * b, t.row0);
    };
    if constexpr (PRE) {
      if (etid == 0 && (int)blockIdx.x < total) {
        z_inflight = 0;
        load_dh(decode(blockIdx.x), z_bar);
      }
    }
    for (;; ++li) {
      const int tile = tile_at(li);
      if (tile >= total) break;
      const Tile ti = decode(tile);
      const int acc = li & 1;
      const uint32_t ap = (uint32_t)(li >> 1) & 1u;
      if (!mbar_wait_bounded(tfull_bar(acc), ap, a.limit_ns, abort_flag, a.status)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
      if constexpr (PRE) {
        if (!mbar_wait_bounded(z_bar, (uint32_t)li & 1u, a.limit_ns, abort_flag, a.status)) break;
        z_inflight = -1;
        // z (fp32, TMEM: 64 gate then 64 up columns per panel) and dh (smem) of this row ->
        // da = dh b sigma (1 + a (1 - sigma)), db = dh a sigma, stored as bf16 straight to dz
        uint16_t* out = (ti.g < N) ? a.out_r : a.out_s;
        const int ld = (ti.g < N) ? a.ld_r : a.ld_s;
        const bool live = row < ti.mvalid;
        uint16_t* orow = out + (size_t)(ti.row0 + row) * ld + ti.nt * BN;
#pragma unroll 1
        for (int g = 0; g < BN / 64; ++g) {
          const int f0 = ehalf * (BN / 4) + g * 16;  // first of 16 dh columns in the tile
          const int p = f0 >> 6, within = f0 & 63;
          uint32_t zg[16], zu[16];
          tmem_ld16(tb + (uint32_t)(p * 128 + within), zg);
          tmem_ld16(tb + (uint32_t)(p * 128 + 64 + within), zu);
          tmem_ld_wait();
          uint32_t og[8], ou[8];
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            const int ch = (within >> 3) + half;
            const uint4 hv = *reinterpret_cast<const uint4*>(sZ + p * (kBM * 128) + row * 128 + ((ch ^ (row & 7)) << 4));
            const uint32_t hw[4] = {hv.x, hv.y, hv.z, hv.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              float dav[2], dbv[2];
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const int c = half * 8 + 2 * j + h;
                const float av = __uint_as_float(zg[c]);
                const float bv = __uint_as_float(zu[c]);
                const float dh = h ? bf16hi(hw[j]) : bf16lo(hw[j]);
                const float sg = __fdividef(1.f, 1.f + __expf(-av));
                dbv[h] = dh * av * sg;
                dav[h] = dh * bv * sg * (1.f + av * (1.f - sg));
              }
              og[half * 4 + j] = pack_bf16x2(dav[0], dav[1]);
              ou[half * 4 + j] = pack_bf16x2(dbv[0], dbv[1]);
            }
          }
          if (live) {
            uint4* dg4 = reinterpret_cast<uint4*>(orow + p * 128 + within);
            uint4* du4 = reinterpret_cast<uint4*>(orow + p * 128 + 64 + within);
            dg4[0] = make_uint4(og[0], og[1], og[2], og[3]);
            dg4[1] = make_uint4(og[4], og[5], og[6], og[7]);
            du4[0] = make_uint4(ou[0], ou[1], ou[2], ou[3]);
            du4[1] = make_uint4(ou[4], ou[5], ou[6], ou[7]);
          }
        }
        tc_fence_before();
        mbar_arrive(tempty_bar(acc));
        fence_proxy_async_shared();  // generic reads of the dh tile before the next TMA write
        named_bar_sync(1, EPI);
        if (etid == 0 && tile_at(li + 1) < total) {
          z_inflight = li + 1;
          load_dh(decode(tile_at(li + 1)), z_bar);
        }
      } else {
        // plain bf16 output (dgrad) or weight gradient (wgrad), staged 64 columns at a time
        const bool partial = WG && ti.g == N && (a.nsplit > 1 || a.part_only);
        const bool empty = WG && ti.nkb == 0;
        uint16_t* out;
        int ld;
        size_t rowoff_lo = 0, rowoff_hi = 0;  // wgrad: element offsets of rows 0 and 64
        uint16_t* out_hi = nullptr;
        if constexpr (WG) {
          const bool sh = ti.g == N;
          ld = sh ? a.ld_s : a.ld_r;
          uint16_t* o1 = sh ? a.out_s : a.out_r;
          uint16_t* o2 = sh ? a.out_s2 : a.out_r2;
          const int e = sh ? 0 : ti.g;
          const int mrows = (sh ? a.mt_s : a.mt_r) * kBM;  // packed output rows per group
          if (o2) {  // packed gate/up: tile rows 0..63 are gate rows, 64..127 the up rows
            const size_t half = (size_t)(mrows / 2) * ld;
            out = o1 + e * half;
            out_hi = o2 + e * half;
            rowoff_lo = (size_t)(ti.mt * 64) * ld;
            rowoff_hi = rowoff_lo;
          } else {
            out = o1 + (size_t)e * mrows * ld;
            out_hi = out;
            rowoff_lo = (size_t)(ti.mt * kBM) * ld;
            rowoff_hi = rowoff_lo + (size_t)64 * ld;
          }
        } else {
          out = (ti.g < N) ? a.out_r : a.out_s;
          ld = (ti.g < N) ? a.ld_r : a.ld_s;
        }
        if (partial) {
          // fp32 partial of one K chunk, straight from registers
          float* P = a.part_s + ((size_t)ti.chunk * a.mt_s * kBM + (size_t)ti.mt * kBM + row) * a.ld_s + ti.nt * BN;
#pragma unroll 1
          for (int g16 = 0; g16 < BN / 16; ++g16) {
            uint32_t r[16];
            if (!empty) {
              tmem_ld16(tb + (uint32_t)(g16 * 16), r);
              tmem_ld_wait();
            } else {
#pragma unroll
              for (int j = 0; j < 16; ++j) r[j] = 0u;
            }
            float4* dst = reinterpret_cast<float4*>(P + g16 * 16);
#pragma unroll
            for (int j = 0; j < 4; ++j)
              dst[j] = make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                                   __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3]));
          }
          tc_fence_before();
          mbar_arrive(tempty_bar(acc));
        } else {
#pragma unroll 1
          for (int c = 0; c < BN / 64; ++c) {
#pragma unroll
            for (int g16 = 0; g16 < 4; ++g16) {
              uint32_t r[16];
              if (!empty) {
                tmem_ld16(tb + (uint32_t)(c * 64 + g16 * 16), r);
                tmem_ld_wait();
              } else {
#pragma unroll
                for (int j = 0; j < 16; ++j) r[j] = 0u;
              }
              uint32_t packed[8];
#pragma unroll
              for (int j = 0; j < 8; ++j)
                packed[j] = pack_bf16x2(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1]));
              uint4* dst = reinterpret_cast<uint4*>(stg + row * kStgRow + g16 * 32);
              dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
              dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
            }
            if (c == BN / 64 - 1) {
              tc_fence_before();
              mbar_arrive(tempty_bar(acc));
            }
            named_bar_sync(1, EPI);
#pragma unroll
            for (int it = 0; it < 8; ++it) {
              const int idx = it * 128 + etid;
              const int r = idx >> 3, ch = idx & 7;
              const uint4 v = *reinterpret_cast<const uint4*>(stg + r * kStgRow + ch * 16);
              const int col = ti.nt * BN + c * 64 + ch * 8;
              if constexpr (WG) {
                uint16_t* dst = (r < 64) ? out + rowoff_lo + (size_t)r * ld
                                         : out_hi + rowoff_hi + (size_t)(r - 64) * ld;
                *reinterpret_cast<uint4*>(dst + col) = v;
              } else {
                if (r < ti.mvalid) *reinterpret_cast<uint4*>(out + (size_t)(ti.row0 + r) * ld + col) = v;
              }
            }
            named_bar_sync(1, EPI);
          }
        }
      }
    }
    // after an abort, a pre-activation load still in flight must land before the CTA exits
    if (z_inflight >= 0) (void)mbar_wait_bounded(z_bar, (uint32_t)z_inflight & 1u, a.limit_ns, nullptr, a.status);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// Sum of the shared expert's fp32 K-chunk partials in chunk order, rounded once to bf16.
// With out2 (packed gate/up), row m of the packed matrix goes to the gate (m % 128 < 64) or
// the up half, row (m / 128) * 64 + m % 64.
__global__ void __launch_bounds__(256) split_reduce_kernel(const float* __restrict__ part, int nsplit, int mrows,
                                                           int ncols, uint16_t* __restrict__ out,
                                                           uint16_t* __restrict__ out2) {
  pdl_wait_then_release();
  const long long n8 = (long long)mrows * ncols / 8;
  const size_t stride = (size_t)mrows * ncols;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += (long long)gridDim.x * blockDim.x) {
    const long long e0 = i * 8;
    const int m = (int)(e0 / ncols);
    const int c = (int)(e0 - (long long)m * ncols);
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
    for (int s = 0; s < nsplit; ++s) {
      const float4* p = reinterpret_cast<const float4*>(part + s * stride + e0);
      const float4 v0 = __ldg(p), v1 = __ldg(p + 1);
      acc[0] += v0.x; acc[1] += v0.y; acc[2] += v0.z; acc[3] += v0.w;
      acc[4] += v1.x; acc[5] += v1.y; acc[6] += v1.z; acc[7] += v1.w;
    }
    uint16_t* dst;
    if (out2) {
      const int w = m & 127;
      dst = (w < 64 ? out : out2) + (size_t)((m >> 7) * 64 + (w & 63)) * ncols + c;
    } else {
      dst = out + (size_t)m * ncols + c;
    }
    *reinterpret_cast<uint4*>(dst) = make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                                                pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
  }
}

// ---------------------------------------------------------------------------------------
// Weight gradients on CTA pairs. C[m, n] = sum_r A[r, m] B[r, n] over one expert's rows (or
// one K chunk of the shared expert's T rows), as kWgrad above, with a pair tile of 256
// output rows x 256 columns: one tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 16, both
// operands MN-major) per 16 rows. Each CTA loads its own 128 output rows of A and its half
// (128) of the 256 columns of B per 64-row k-block: 32 KB, against 48 KB for the same work
// on one CTA (a 128 x 256 tile), so a third less operand data crosses into shared memory per
// flop. Each CTA's TMEM holds its 128 output rows x 256 columns, drained by the kWgrad
// epilogue as the 128-row tile 2 p + rank of pair tile p.
// A full k-block's copies (both CTAs') complete on the leader's full barrier, as in the
// forward's pair kernel. The rows of an expert's last k-block past its end (another
// expert's rows, or rows never written) are zeroed before the MMA reads them, in both CTAs:
// that k-block's copies complete on a barrier of the CTA's own, and a ready warp in each CTA
// waits for it and zeroes those rows: the leader's then gives the full barrier its one
// arrival, the other CTA's arrives on the leader's zeroed barrier, and the MMA thread waits
// for both. (Remote arrivals on every k-block, from the producer or a ready warp, measured
// 1.5-2 times slower.)
// Roles (224 threads per CTA): warp 0 lane 0 TMA producer; warp 1 TMEM allocation and, in
// the leader, the single MMA thread; warps 2-5 epilogue; warp 6 ready warp. Every wait is
// bounded.
// Bounded wait with cluster-scope acquire, for a barrier that the other CTA of the pair
// arrives on after writing shared memory the waiter's MMAs read. Returns false (and records
// a timeout in *status) if limit_ns passed or *abort became non-zero meanwhile.
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred P;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 P, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, P;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_bounded_cluster(uint32_t bar, uint32_t parity, unsigned long long limit_ns,
                                                          volatile int* abort, uint32_t* status) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  uint32_t spins = 0;
  while (true) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
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

constexpr int kPStages = 6;
constexpr int kPThreads = 224;
constexpr int kPBN = 256;

struct PairWSmem {
  static constexpr int A_BYTES = kBM * kBK * 2;             // 16 KB: this CTA's 128 output rows
  static constexpr int B_BYTES = (kPBN / 2) * kBK * 2;      // 16 KB: this CTA's 128 columns
  static constexpr size_t off_a = 0;
  static constexpr size_t off_b = off_a + (size_t)kPStages * A_BYTES;
  static constexpr size_t off_stg = off_b + (size_t)kPStages * B_BYTES;
  static constexpr size_t off_bar = off_stg + (size_t)kBM * kStgRow;
  static constexpr int n_bar = 4 * kPStages + 5;  // lfull, full, empty, zdone, tfull[2], tempty[2], drain
  static constexpr size_t off_misc = off_bar + 8 * n_bar;
  static constexpr size_t off_tab = off_misc + 16;
  static constexpr size_t end = off_tab + sizeof(int) * 3 * (kMaxN + 2);
  static constexpr size_t bytes = end + 1024;
  static_assert(bytes <= 232448, "shared memory per CTA");
};

// a.mt_r / a.mt_s count pair tiles here (output rows / 256).
__global__ void __launch_bounds__(kPThreads, 1)
wgrad_pair_kernel(const __grid_constant__ CUtensorMap tmA_r, const __grid_constant__ CUtensorMap tmB_r,
                  const __grid_constant__ CUtensorMap tmA_s, const __grid_constant__ CUtensorMap tmB_s, const Args a) {
  pdl_wait_then_release();
  using SM = PairWSmem;
  constexpr int BN = kPBN;
  constexpr uint32_t TMEM_COLS = 2 * BN;
  constexpr uint32_t IDESC = idesc_t(2 * kBM, BN, true, true);
  constexpr uint32_t TX_BYTES = SM::A_BYTES + SM::B_BYTES;  // this CTA's copies of one stage

  extern __shared__ unsigned char smem_raw[];
  unsigned char* base =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sA = base + SM::off_a;
  unsigned char* sB = base + SM::off_b;
  unsigned char* stg = base + SM::off_stg;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + SM::off_bar);
  volatile int* misc = reinterpret_cast<volatile int*>(base + SM::off_misc);  // [0] tmem, [1] abort
  int* s_tstart = reinterpret_cast<int*>(base + SM::off_tab);
  int* s_row0 = s_tstart + (kMaxN + 2);
  int* s_m = s_row0 + (kMaxN + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int N = a.N;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  auto lfull_bar = [&](int s) { return smem_u32(bars + s); };
  auto full_bar = [&](int s) { return smem_u32(bars + kPStages + s); };
  auto empty_bar = [&](int s) { return smem_u32(bars + 2 * kPStages + s); };
  auto zdone_bar = [&](int s) { return smem_u32(bars + 3 * kPStages + s); };
  auto tfull_bar = [&](int s) { return smem_u32(bars + 4 * kPStages + s); };
  auto tempty_bar = [&](int s) { return smem_u32(bars + 4 * kPStages + 2 + s); };
  const uint32_t drain_bar = smem_u32(bars + 4 * kPStages + 4);
  volatile int* abort_flag = misc + 1;

  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA_r);
    prefetch_tmap(&tmB_r);
    if (a.has_shared) {
      prefetch_tmap(&tmA_s);
      prefetch_tmap(&tmB_s);
    }
    for (int s = 0; s < kPStages; ++s) {
      mbar_init(lfull_bar(s), 1);  // a last k-block: this CTA's expect_tx arrival and its bytes
      mbar_init(full_bar(s), 1);   // leader: its expect_tx arrival (with both CTAs' bytes), or,
                                   // for a last k-block, its ready warp's arrival
      mbar_init(empty_bar(s), 1);  // one commit from the leader's MMA thread
      mbar_init(zdone_bar(s), 1);  // leader: the other CTA's tail rows are zeroed
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
    // Per-group tile table from the device-resident offsets (both CTAs build the same one);
    // the shared expert's K chunks come first: they are the longest tiles.
    int acc = 0, prev = 0;
    bool bad = false;
    if (a.has_shared) {
      s_tstart[N] = 0;
      acc = a.nsplit * a.mt_s * a.nt_s;
    }
    for (int g = 0; g <= N; ++g) {
      int m, row0;
      if (g < N) {
        const int o0 = a.offsets[g], o1 = a.offsets[g + 1];
        if (o0 != prev || o1 < o0 || (long long)o1 > a.rows_cap) bad = true;
        prev = o1;
        m = bad ? 0 : o1 - o0;
        row0 = o0;
        s_tstart[g] = acc;
        acc += a.mt_r * a.nt_r;
      } else {
        m = a.has_shared ? a.T : 0;
        row0 = 0;
      }
      s_row0[g] = row0;
      s_m[g] = m;
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

  // t.mt: pair tile (256 output rows); this CTA's 128-row tile is 2 t.mt + rank
  auto decode = [&](int tile) {
    Tile ti;
    const int nsh = a.has_shared ? a.nsplit * a.mt_s * a.nt_s : 0;
    if (tile < nsh) {
      const int per = a.mt_s * a.nt_s;
      ti.g = N;
      ti.chunk = tile / per;
      const int local = tile - ti.chunk * per;
      ti.mt = local / a.nt_s;
      ti.nt = local - ti.mt * a.nt_s;
      ti.row0 = ti.chunk * a.chunk_kb * kBK;
      ti.krows = max(0, min(a.chunk_kb * kBK, s_m[N] - ti.row0));
    } else {
      const int per = a.mt_r * a.nt_r;
      const int e = (tile - nsh) / per;
      const int local = tile - nsh - e * per;
      ti.g = e;
      ti.chunk = 0;
      ti.mt = local / a.nt_r;
      ti.nt = local - ti.mt * a.nt_r;
      ti.row0 = s_row0[e];
      ti.krows = s_m[e];
    }
    ti.nkb = (ti.krows + kBK - 1) / kBK;
    ti.mvalid = kBM;
    ti.brow = 0;
    return ti;
  };
  auto tile_at = [&](int r) { return r * npairs + pair; };

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------ TMA producer (both CTAs): this CTA's A rows and B half
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_par = 0;     // stages whose copies count on the leader's barrier
      uint32_t larmed = 0, lpar = 0;         // stages whose copies count on this CTA's barrier
      for (int r = 0;; ++r) {
        const int tile = tile_at(r);
        if (tile >= total) break;
        const Tile ti = decode(tile);
        const void* ta = (ti.g < N) ? (const void*)&tmA_r : (const void*)&tmA_s;
        const void* tb = (ti.g < N) ? (const void*)&tmB_r : (const void*)&tmB_s;
        const int ax = (2 * ti.mt + (int)rank) * kBM;
        const int bx = ti.nt * BN + (int)rank * (BN / 2);
        bool ok = true;
        for (int kb = 0; kb < ti.nkb; ++kb) {
          if (!mbar_wait_bounded(empty_bar(stage), phase ^ 1u, a.limit_ns, abort_flag, a.status)) {
            ok = false;
            break;
          }
          const uint32_t dA = smem_u32(sA + stage * SM::A_BYTES);
          const uint32_t dB = smem_u32(sB + stage * SM::B_BYTES);
          const int kr = ti.row0 + kb * kBK;
          if (ti.krows - kb * kBK >= kBK) {
            const uint32_t fb = map_to_rank(full_bar(stage), 0);
            if (leader) mbar_arrive_expect_tx(full_bar(stage), 2 * TX_BYTES);
            tma_load_2d_pair(dA, ta, fb, ax, kr);
            tma_load_2d_pair(dA + kBox, ta, fb, ax + 64, kr);
            tma_load_2d_pair(dB, tb, fb, bx, kr);
            tma_load_2d_pair(dB + kBox, tb, fb, bx + 64, kr);
            armed |= 1u << stage;
            armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
          } else {
            // the expert's last k-block: the ready warp zeroes its tail rows first
            mbar_arrive_expect_tx(lfull_bar(stage), TX_BYTES);
            tma_load_2d(dA, ta, lfull_bar(stage), ax, kr);
            tma_load_2d(dA + kBox, ta, lfull_bar(stage), ax + 64, kr);
            tma_load_2d(dB, tb, lfull_bar(stage), bx, kr);
            tma_load_2d(dB + kBox, tb, lfull_bar(stage), bx + 64, kr);
            larmed |= 1u << stage;
            lpar ^= 1u << stage;  // parity of the phase this use completes, plus one
          }
          if (++stage == kPStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
      }
      if (*abort_flag) {
        // copies still in flight land before the CTA leaves: a full k-block's on the leader's
        // barrier (both CTAs' bytes), a last one's on this CTA's
        for (int s = 0; s < kPStages; ++s) {
          if (leader && (armed & (1u << s)))
            (void)mbar_wait_bounded(full_bar(s), (armed_par >> s) & 1u, a.limit_ns, nullptr, a.status);
          if (larmed & (1u << s))
            (void)mbar_wait_bounded(lfull_bar(s), ((lpar >> s) & 1u) ^ 1u, a.limit_ns, nullptr, a.status);
        }
      }
    }
  } else if (warp == 6) {
    // ------------------------------ ready warp (both CTAs): an expert's last k-block has its
    // tail rows zeroed in both CTAs before the leader's full barrier counts it
    int stage = 0;
    uint32_t lpar = 0;  // per stage: parity of the next phase of this CTA's barrier
    for (int r = 0;; ++r) {
      const int tile = tile_at(r);
      if (tile >= total) break;
      const Tile ti = decode(tile);
      bool ok = true;
      for (int kb = 0; kb < ti.nkb; ++kb) {
        const int rem = ti.krows - kb * kBK;
        if (rem >= kBK) {
          if (++stage == kPStages) stage = 0;
          continue;
        }
        int f = 1;
        if (lane == 0)
          f = mbar_wait_bounded(lfull_bar(stage), (lpar >> stage) & 1u, a.limit_ns, abort_flag, a.status);
        if (!__shfl_sync(0xffffffffu, f, 0)) {
          ok = false;
          break;
        }
        {
          // rows [rem, 16 * ceil(rem / 16)) of every box belong to another expert (or were
          // never written): zeroed in both operands; later 16-row steps are skipped
          const int z0 = rem, z1 = ((rem + 15) >> 4) * 16;
          const int nrows = z1 - z0;
          for (int i = lane; i < 4 * nrows * 8; i += 32) {
            const int box = i / (nrows * 8);
            const int rr = (i / 8) % nrows + z0;
            const int ch = i & 7;
            unsigned char* p = (box < 2) ? sA + stage * SM::A_BYTES + box * kBox
                                         : sB + stage * SM::B_BYTES + (box - 2) * kBox;
            *reinterpret_cast<uint4*>(p + rr * 128 + ch * 16) = make_uint4(0u, 0u, 0u, 0u);
          }
          fence_proxy_async_shared();
        }
        __syncwarp();
        if (lane == 0) {
          if (leader) mbar_arrive(full_bar(stage));
          else mbar_arrive_cluster(map_to_rank(zdone_bar(stage), 0));
        }
        lpar ^= 1u << stage;
        if (++stage == kPStages) stage = 0;
      }
      if (!ok) break;
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ------------------------------ MMA issuer (leader CTA, one thread)
      int stage = 0;
      uint32_t phase = 0;
      uint32_t zpar = 0;  // per stage: parity of the next phase of the zeroed barrier
      for (int li = 0;; ++li) {
        const int tile = tile_at(li);
        if (tile >= total) break;
        const Tile ti = decode(tile);
        const int acc = li & 1;
        const uint32_t ap = (uint32_t)(li >> 1) & 1u;
        if (!mbar_wait_bounded_cluster(tempty_bar(acc), ap ^ 1u, a.limit_ns, abort_flag, a.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        bool ok = true;
        for (int kb = 0; kb < ti.nkb; ++kb) {
          if (!mbar_wait_bounded(full_bar(stage), phase, a.limit_ns, abort_flag, a.status)) {
            ok = false;
            break;
          }
          const int rem = ti.krows - kb * kBK;
          if (rem < kBK) {
            // an expert's last k-block: the other CTA's tail rows are zeroed too
            if (!mbar_wait_bounded_cluster(zdone_bar(stage), (zpar >> stage) & 1u, a.limit_ns, abort_flag,
                                           a.status)) {
              ok = false;
              break;
            }
            zpar ^= 1u << stage;
          }
          tc_fence_after();
          const int nk16 = (rem < kBK) ? (rem + 15) >> 4 : kBK / 16;
          const uint32_t aS = smem_u32(sA + stage * SM::A_BYTES);
          const uint32_t bS = smem_u32(sB + stage * SM::B_BYTES);
          for (int k = 0; k < nk16; ++k)
            tc_mma_pair(d_tmem, desc_mn_sw128(aS + (uint32_t)(k * 2048), kBox),
                        desc_mn_sw128(bS + (uint32_t)(k * 2048), kBox), IDESC, (kb | k) != 0 ? 1u : 0u);
          // free this stage in both CTAs
          tc_commit_pair(empty_bar(stage));
          tc_commit_pair(map_to_rank(empty_bar(stage), 1));
          if (++stage == kPStages) {
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
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const int etid = (warp - 2) * 32 + lane;
    const uint32_t tempty_leader = map_to_rank(tempty_bar(0), 0);
    for (int li = 0;; ++li) {
      const int tile = tile_at(li);
      if (tile >= total) break;
      const Tile ti = decode(tile);
      const int acc = li & 1;
      const uint32_t ap = (uint32_t)(li >> 1) & 1u;
      if (!mbar_wait_bounded(tfull_bar(acc), ap, a.limit_ns, abort_flag, a.status)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
      const int mt = 2 * ti.mt + (int)rank;  // this CTA's 128-row output tile
      const bool sh = ti.g == N;
      const bool partial = sh && (a.nsplit > 1 || a.part_only);
      const bool empty = ti.nkb == 0;
      const int ld = sh ? a.ld_s : a.ld_r;
      if (partial) {
        // fp32 partial of one K chunk, straight from registers
        const size_t mrows_s = (size_t)a.mt_s * 2 * kBM;
        float* P = a.part_s + ((size_t)ti.chunk * mrows_s + (size_t)mt * kBM + row) * a.ld_s + ti.nt * BN;
#pragma unroll 1
        for (int g16 = 0; g16 < BN / 16; ++g16) {
          uint32_t r[16];
          if (!empty) {
            tmem_ld16(tb + (uint32_t)(g16 * 16), r);
            tmem_ld_wait();
          } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) r[j] = 0u;
          }
          float4* dst = reinterpret_cast<float4*>(P + g16 * 16);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            dst[j] = make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                                 __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3]));
        }
        tc_fence_before();
        mbar_arrive_cluster(tempty_leader + 8u * (uint32_t)acc);
      } else {
        uint16_t* o1 = sh ? a.out_s : a.out_r;
        uint16_t* o2 = sh ? a.out_s2 : a.out_r2;
        const int e = sh ? 0 : ti.g;
        const int mrows = (sh ? a.mt_s : a.mt_r) * 2 * kBM;  // packed output rows per group
        uint16_t *out, *out_hi;
        size_t rowoff_lo, rowoff_hi;
        if (o2) {  // packed gate/up: tile rows 0..63 are gate rows, 64..127 the up rows
          const size_t half = (size_t)(mrows / 2) * ld;
          out = o1 + e * half;
          out_hi = o2 + e * half;
          rowoff_lo = (size_t)(mt * 64) * ld;
          rowoff_hi = rowoff_lo;
        } else {
          out = o1 + (size_t)e * mrows * ld;
          out_hi = out;
          rowoff_lo = (size_t)(mt * kBM) * ld;
          rowoff_hi = rowoff_lo + (size_t)64 * ld;
        }
#pragma unroll 1
        for (int c = 0; c < BN / 64; ++c) {
#pragma unroll
          for (int g16 = 0; g16 < 4; ++g16) {
            uint32_t r[16];
            if (!empty) {
              tmem_ld16(tb + (uint32_t)(c * 64 + g16 * 16), r);
              tmem_ld_wait();
            } else {
#pragma unroll
              for (int j = 0; j < 16; ++j) r[j] = 0u;
            }
            uint32_t packed[8];
#pragma unroll
            for (int j = 0; j < 8; ++j)
              packed[j] = pack_bf16x2(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1]));
            uint4* dst = reinterpret_cast<uint4*>(stg + row * kStgRow + g16 * 32);
            dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
            dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
          }
          if (c == BN / 64 - 1) {
            // this CTA's half of the accumulator is drained: let the leader reuse it
            tc_fence_before();
            mbar_arrive_cluster(tempty_leader + 8u * (uint32_t)acc);
          }
          named_bar_sync(1, 128);
#pragma unroll
          for (int it = 0; it < 8; ++it) {
            const int idx = it * 128 + etid;
            const int rr = idx >> 3, ch = idx & 7;
            const uint4 v = *reinterpret_cast<const uint4*>(stg + rr * kStgRow + ch * 16);
            const int col = ti.nt * BN + c * 64 + ch * 8;
            uint16_t* dst = (rr < 64) ? out + rowoff_lo + (size_t)rr * ld : out_hi + rowoff_hi + (size_t)(rr - 64) * ld;
            *reinterpret_cast<uint4*>(dst + col) = v;
          }
          named_bar_sync(1, 128);
        }
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

template <int BN, int MODE>
static int launch(const CUtensorMap& ar, const CUtensorMap& br, const CUtensorMap& as_, const CUtensorMap& bs,
                  const CUtensorMap& zr, const CUtensorMap& zs, const Args& a, long long max_tiles, cudaStream_t st) {
  using SM = Smem<BN, MODE>;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(bwd_gemm_kernel<BN, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SM::bytes);
    if (e != cudaSuccess) return cuda_status(e);
    attr_set[dev] = true;
  }
  long long grid = sm_count();
  if (max_tiles < grid) grid = max_tiles;
  if (grid < 1) grid = 1;
  return launch_pdl(bwd_gemm_kernel<BN, MODE>, dim3((unsigned)grid), dim3(Threads<MODE>::total), SM::bytes, st, ar, br, as_, bs,
                    zr, zs, a);
}

static Args base_args(const moe_dims_t& d, const int32_t* offsets, uint32_t* status) {
  Args a{};
  a.offsets = offsets;
  a.N = d.N;
  a.T = d.T;
  a.rows_cap = (long long)d.T * d.K;
  a.status = status;
  a.limit_ns = kWaitLimitNs;
  a.has_shared = 1;
  a.nsplit = 1;
  a.chunk_kb = 1;
  return a;
}

static long long dgrad_max_tiles(const moe_dims_t& d, int nt_r, int nt_s) {
  const long long rcap = (long long)d.T * d.K;
  return (rcap / kBM + d.N) * nt_r + (long long)((d.T + kBM - 1) / kBM) * nt_s;
}

static int wgrad_bn(int a, int b) {
  for (int bn = 256; bn >= 64; bn >>= 1)
    if (a % bn == 0 && b % bn == 0) return bn;
  return 0;
}

}  // namespace bwd

using namespace bwd;

// K chunks of the shared expert's weight gradients: at least 32 k-blocks (2048 rows) each,
// at most 16 chunks.
int bwd_shared_split(const moe_dims_t& d, int* chunk_kb) {
  const int kb = (d.T + kBK - 1) / kBK;
  int ck = 32;
  if ((kb + ck - 1) / ck > 16) ck = (kb + 15) / 16;
  if (chunk_kb) *chunk_kb = ck;
  const int n = (kb + ck - 1) / ck;
  return n < 1 ? 1 : n;
}

size_t bwd_split_partial_floats(const moe_dims_t& d) {
  const int ns = bwd_shared_split(d, nullptr);
  if (ns <= 1) return 0;
  const size_t a = (size_t)d.d * d.F_shared, b = (size_t)2 * d.F_shared * d.d;
  return (size_t)ns * (a > b ? a : b);
}

static int dgrad_bn(int a, int b) {
  for (int bn = 256; bn >= 64; bn >>= 1)
    if (a % bn == 0 && b % bn == 0) return bn;
  return 0;
}

// dh = dys W_d (routed rows) and dh_shared = dy W_sd (all T rows).
int launch_dgrad_down(const moe_dims_t& d, const int32_t* offsets, const uint16_t* dys, const uint16_t* dy,
                      const uint16_t* w_down, const uint16_t* sdown, uint16_t* dh, uint16_t* dh_shared,
                      uint32_t* status, cudaStream_t st) {
  const long long rcap = (long long)d.T * d.K;
  const int BN = dgrad_bn(d.F, d.F_shared);
  if (BN == 0) return MOE_ERR_UNSUPPORTED;
  Args a = base_args(d, offsets, status);
  a.kb_r = a.kb_s = d.d / kBK;
  a.nt_r = d.F / BN;
  a.nt_s = d.F_shared / BN;
  a.kdim_r = d.d;
  a.out_r = dh;
  a.ld_r = d.F;
  a.out_s = dh_shared;
  a.ld_s = d.F_shared;
  CUtensorMap ar, br, as_, bs;
  if (!(make_tmap_bf16(&ar, dys, rcap, d.d, kBM) && make_tmap_bf16(&br, w_down, (uint64_t)d.N * d.d, d.F, 64) &&
        make_tmap_bf16(&as_, dy, d.T, d.d, kBM) && make_tmap_bf16(&bs, sdown, d.d, d.F_shared, 64)))
    return MOE_ERR_CUDA;
  const long long mt = dgrad_max_tiles(d, a.nt_r, a.nt_s);
  switch (BN) {
    case 256: return launch<256, kDgradPlain>(ar, br, as_, bs, ar, ar, a, mt, st);
    case 128: return launch<128, kDgradPlain>(ar, br, as_, bs, ar, ar, a, mt, st);
    default: return launch<64, kDgradPlain>(ar, br, as_, bs, ar, ar, a, mt, st);
  }
}

// The gate/up pre-activations z recomputed in TMEM (fp32) and, in the epilogue, the SwiGLU
// derivative dz = [da | db] (packed column order) from z and dh.
int launch_swiglu_backward(const moe_dims_t& d, const int32_t* offsets, const uint16_t* xs, const uint16_t* x,
                           const uint16_t* gate_up, const uint16_t* sgate_up, const uint16_t* dh,
                           const uint16_t* dh_shared, uint16_t* dz, uint16_t* dzs, uint32_t* status,
                           cudaStream_t st) {
  const long long rcap = (long long)d.T * d.K;
  const int BN = (d.F % 128 == 0 && d.F_shared % 128 == 0) ? 256 : 128;
  Args a = base_args(d, offsets, status);
  a.kb_r = a.kb_s = d.d / kBK;
  a.nt_r = 2 * d.F / BN;
  a.nt_s = 2 * d.F_shared / BN;
  a.kdim_r = 2 * d.F;
  a.out_r = dz;
  a.ld_r = 2 * d.F;
  a.out_s = dzs;
  a.ld_s = 2 * d.F_shared;
  CUtensorMap ar, br, as_, bs, hr, hs;
  if (!(make_tmap_bf16(&ar, xs, rcap, d.d, kBM) && make_tmap_bf16(&br, gate_up, (uint64_t)d.N * 2 * d.F, d.d, BN) &&
        make_tmap_bf16(&as_, x, d.T, d.d, kBM) && make_tmap_bf16(&bs, sgate_up, (uint64_t)2 * d.F_shared, d.d, BN) &&
        make_tmap_bf16(&hr, dh, rcap, d.F, kBM) && make_tmap_bf16(&hs, dh_shared, d.T, d.F_shared, kBM)))
    return MOE_ERR_CUDA;
  const long long mt = dgrad_max_tiles(d, a.nt_r, a.nt_s);
  return BN == 256 ? launch<256, kPreactSwiglu>(ar, br, as_, bs, hr, hs, a, mt, st)
                   : launch<128, kPreactSwiglu>(ar, br, as_, bs, hr, hs, a, mt, st);
}

int launch_dgrad_gate_up(const moe_dims_t& d, const int32_t* offsets, const uint16_t* dz, const uint16_t* dzs,
                         const uint16_t* gate_up, const uint16_t* sgate_up, const uint16_t* dsplit,
                         const uint16_t* w2, uint16_t* dxs, uint16_t* dx_shared, uint32_t* status, cudaStream_t st) {
  const long long rcap = (long long)d.T * d.K;
  const int BN = (d.d % 256 == 0) ? 256 : 128;
  Args a = base_args(d, offsets, status);
  a.kb_r = 2 * d.F / kBK;
  a.kb_s = 2 * d.F_shared / kBK;
  a.nt_r = a.nt_s = d.d / BN;
  a.kdim_r = 2 * d.F;
  a.out_r = dxs;
  a.ld_r = d.d;
  a.out_s = dx_shared;
  a.ld_s = d.d;
  CUtensorMap ar, br, as_, bs, xr, xw;
  if (!(make_tmap_bf16(&ar, dz, rcap, 2 * d.F, kBM) &&
        make_tmap_bf16(&br, gate_up, (uint64_t)d.N * 2 * d.F, d.d, 64) &&
        make_tmap_bf16(&as_, dzs, d.T, 2 * d.F_shared, kBM) &&
        make_tmap_bf16(&bs, sgate_up, (uint64_t)2 * d.F_shared, d.d, 64)))
    return MOE_ERR_CUDA;
  xr = ar;
  xw = ar;
  if (dsplit && w2) {
    const int rp = router_split_rows(d);
    a.xrp = rp;
    a.kb_x = 3 * (rp / kBK);  // (hi, hi), (hi, lo), (lo, hi) over RP/64 k-blocks each
    if (!(make_tmap_bf16(&xr, dsplit, d.T, 2 * rp, kBM) && make_tmap_bf16(&xw, w2, (uint64_t)2 * rp, d.d, 64)))
      return MOE_ERR_CUDA;
  }
  const long long mt = dgrad_max_tiles(d, a.nt_r, a.nt_s);
  return BN == 256 ? launch<256, kDgradPlain>(ar, br, as_, bs, xr, xw, a, mt, st)
                   : launch<128, kDgradPlain>(ar, br, as_, bs, xr, xw, a, mt, st);
}

// One wave of CTA pairs (clusters of two), at most one per pair tile.
static int launch_wgrad_pair(const CUtensorMap& ar, const CUtensorMap& br, const CUtensorMap& as_,
                             const CUtensorMap& bs, const Args& a, long long max_tiles, cudaStream_t st) {
  static int clusters[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  auto kern = wgrad_pair_kernel;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // see launch_pdl
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.blockDim = dim3(kPThreads, 1, 1);
  cfg.dynamicSmemBytes = PairWSmem::bytes;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;  // the occupancy query below sees the cluster shape only
  if (dev >= 0 && dev < 64 && clusters[dev] == 0) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)PairWSmem::bytes);
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

// With MOE_FLAG_WGRAD_CTA_PAIR, 256-column tiles and an even number of 128-row output tiles
// per group, the weight gradients run on CTA pairs (wgrad_pair_kernel); else on one CTA.
static int launch_wgrad(const moe_dims_t& d, const Args& a0, int BN, const CUtensorMap& ar, const CUtensorMap& br,
                        const CUtensorMap& as_, const CUtensorMap& bs, int mrows_s, uint16_t* out_s,
                        uint16_t* out_s2, cudaStream_t st) {
  Args a = a0;
  if (a.nsplit > 1 && !a.part_s) return MOE_ERR_INVALID_ARG;
  int r;
  if ((d.flags & MOE_FLAG_WGRAD_CTA_PAIR) && BN == kPBN && a.mt_r % 2 == 0 && a.mt_s % 2 == 0) {
    a.mt_r /= 2;
    a.mt_s /= 2;
    const long long tiles = (long long)a.nsplit * a.mt_s * a.nt_s + (long long)d.N * a.mt_r * a.nt_r;
    r = launch_wgrad_pair(ar, br, as_, bs, a, tiles, st);
  } else {
    const long long tiles = (long long)a.nsplit * a.mt_s * a.nt_s + (long long)d.N * a.mt_r * a.nt_r;
    switch (BN) {
      case 256: r = launch<256, kWgrad>(ar, br, as_, bs, ar, ar, a, tiles, st); break;
      case 128: r = launch<128, kWgrad>(ar, br, as_, bs, ar, ar, a, tiles, st); break;
      default: r = launch<64, kWgrad>(ar, br, as_, bs, ar, ar, a, tiles, st); break;
    }
  }
  if (r != MOE_OK || a.nsplit <= 1) return r;
  const long long n8 = (long long)mrows_s * a.ld_s / 8;
  long long grid = (n8 + 255) / 256;
  if (grid > (long long)sm_count() * 8) grid = (long long)sm_count() * 8;
  return launch_pdl(split_reduce_kernel, dim3((unsigned)grid), dim3(256), 0, st, (const float*)a.part_s, a.nsplit,
                    mrows_s, a.ld_s, out_s, out_s2);
}

int launch_wgrad_down(const moe_dims_t& d, const int32_t* offsets, const uint16_t* dys, const uint16_t* dy,
                      const uint16_t* h, const uint16_t* h_shared, uint16_t* dw_down, uint16_t* dws_down,
                      float* partials, uint32_t* status, cudaStream_t st) {
  const long long rcap = (long long)d.T * d.K;
  const int BN = wgrad_bn(d.F, d.F_shared);
  if (BN == 0) return MOE_ERR_UNSUPPORTED;
  Args a = base_args(d, offsets, status);
  a.mt_r = a.mt_s = d.d / kBM;
  a.nt_r = d.F / BN;
  a.nt_s = d.F_shared / BN;
  a.nsplit = bwd_shared_split(d, &a.chunk_kb);
  a.out_r = dw_down;
  a.ld_r = d.F;
  a.out_s = dws_down;
  a.ld_s = d.F_shared;
  a.part_s = partials;
  CUtensorMap ar, br, as_, bs;
  if (!(make_tmap_bf16(&ar, dys, rcap, d.d, 64) && make_tmap_bf16(&br, h, rcap, d.F, 64) &&
        make_tmap_bf16(&as_, dy, d.T, d.d, 64) && make_tmap_bf16(&bs, h_shared, d.T, d.F_shared, 64)))
    return MOE_ERR_CUDA;
  return launch_wgrad(d, a, BN, ar, br, as_, bs, d.d, dws_down, nullptr, st);
}

int launch_wgrad_gate_up(const moe_dims_t& d, const int32_t* offsets, const uint16_t* dz, const uint16_t* dzs,
                         const uint16_t* xs, const uint16_t* x, uint16_t* dw_gate, uint16_t* dw_up,
                         uint16_t* dws_gate, uint16_t* dws_up, float* partials, uint32_t* status,
                         cudaStream_t st) {
  const long long rcap = (long long)d.T * d.K;
  const int BN = (d.d % 256 == 0) ? 256 : 128;
  Args a = base_args(d, offsets, status);
  a.mt_r = 2 * d.F / kBM;
  a.mt_s = 2 * d.F_shared / kBM;
  a.nt_r = a.nt_s = d.d / BN;
  a.nsplit = bwd_shared_split(d, &a.chunk_kb);
  a.out_r = dw_gate;
  a.out_r2 = dw_up;
  a.ld_r = d.d;
  a.out_s = dws_gate;
  a.out_s2 = dws_up;
  a.ld_s = d.d;
  a.part_s = partials;
  CUtensorMap ar, br, as_, bs;
  if (!(make_tmap_bf16(&ar, dz, rcap, 2 * d.F, 64) && make_tmap_bf16(&br, xs, rcap, d.d, 64) &&
        make_tmap_bf16(&as_, dzs, d.T, 2 * d.F_shared, 64) && make_tmap_bf16(&bs, x, d.T, d.d, 64)))
    return MOE_ERR_CUDA;
  return launch_wgrad(d, a, BN, ar, br, as_, bs, 2 * d.F_shared, dws_gate, dws_up, st);
}

// K chunks of the router weight gradient dsplit^T x: at least 16 k-blocks each, at most 16
// chunks (on the 0.6B-shaped workload one round of 128 tiles, 16.8 MB of partials).
int router_wgrad_split(const moe_dims_t& d, int* chunk_kb) {
  const int kb = (d.T + kBK - 1) / kBK;
  int ck = 16;
  if ((kb + ck - 1) / ck > 16) ck = (kb + 15) / 16;
  if (chunk_kb) *chunk_kb = ck;
  const int n = (kb + ck - 1) / ck;
  return n < 1 ? 1 : n;
}

// Router weight gradient on the tensor cores: fp32 partials of dsplit^T x per K chunk
// ([chunks, 2 RP, d]: hi-term rows, then lo-term rows), reduced by
// launch_router_wgrad_reduce. The weight-gradient kernel runs with no routed group.
int launch_router_wgrad_tc(const moe_dims_t& d, const uint16_t* dsplit, const uint16_t* x, float* part,
                           uint32_t* status, cudaStream_t st) {
  const int rp = router_split_rows(d);
  const int BN = (d.d % 256 == 0) ? 256 : 128;
  moe_dims_t d0 = d;
  d0.N = 0;
  Args a = base_args(d0, nullptr, status);
  a.mt_r = a.nt_r = 0;
  a.mt_s = 2 * rp / kBM;
  a.nt_s = d.d / BN;
  a.nsplit = router_wgrad_split(d, &a.chunk_kb);
  a.part_only = 1;
  a.part_s = part;
  a.ld_s = d.d;
  a.rows_cap = d.T;
  CUtensorMap as_, bs;
  if (!(make_tmap_bf16(&as_, dsplit, d.T, 2 * rp, 64) && make_tmap_bf16(&bs, x, d.T, d.d, 64))) return MOE_ERR_CUDA;
  const long long tiles = (long long)a.nsplit * a.mt_s * a.nt_s;
  return BN == 256 ? launch<256, kWgrad>(as_, bs, as_, bs, as_, as_, a, tiles, st)
                   : launch<128, kWgrad>(as_, bs, as_, bs, as_, as_, a, tiles, st);
}

}  // namespace moe
