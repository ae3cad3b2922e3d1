// Backward pass of the layer outside the expert GEMMs: the combine, the router (gates,
// load-balance and Z-loss terms), the router's weight gradient and the input gradient.
//
// Kilian et al., "Improving MoE Compute Efficiency by Composing Weight and Data Sparsity"
// (review page): y = E_shared(x) + sum_i g_i E_i(x) (三 / 核心公式), gates renormalised
// over the selected real experts (三 / Null Expert 机制), L_bal = N sum_i f_i P_i
// (三 / 负载均衡损失) and L_z = mean_t lse_t^2 (三 / Z-Loss), trained with the two losses
// at fixed weights (四 / 训练配置). The objective differentiated is
// <y, dy> + alpha L_bal + beta L_z. Top-K choices and the load fractions f_i are
// piecewise constant in the logits and carry no gradient. MoE++ copy and constant experts
// (MoE++ explainer page, 三种零计算专家) take gates like real experts and output x and c_j.
#include "moe_internal.cuh"

namespace moe {

constexpr int kBwdThreads = 256;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float dot8(const uint4& a, const uint4& b) {
  float s = bf16lo(a.x) * bf16lo(b.x);
  s = fmaf(bf16hi(a.x), bf16hi(b.x), s);
  s = fmaf(bf16lo(a.y), bf16lo(b.y), s);
  s = fmaf(bf16hi(a.y), bf16hi(b.y), s);
  s = fmaf(bf16lo(a.z), bf16lo(b.z), s);
  s = fmaf(bf16hi(a.z), bf16hi(b.z), s);
  s = fmaf(bf16lo(a.w), bf16lo(b.w), s);
  s = fmaf(bf16hi(a.w), bf16hi(b.w), s);
  return s;
}
__device__ __forceinline__ uint4 scale8(float g, const uint4& v) {
  return make_uint4(pack_bf16x2(g * bf16lo(v.x), g * bf16hi(v.x)), pack_bf16x2(g * bf16lo(v.y), g * bf16hi(v.y)),
                    pack_bf16x2(g * bf16lo(v.z), g * bf16hi(v.z)), pack_bf16x2(g * bf16lo(v.w), g * bf16hi(v.w)));
}

// ---------------------------------------------------------------------------------------
// Combine backward: for each selected slot of token t, dg[t,k] = <dy_t, out_k> with out_k
// the slot's expert output (a row of ys, x_t for a copy expert, c_j for a constant
// expert; 0 for a null copy), and for a real slot dys[row] = g[t,k] dy_t (bf16), the
// upstream gradient of that expert row. The shared expert's upstream gradient is dy.
// One warp per token, slots in groups of four: for each group, passes of 64 16-byte
// chunks (two per lane) load the dy chunks and the four slots' chunks together before any
// is used; dot products accumulate in fp32 per lane and are reduced across the warp in a
// fixed order.
__global__ void __launch_bounds__(kBwdThreads)
combine_bwd_kernel(const uint16_t* __restrict__ dy, const uint16_t* __restrict__ ys,
                   const float* __restrict__ gate, const int32_t* __restrict__ slot_row,
                   const int32_t* __restrict__ topk_idx, const uint16_t* __restrict__ x,
                   const uint16_t* __restrict__ cv, uint16_t* __restrict__ dys, float* __restrict__ dg, int T,
                   int d, int K, long long rcap, int NM, int C, int V, uint32_t* status) {
  pdl_wait_then_release();
  const int lane = threadIdx.x & 31;
  const int wpb = kBwdThreads / 32;
  const int nch = d >> 3;
  for (int t = blockIdx.x * wpb + (threadIdx.x >> 5); t < T; t += gridDim.x * wpb) {
    int row = -1;
    float g = 0.f;
    if (lane < K) {
      row = __ldg(slot_row + (size_t)t * K + lane);
      g = __ldg(gate + (size_t)t * K + lane);
      if (row >= rcap) {
        atomicOr(status, kStatusBounds);
        row = -1;
      }
      if (row < 0 && C + V > 0) {
        const int id = __ldg(topk_idx + (size_t)t * K + lane) - NM;
        if (id >= 0 && id < C) row = -2;
        else if (id >= C && id < C + V) row = -3 - (id - C);
      }
    }
    const uint4* dyr = reinterpret_cast<const uint4*>(dy + (size_t)t * d);
    float mydg = 0.f;
    for (int k0 = 0; k0 < K; k0 += 4) {
      int rq[4];
      float gq[4], dot[4];
      const uint4* src[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int k = k0 + u;
        rq[u] = __shfl_sync(0xffffffffu, row, k & 31);
        gq[u] = __shfl_sync(0xffffffffu, g, k & 31);
        if (k >= K) rq[u] = -1;
        const uint16_t* sp = (rq[u] >= 0)    ? ys + (size_t)rq[u] * d
                             : (rq[u] == -2) ? x + (size_t)t * d
                             : (rq[u] <= -3) ? cv + (size_t)(-3 - rq[u]) * d
                                             : ys;
        src[u] = reinterpret_cast<const uint4*>(sp);
        dot[u] = 0.f;
      }
      if (rq[0] == -1 && rq[1] == -1 && rq[2] == -1 && rq[3] == -1) continue;  // all null copies
      for (int c0 = 0; c0 < nch; c0 += 64) {
        const int ca = c0 + lane, cb = c0 + 32 + lane;
        const bool oka = ca < nch, okb = cb < nch;
        const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
        const uint4 ya = oka ? __ldg(dyr + ca) : z4;
        const uint4 yb = okb ? __ldg(dyr + cb) : z4;
        uint4 va[4], vb[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          va[u] = (rq[u] != -1 && oka) ? __ldg(src[u] + ca) : z4;
          vb[u] = (rq[u] != -1 && okb) ? __ldg(src[u] + cb) : z4;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if (rq[u] == -1) continue;
          dot[u] += dot8(ya, va[u]) + dot8(yb, vb[u]);
          if (rq[u] >= 0) {
            uint4* dst = reinterpret_cast<uint4*>(dys + (size_t)rq[u] * d);
            if (oka) dst[ca] = scale8(gq[u], ya);
            if (okb) dst[cb] = scale8(gq[u], yb);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float sdot = warp_sum(dot[u]);
        if (lane == k0 + u) mydg = sdot;
      }
    }
    if (lane < K) dg[(size_t)t * K + lane] = mydg;
  }
}

// ---------------------------------------------------------------------------------------
// Router backward: the logit gradient ds[t, j] for every router row j, one warp per token.
//   gates: for the selected slots that are not null copies, g = softmax of their logits, so
//     ds[col(k)] += g_k (dg_k - sum_l g_l dg_l);
//   alpha L_bal, with p the pool softmax and f_i = counts_ext[i] / T_total:
//     dv_i = alpha (N / T_total) p_i (f_i - sum_l f_l p_l);
//   beta L_z: dv_i = beta (2 / T_total) lse p_i.
// The M null copies all read the null logit (column N), so its gradient is the sum over
// the copies; with M = 0 the null logit is not in the pool and gets 0.
// Besides ds (fp32) the kernel writes ds as two bf16 terms, hi = bf16(ds) and
// lo = bf16(ds - hi), in dsplit [T, 2 RP] (columns j and RP + j, zero past the router
// rows), the operand of the tensor-core products ds^T x and ds W_r, and per-warp column
// sums of ds for the bias gradient.
constexpr int kRouterBwdMaxGrid = 1184;  // 8 CTAs per SM on 148 SMs; also sizes the bias partials

__global__ void __launch_bounds__(kBwdThreads)
router_bwd_kernel(const float* __restrict__ logits, const int32_t* __restrict__ topk_idx,
                  const float* __restrict__ gate, const float* __restrict__ dg,
                  const int32_t* __restrict__ counts_ext, double inv_t, float alpha, float beta,
                  float* __restrict__ ds, float* __restrict__ dtnb, uint16_t* __restrict__ dsplit, int rp,
                  float* __restrict__ bpart, int T, int N, int M, int K, int C, int V) {
  pdl_wait_then_release();
  __shared__ float s_ds[kBwdThreads / 32][kMaxRows];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int rows = N + 1 + C + V;
  const float invT = (float)inv_t;
  // null copies' load fraction (sum over the M copies), the same for every token
  float fnull = 0.f;
  for (int c = lane; c < M; c += 32) fnull += (float)__ldg(counts_ext + N + c);
  fnull = warp_sum(fnull) * invT;
  float bsum[3] = {0.f, 0.f, 0.f};
  for (int t = blockIdx.x * (kBwdThreads / 32) + w; t < T; t += gridDim.x * (kBwdThreads / 32)) {
    const float* sr = logits + (size_t)t * rows;
    float s[3], f[3];
    float m = -INFINITY;
#pragma unroll
    for (int u = 0; u < 3; ++u) {
      const int j = lane + 32 * u;
      s[u] = (j < rows) ? __ldg(sr + j) : -INFINITY;
      f[u] = 0.f;
      if (j < N) f[u] = (float)__ldg(counts_ext + j) * invT;
      else if (j > N && j < rows) f[u] = (float)__ldg(counts_ext + M + j - 1) * invT;
      const bool in_pool = (j < rows) && (j != N || M > 0);
      if (in_pool) m = fmaxf(m, s[u]);
    }
    m = warp_max(m);
    float e[3];
    float z = 0.f;
#pragma unroll
    for (int u = 0; u < 3; ++u) {
      const int j = lane + 32 * u;
      e[u] = 0.f;
      if (j < rows && (j != N || M > 0)) e[u] = __expf(s[u] - m);
      z += (j == N) ? (float)M * e[u] : e[u];
    }
    z = warp_sum(z);
    const float lse = m + __logf(z);
    const float rz = 1.f / z;
    float fp = 0.f;  // sum over the pool of f_i p_i
#pragma unroll
    for (int u = 0; u < 3; ++u) {
      const int j = lane + 32 * u;
      const float p = e[u] * rz;
      fp += (j == N) ? fnull * p : f[u] * p;
    }
    fp = warp_sum(fp);
    const float cb = alpha * (float)N * invT, cz = beta * 2.f * invT * lse;
#pragma unroll
    for (int u = 0; u < 3; ++u) {
      const int j = lane + 32 * u;
      if (j < rows) {
        const float p = e[u] * rz;
        float v;
        if (j == N) v = (M > 0) ? cb * p * (fnull - (float)M * fp) + cz * (float)M * p : 0.f;
        else v = cb * p * (f[u] - fp) + cz * p;
        s_ds[w][j] = v;
      }
    }
    // gates: the selected slots that are not null copies
    int col = -1;
    float gk = 0.f, dgk = 0.f;
    if (lane < K) {
      const int id = __ldg(topk_idx + (size_t)t * K + lane);
      if (id < N) col = id;
      else if (id >= N + M) col = id - M + 1;
      if (col >= 0) {
        gk = __ldg(gate + (size_t)t * K + lane);
        dgk = __ldg(dg + (size_t)t * K + lane);
      }
    }
    const float mean = warp_sum(gk * dgk);
    __syncwarp();
    if (col >= 0) s_ds[w][col] += gk * (dgk - mean);
    __syncwarp();
    for (int j = lane; j < rows; j += 32) ds[(size_t)t * rows + j] = s_ds[w][j];
    if (dtnb && lane == 0) dtnb[t] = s_ds[w][N];
    uint16_t* sp = dsplit + (size_t)t * 2 * rp;
    for (int j = lane; j < rp; j += 32) {
      const float v = (j < rows) ? s_ds[w][j] : 0.f;
      const uint32_t hb = pack_bf16x2(v, 0.f) & 0xFFFFu;
      const float hv = __uint_as_float(hb << 16);
      const uint32_t lb = pack_bf16x2(v - hv, 0.f) & 0xFFFFu;
      sp[j] = (uint16_t)hb;
      sp[rp + j] = (uint16_t)lb;
    }
#pragma unroll
    for (int u = 0; u < 3; ++u) {
      const int j = lane + 32 * u;
      if (j < rows) bsum[u] += s_ds[w][j];
    }
    __syncwarp();
  }
  // the CTA's column sums, its warps added in order
  __syncthreads();
#pragma unroll
  for (int u = 0; u < 3; ++u) {
    const int j = lane + 32 * u;
    if (j < rows) s_ds[w][j] = bsum[u];
  }
  __syncthreads();
  for (int j = threadIdx.x; j < rows; j += kBwdThreads) {
    float acc = 0.f;
    for (int ww = 0; ww < kBwdThreads / 32; ++ww) acc += s_ds[ww][j];
    bpart[(size_t)blockIdx.x * rows + j] = acc;
  }
}

// W_r [rows, d] fp32 -> two bf16 terms W2 [2 RP, d]: rows j and RP + j hold hi = bf16(w) and
// lo = bf16(w - hi); rows past the router rows are zero.
__global__ void __launch_bounds__(kBwdThreads)
router_split2_kernel(const float* __restrict__ w, uint16_t* __restrict__ w2, int rows, int rp, int d) {
  pdl_wait_then_release();
  const long long n = (long long)rp * d;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const int j = (int)(i / d);
    const float v = (j < rows) ? __ldg(w + i) : 0.f;
    const uint32_t hb = pack_bf16x2(v, 0.f) & 0xFFFFu;
    const float hv = __uint_as_float(hb << 16);
    w2[i] = (uint16_t)hb;
    w2[n + i] = (uint16_t)(pack_bf16x2(v - hv, 0.f) & 0xFFFFu);
  }
}

// dW_r[j, c] = sum over K chunks of the two term rows j and RP + j of the chunk partials of
// dsplit^T x (in chunk order), and dbias[j] = sum of the per-CTA column sums of the router
// backward (one CTA per row j after the dW_r CTAs; fixed order within the CTA).
__global__ void __launch_bounds__(kBwdThreads)
router_wgrad_reduce_kernel(const float* __restrict__ part, int nchunk, int rp, const float* __restrict__ bpart,
                           int nparts, int rows, int d, float* __restrict__ dw, float* __restrict__ dbias,
                           int dw_ctas) {
  pdl_wait_then_release();
  if ((int)blockIdx.x >= dw_ctas) {
    __shared__ float s_red[kBwdThreads / 32];
    const int j = blockIdx.x - dw_ctas;
    float acc = 0.f;
    for (int i = threadIdx.x; i < nparts; i += kBwdThreads) acc += bpart[(size_t)i * rows + j];
    acc = warp_sum(acc);
    if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
      float t = 0.f;
      for (int ww = 0; ww < kBwdThreads / 32; ++ww) t += s_red[ww];
      dbias[j] = t;
    }
    return;
  }
  const long long n4 = (long long)rows * d / 4;
  const size_t slab = (size_t)2 * rp * d;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (long long)dw_ctas * blockDim.x) {
    const long long e = i * 4;
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
    for (int c = 0; c < nchunk; ++c) {
      const float4 h = __ldg(reinterpret_cast<const float4*>(part + c * slab + e));
      const float4 l = __ldg(reinterpret_cast<const float4*>(part + c * slab + (size_t)rp * d + e));
      a.x += h.x + l.x; a.y += h.y + l.y; a.z += h.z + l.z; a.w += h.w + l.w;
    }
    reinterpret_cast<float4*>(dw)[i] = a;
  }
}

// ---------------------------------------------------------------------------------------
// Constant experts' gradient: dconst[j] = sum over the tokens that selected constant
// expert j of g dy_t (fp32). Grid: (d / 256 column tiles) x V; 32 warps per CTA, each
// taking every 32nd block of 32 tokens (lane: 8 columns), then the 32 warp sums added in warp
// order, so the result is deterministic.
constexpr int kConstCols = 256;
constexpr int kConstWarps = 32;

__global__ void __launch_bounds__(kConstWarps * 32)
const_grad_kernel(const int32_t* __restrict__ topk_idx, const float* __restrict__ gate,
                  const uint16_t* __restrict__ dy, float* __restrict__ dconst, int T, int d, int K, int pool_id0) {
  pdl_wait_then_release();
  __shared__ __align__(16) float s_acc[kConstWarps][kConstCols];
  const int j = blockIdx.y;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int c0 = blockIdx.x * kConstCols;
  const int col = c0 + lane * 8;
  const bool colok = col < d;
  const int target = pool_id0 + j;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  // warp w takes blocks of 32 tokens (block index = w mod 32): each lane tests one token,
  // then the tokens that chose expert j are visited in ascending order
  for (int t0 = w * 32; t0 < T; t0 += kConstWarps * 32) {
    const int t = t0 + lane;
    float gj = 0.f;
    if (t < T)
      for (int k = 0; k < K; ++k)
        if (__ldg(topk_idx + (size_t)t * K + k) == target) gj = __ldg(gate + (size_t)t * K + k);
    unsigned m = __ballot_sync(0xffffffffu, gj != 0.f);
    while (m) {
      const int src = __ffs(m) - 1;
      m &= m - 1;
      const float g = __shfl_sync(0xffffffffu, gj, src);
      if (colok) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(dy + (size_t)(t0 + src) * d + col));
        acc[0] = fmaf(g, bf16lo(v.x), acc[0]); acc[1] = fmaf(g, bf16hi(v.x), acc[1]);
        acc[2] = fmaf(g, bf16lo(v.y), acc[2]); acc[3] = fmaf(g, bf16hi(v.y), acc[3]);
        acc[4] = fmaf(g, bf16lo(v.z), acc[4]); acc[5] = fmaf(g, bf16hi(v.z), acc[5]);
        acc[6] = fmaf(g, bf16lo(v.w), acc[6]); acc[7] = fmaf(g, bf16hi(v.w), acc[7]);
      }
    }
  }
#pragma unroll
  for (int u = 0; u < 8; ++u) s_acc[w][lane * 8 + u] = acc[u];
  __syncthreads();
  if (threadIdx.x < kConstCols && c0 + (int)threadIdx.x < d) {
    float sum = 0.f;
    for (int ww = 0; ww < kConstWarps; ++ww) sum += s_acc[ww][threadIdx.x];
    dconst[(size_t)j * d + c0 + threadIdx.x] = sum;
  }
}

// ---------------------------------------------------------------------------------------
// SwiGLU backward from saved pre-activations (training mode): for every routed row below
// offsets[N] and every shared row, dz = [da | db] with a, b the saved gate/up values (bf16,
// packed order: 64-column panels of 64 gate then 64 up columns) and dh the gradient of h:
// da = dh b sigma(a) (1 + a (1 - sigma(a))), db = dh a sigma(a). One item = 8 consecutive h
// columns (one 16-byte chunk of dh, two of z, two of dz).
__global__ void __launch_bounds__(kBwdThreads)
swiglu_bwd_saved_kernel(const int32_t* __restrict__ offsets, int N, long long rcap, const uint16_t* __restrict__ z,
                        const uint16_t* __restrict__ dh, uint16_t* __restrict__ dz, int F,
                        const uint16_t* __restrict__ zs, const uint16_t* __restrict__ dhs, uint16_t* __restrict__ dzs,
                        int Fs, int T, uint32_t* status) {
  pdl_wait_then_release();
  long long R = __ldg(offsets + N);
  if (R < 0 || R > rcap) {
    if (threadIdx.x == 0 && blockIdx.x == 0) atomicOr(status, kStatusBounds);
    R = 0;
  }
  const long long cr = F / 8, cs = Fs / 8;
  const long long n_r = R * cr, n_all = n_r + (long long)T * cs;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n_all; i += (long long)gridDim.x * blockDim.x) {
    const bool routed = i < n_r;
    const long long k = routed ? i : i - n_r;
    const long long cpr = routed ? cr : cs;
    const long long row = k / cpr;
    const int f = (int)(k - row * cpr) * 8;
    const int w = routed ? F : Fs;
    const uint16_t* zr = (routed ? z : zs) + (size_t)row * 2 * w + (f >> 6) * 128 + (f & 63);
    const uint4 hv = __ldg(reinterpret_cast<const uint4*>((routed ? dh : dhs) + (size_t)row * w + f));
    const uint4 gv = __ldg(reinterpret_cast<const uint4*>(zr));
    const uint4 uv = __ldg(reinterpret_cast<const uint4*>(zr + 64));
    const uint32_t hw[4] = {hv.x, hv.y, hv.z, hv.w}, gw[4] = {gv.x, gv.y, gv.z, gv.w}, uw[4] = {uv.x, uv.y, uv.z, uv.w};
    uint32_t og[4], ou[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float da[2], db[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float a = h ? bf16hi(gw[j]) : bf16lo(gw[j]);
        const float b = h ? bf16hi(uw[j]) : bf16lo(uw[j]);
        const float g = h ? bf16hi(hw[j]) : bf16lo(hw[j]);
        const float sg = __fdividef(1.f, 1.f + __expf(-a));
        db[h] = g * a * sg;
        da[h] = g * b * sg * (1.f + a * (1.f - sg));
      }
      og[j] = pack_bf16x2(da[0], da[1]);
      ou[j] = pack_bf16x2(db[0], db[1]);
    }
    uint16_t* dr = (routed ? dz : dzs) + (size_t)row * 2 * w + (f >> 6) * 128 + (f & 63);
    *reinterpret_cast<uint4*>(dr) = make_uint4(og[0], og[1], og[2], og[3]);
    *reinterpret_cast<uint4*>(dr + 64) = make_uint4(ou[0], ou[1], ou[2], ou[3]);
  }
}

// ---------------------------------------------------------------------------------------
// Host launchers.

static int grid_warps(long long items, int occ_cap) {
  const int wpb = kBwdThreads / 32;
  long long g = (items + wpb - 1) / wpb;
  if (g > occ_cap) g = occ_cap;
  return g < 1 ? 1 : (int)g;
}

int launch_combine_bwd(const moe_dims_t& d, const uint16_t* dy, const uint16_t* ys, const float* topk_gate,
                       const int32_t* slot_row, const int32_t* topk_idx, const uint16_t* x,
                       const uint16_t* const_vectors, uint16_t* dys, float* dg, uint32_t* status, cudaStream_t st) {
  const int grid = grid_warps(d.T, sm_count() * 8);
  return launch_pdl(combine_bwd_kernel, dim3(grid), dim3(kBwdThreads), 0, st, dy, ys, topk_gate, slot_row, topk_idx,
                    x, const_vectors, dys, dg, d.T, d.d, d.K, (long long)d.T * d.K, d.N + d.M, d.C, d.V, status);
}

int router_bwd_grid(const moe_dims_t& d) {
  const int wpb = kBwdThreads / 32;
  int g = (d.T + wpb - 1) / wpb;
  if (g > kRouterBwdMaxGrid) g = kRouterBwdMaxGrid;
  return g < 1 ? 1 : g;
}

int launch_router_bwd(const moe_dims_t& d, const float* logits, const int32_t* topk_idx, const float* topk_gate,
                      const float* dg, const int32_t* counts_ext, long long t_total, float alpha, float beta,
                      float* ds, float* dtnb, uint16_t* dsplit, float* bpart, cudaStream_t st) {
  return launch_pdl(router_bwd_kernel, dim3(router_bwd_grid(d)), dim3(kBwdThreads), 0, st, logits, topk_idx,
                    topk_gate, dg, counts_ext, 1.0 / (double)t_total, alpha, beta, ds, dtnb, dsplit,
                    router_split_rows(d), bpart, d.T, d.N, d.M, d.K, d.C, d.V);
}

int launch_router_split2(const moe_dims_t& d, const float* w_router, uint16_t* w2, cudaStream_t st) {
  const int rp = router_split_rows(d);
  long long n = (long long)rp * d.d;
  long long g = (n + kBwdThreads - 1) / kBwdThreads;
  if (g > sm_count() * 4) g = sm_count() * 4;
  return launch_pdl(router_split2_kernel, dim3((unsigned)g), dim3(kBwdThreads), 0, st, w_router, w2,
                    router_rows(d), rp, d.d);
}

int launch_router_wgrad_reduce(const moe_dims_t& d, const float* part, int nchunk, const float* bpart, float* dw,
                               float* dbias, cudaStream_t st) {
  const int rows = router_rows(d);
  long long n4 = (long long)rows * d.d / 4;
  long long g = (n4 + kBwdThreads - 1) / kBwdThreads;
  if (g > sm_count() * 4) g = sm_count() * 4;
  const int extra = dbias ? rows : 0;
  return launch_pdl(router_wgrad_reduce_kernel, dim3((unsigned)(g + extra)), dim3(kBwdThreads), 0, st, part, nchunk,
                    router_split_rows(d), bpart, router_bwd_grid(d), rows, d.d, dw, dbias, (int)g);
}

int launch_const_grad(const moe_dims_t& d, const int32_t* topk_idx, const float* topk_gate, const uint16_t* dy,
                      float* dconst, cudaStream_t st) {
  if (d.V == 0) return MOE_OK;
  const dim3 grid((d.d + kConstCols - 1) / kConstCols, d.V);
  return launch_pdl(const_grad_kernel, grid, dim3(kConstWarps * 32), 0, st, topk_idx, topk_gate, dy, dconst, d.T, d.d, d.K,
                    d.N + d.M + d.C);
}

int launch_swiglu_bwd_saved(const moe_dims_t& d, const int32_t* offsets, const uint16_t* z, const uint16_t* zs,
                            const uint16_t* dh, const uint16_t* dhs, uint16_t* dz, uint16_t* dzs, uint32_t* status,
                            cudaStream_t st) {
  return launch_pdl(swiglu_bwd_saved_kernel, dim3(sm_count() * 8), dim3(kBwdThreads), 0, st, offsets, d.N,
                    (long long)d.T * d.K, z, dh, dz, d.F, zs, dhs, dzs, d.F_shared, d.T, status);
}

}  // namespace moe
