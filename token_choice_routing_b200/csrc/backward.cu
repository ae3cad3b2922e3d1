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
// One warp per token; dot products in fp32, reduced across the warp in a fixed order.
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
    for (int k = 0; k < K; ++k) {
      const int rk = __shfl_sync(0xffffffffu, row, k);
      const float gk = __shfl_sync(0xffffffffu, g, k);
      if (rk == -1) continue;
      const uint16_t* src = (rk >= 0) ? ys + (size_t)rk * d : (rk == -2) ? x + (size_t)t * d : cv + (size_t)(-3 - rk) * d;
      const uint4* sr = reinterpret_cast<const uint4*>(src);
      uint4* dst = (rk >= 0) ? reinterpret_cast<uint4*>(dys + (size_t)rk * d) : nullptr;
      float s = 0.f;
#pragma unroll 4
      for (int c = lane; c < nch; c += 32) {
        const uint4 a = __ldg(dyr + c);
        const uint4 b = __ldg(sr + c);
        s += dot8(a, b);
        if (dst) dst[c] = scale8(gk, a);
      }
      s = warp_sum(s);
      if (lane == k) mydg = s;
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
__global__ void __launch_bounds__(kBwdThreads)
router_bwd_kernel(const float* __restrict__ logits, const int32_t* __restrict__ topk_idx,
                  const float* __restrict__ gate, const float* __restrict__ dg,
                  const int32_t* __restrict__ counts_ext, double inv_t, float alpha, float beta,
                  float* __restrict__ ds, float* __restrict__ dtnb, int T, int N, int M, int K, int C, int V) {
  pdl_wait_then_release();
  __shared__ float s_ds[kBwdThreads / 32][kMaxRows];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int rows = N + 1 + C + V;
  const float invT = (float)inv_t;
  // null copies' load fraction (sum over the M copies), the same for every token
  float fnull = 0.f;
  for (int c = lane; c < M; c += 32) fnull += (float)__ldg(counts_ext + N + c);
  fnull = warp_sum(fnull) * invT;
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
    __syncwarp();
  }
}

// ---------------------------------------------------------------------------------------
// Router weight gradient dW_r = ds^T x and dbias = sum_t ds, on the fp32 CUDA cores.
// Grid: (d / 256 column tiles) x (token chunks). A CTA stages 32 tokens at a time (ds
// [32 x rows], x [32 x 256] widened from bf16) and accumulates a rows x 256 tile, 10 rows
// x 8 columns per thread; partials of every chunk go to a buffer that the reduce kernel
// sums in chunk order, so the result is deterministic.
constexpr int kRwRows = 80;   // row capacity (kMaxRows)
constexpr int kRwCols = 256;
constexpr int kRwSub = 32;

__global__ void __launch_bounds__(kBwdThreads)
router_wgrad_kernel(const float* __restrict__ ds, const uint16_t* __restrict__ x, float* __restrict__ part,
                    float* __restrict__ bpart, int T, int d, int rows, int chunk) {
  pdl_wait_then_release();
  __shared__ float s_ds[kRwSub][kRwRows];
  __shared__ __align__(16) float s_x[kRwSub][kRwCols];
  const int tid = threadIdx.x;
  const int jg = tid >> 5;   // rows jg*10 .. jg*10+9
  const int cg = tid & 31;   // columns cg*8 .. cg*8+7
  const int c0 = blockIdx.x * kRwCols;
  const int t0 = blockIdx.y * chunk, t1 = min(T, t0 + chunk);
  float acc[10][8];
#pragma unroll
  for (int i = 0; i < 10; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
  float bsum = 0.f;  // thread tid < rows: its row's ds sum (column tile 0 only)
  for (int tb = t0; tb < t1; tb += kRwSub) {
    const int nt = min(kRwSub, t1 - tb);
    __syncthreads();
    for (int i = tid; i < kRwSub * kRwRows; i += kBwdThreads) {
      const int tt = i / kRwRows, j = i - tt * kRwRows;
      s_ds[tt][j] = (tt < nt && j < rows) ? __ldg(ds + (size_t)(tb + tt) * rows + j) : 0.f;
    }
    for (int i = tid; i < kRwSub * (kRwCols / 8); i += kBwdThreads) {
      const int tt = i / (kRwCols / 8), ch = i - tt * (kRwCols / 8);
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (tt < nt && c0 + ch * 8 < d) v = __ldg(reinterpret_cast<const uint4*>(x + (size_t)(tb + tt) * d + c0) + ch);
      float4* dst = reinterpret_cast<float4*>(&s_x[tt][ch * 8]);
      dst[0] = make_float4(bf16lo(v.x), bf16hi(v.x), bf16lo(v.y), bf16hi(v.y));
      dst[1] = make_float4(bf16lo(v.z), bf16hi(v.z), bf16lo(v.w), bf16hi(v.w));
    }
    __syncthreads();
    if (blockIdx.x == 0 && tid < rows)
      for (int tt = 0; tt < nt; ++tt) bsum += s_ds[tt][tid];
    for (int tt = 0; tt < nt; ++tt) {
      const float4 xa = *reinterpret_cast<const float4*>(&s_x[tt][cg * 8]);
      const float4 xb = *reinterpret_cast<const float4*>(&s_x[tt][cg * 8 + 4]);
      const float xv[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
#pragma unroll
      for (int i = 0; i < 10; ++i) {
        const float dv = s_ds[tt][jg * 10 + i];
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(dv, xv[j], acc[i][j]);
      }
    }
  }
  float* P = part + (size_t)blockIdx.y * rows * d;
#pragma unroll
  for (int i = 0; i < 10; ++i) {
    const int j = jg * 10 + i;
    const int c = c0 + cg * 8;
    if (j < rows && c < d) {
      float4* dst = reinterpret_cast<float4*>(P + (size_t)j * d + c);
      dst[0] = make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
      dst[1] = make_float4(acc[i][4], acc[i][5], acc[i][6], acc[i][7]);
    }
  }
  if (blockIdx.x == 0 && tid < rows) bpart[(size_t)blockIdx.y * rows + tid] = bsum;
}

__global__ void __launch_bounds__(kBwdThreads)
router_wgrad_reduce_kernel(const float* __restrict__ part, const float* __restrict__ bpart, int nchunk, int rows,
                           int d, float* __restrict__ dw, float* __restrict__ dbias) {
  pdl_wait_then_release();
  const long long n4 = (long long)rows * d / 4;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (long long)gridDim.x * blockDim.x) {
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int c = 0; c < nchunk; ++c) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(part + (size_t)c * rows * d) + i);
      a.x += v.x; a.y += v.y; a.z += v.z; a.w += v.w;
    }
    reinterpret_cast<float4*>(dw)[i] = a;
  }
  if (dbias && blockIdx.x == 0)
    for (int j = threadIdx.x; j < rows; j += blockDim.x) {
      float s = 0.f;
      for (int c = 0; c < nchunk; ++c) s += bpart[(size_t)c * rows + j];
      dbias[j] = s;
    }
}

// ---------------------------------------------------------------------------------------
// Input gradient: dx[t] = dx_shared[t] + sum over real slots of dxs[row] + sum over copy
// slots of g dy[t] + sum_j ds[t, j] W_r[j, :], accumulated in fp32, rounded once to bf16.
// CTA = 64 tokens x 256 columns: W_r's 256-column slice and the tokens' ds rows in shared
// memory, 8 tokens x 8 columns per thread (warp w: tokens 8w..8w+7, lane: 8 columns).
constexpr int kIgTok = 64;

__global__ void __launch_bounds__(kBwdThreads)
input_grad_kernel(const uint16_t* __restrict__ dx_shared, const uint16_t* __restrict__ dxs,
                  const int32_t* __restrict__ slot_row, const int32_t* __restrict__ topk_idx,
                  const float* __restrict__ gate, const uint16_t* __restrict__ dy, const float* __restrict__ ds,
                  const float* __restrict__ w_r, uint16_t* __restrict__ dx, int T, int d, int K, int rows,
                  long long rcap, int NM, int C, uint32_t* status) {
  pdl_wait_then_release();
  extern __shared__ __align__(16) float sm_ig[];
  float* s_w = sm_ig;                          // [rows][256]
  float* s_ds = sm_ig + (size_t)rows * kRwCols;  // [64][rows]
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int c0 = blockIdx.x * kRwCols;
  const int ncol = min(kRwCols, d - c0);
  for (int i = tid; i < rows * (kRwCols / 4); i += kBwdThreads) {
    const int j = i / (kRwCols / 4), c4 = i - j * (kRwCols / 4);
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (c4 * 4 < ncol) v = __ldg(reinterpret_cast<const float4*>(w_r + (size_t)j * d + c0) + c4);
    reinterpret_cast<float4*>(s_w + (size_t)j * kRwCols)[c4] = v;
  }
  const int col = c0 + lane * 8;
  const bool colok = lane * 8 < ncol;
  for (int tb = blockIdx.y * kIgTok; tb < T; tb += gridDim.y * kIgTok) {
    __syncthreads();
    for (int i = tid; i < kIgTok * rows; i += kBwdThreads) {
      const int tt = i / rows, j = i - tt * rows;
      s_ds[i] = (tb + tt < T) ? __ldg(ds + (size_t)(tb + tt) * rows + j) : 0.f;
    }
    __syncthreads();
    float acc[8][8];
#pragma unroll
    for (int u = 0; u < 8; ++u)
#pragma unroll
      for (int v = 0; v < 8; ++v) acc[u][v] = 0.f;
    for (int j = 0; j < rows; ++j) {
      const float4 wa = *reinterpret_cast<const float4*>(s_w + (size_t)j * kRwCols + lane * 8);
      const float4 wb = *reinterpret_cast<const float4*>(s_w + (size_t)j * kRwCols + lane * 8 + 4);
      const float wv[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const float dv = s_ds[(w * 8 + u) * rows + j];
#pragma unroll
        for (int v = 0; v < 8; ++v) acc[u][v] = fmaf(dv, wv[v], acc[u][v]);
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int t = tb + w * 8 + u;
      if (t >= T || !colok) continue;
      float a[8];
#pragma unroll
      for (int v = 0; v < 8; ++v) a[v] = acc[u][v];
      const uint4 sv = __ldg(reinterpret_cast<const uint4*>(dx_shared + (size_t)t * d + col));
      a[0] += bf16lo(sv.x); a[1] += bf16hi(sv.x); a[2] += bf16lo(sv.y); a[3] += bf16hi(sv.y);
      a[4] += bf16lo(sv.z); a[5] += bf16hi(sv.z); a[6] += bf16lo(sv.w); a[7] += bf16hi(sv.w);
      for (int k = 0; k < K; ++k) {
        int row = __ldg(slot_row + (size_t)t * K + k);
        float gk = 1.f;
        const uint16_t* src = nullptr;
        if (row >= 0) {
          if (row >= rcap) {
            atomicOr(status, kStatusBounds);
            continue;
          }
          src = dxs + (size_t)row * d;
        } else if (C > 0) {
          const int id = __ldg(topk_idx + (size_t)t * K + k) - NM;
          if (id >= 0 && id < C) {
            src = dy + (size_t)t * d;
            gk = __ldg(gate + (size_t)t * K + k);
          }
        }
        if (!src) continue;
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(src + col));
        a[0] = fmaf(gk, bf16lo(v.x), a[0]); a[1] = fmaf(gk, bf16hi(v.x), a[1]);
        a[2] = fmaf(gk, bf16lo(v.y), a[2]); a[3] = fmaf(gk, bf16hi(v.y), a[3]);
        a[4] = fmaf(gk, bf16lo(v.z), a[4]); a[5] = fmaf(gk, bf16hi(v.z), a[5]);
        a[6] = fmaf(gk, bf16lo(v.w), a[6]); a[7] = fmaf(gk, bf16hi(v.w), a[7]);
      }
      *reinterpret_cast<uint4*>(dx + (size_t)t * d + col) =
          make_uint4(pack_bf16x2(a[0], a[1]), pack_bf16x2(a[2], a[3]), pack_bf16x2(a[4], a[5]),
                     pack_bf16x2(a[6], a[7]));
    }
  }
}

// ---------------------------------------------------------------------------------------
// Constant experts' gradient: dconst[j] = sum over the tokens that selected constant
// expert j of g dy_t (fp32, token order). Grid: (d / 256 column tiles) x V.
__global__ void __launch_bounds__(kBwdThreads)
const_grad_kernel(const int32_t* __restrict__ topk_idx, const float* __restrict__ gate,
                  const uint16_t* __restrict__ dy, float* __restrict__ dconst, int T, int d, int K, int pool_id0) {
  pdl_wait_then_release();
  __shared__ float s_g[kBwdThreads];
  const int j = blockIdx.y;
  const int c = blockIdx.x * kRwCols + threadIdx.x;
  const int target = pool_id0 + j;
  float acc = 0.f;
  for (int tb = 0; tb < T; tb += kBwdThreads) {
    // gate of constant expert j for each of 256 tokens (0 if the token did not select it)
    const int t = tb + threadIdx.x;
    float gj = 0.f;
    if (t < T)
      for (int k = 0; k < K; ++k)
        if (__ldg(topk_idx + (size_t)t * K + k) == target) gj = __ldg(gate + (size_t)t * K + k);
    __syncthreads();
    s_g[threadIdx.x] = gj;
    __syncthreads();
    const int nt = min(kBwdThreads, T - tb);
    for (int u = 0; u < nt; ++u) {
      const float g = s_g[u];
      if (g != 0.f && c < d) acc = fmaf(g, __uint_as_float((uint32_t)dy[(size_t)(tb + u) * d + c] << 16), acc);
    }
  }
  if (c < d) dconst[(size_t)j * d + c] = acc;
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

int launch_router_bwd(const moe_dims_t& d, const float* logits, const int32_t* topk_idx, const float* topk_gate,
                      const float* dg, const int32_t* counts_ext, long long t_total, float alpha, float beta,
                      float* ds, float* dtnb, cudaStream_t st) {
  const int grid = grid_warps(d.T, sm_count() * 8);
  return launch_pdl(router_bwd_kernel, dim3(grid), dim3(kBwdThreads), 0, st, logits, topk_idx, topk_gate, dg,
                    counts_ext, 1.0 / (double)t_total, alpha, beta, ds, dtnb, d.T, d.N, d.M, d.K, d.C, d.V);
}

// token chunks of the router weight gradient: about two CTAs per SM over all column tiles
int router_wgrad_chunks(const moe_dims_t& d, int* chunk_tokens) {
  const int ctiles = (d.d + kRwCols - 1) / kRwCols;
  int nch = (2 * 148 + ctiles - 1) / ctiles;
  const int maxch = (d.T + kRwSub - 1) / kRwSub;
  if (nch > maxch) nch = maxch;
  if (nch < 1) nch = 1;
  int ct = (d.T + nch - 1) / nch;
  ct = (ct + kRwSub - 1) / kRwSub * kRwSub;
  if (ct < kRwSub) ct = kRwSub;
  nch = (d.T + ct - 1) / ct;
  if (nch < 1) nch = 1;
  if (chunk_tokens) *chunk_tokens = ct;
  return nch;
}

int launch_router_wgrad(const moe_dims_t& d, const float* ds, const uint16_t* x, float* part, float* bpart,
                        float* dw_router, float* dbias, cudaStream_t st) {
  const int rows = router_rows(d);
  int ct = 0;
  const int nch = router_wgrad_chunks(d, &ct);
  const dim3 grid((d.d + kRwCols - 1) / kRwCols, nch);
  int r = launch_pdl(router_wgrad_kernel, grid, dim3(kBwdThreads), 0, st, ds, x, part, bpart, d.T, d.d, rows, ct);
  if (r != MOE_OK) return r;
  long long n4 = (long long)rows * d.d / 4;
  long long g = (n4 + kBwdThreads - 1) / kBwdThreads;
  if (g > sm_count() * 4) g = sm_count() * 4;
  return launch_pdl(router_wgrad_reduce_kernel, dim3((unsigned)g), dim3(kBwdThreads), 0, st, (const float*)part,
                    (const float*)bpart, nch, rows, d.d, dw_router, dbias);
}

int launch_input_grad(const moe_dims_t& d, const uint16_t* dx_shared, const uint16_t* dxs, const int32_t* slot_row,
                      const int32_t* topk_idx, const float* topk_gate, const uint16_t* dy, const float* ds,
                      const float* w_router, uint16_t* dx, uint32_t* status, cudaStream_t st) {
  const int rows = router_rows(d);
  const size_t smem = sizeof(float) * ((size_t)rows * kRwCols + (size_t)kIgTok * rows);
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(input_grad_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)(sizeof(float) * ((size_t)kMaxRows * kRwCols + (size_t)kIgTok * kMaxRows)));
    if (e != cudaSuccess) return cuda_status(e);
    attr_set[dev] = true;
  }
  const int ctiles = (d.d + kRwCols - 1) / kRwCols;
  int gy = (d.T + kIgTok - 1) / kIgTok;
  const int cap = (2 * sm_count() + ctiles - 1) / ctiles;
  if (gy > cap) gy = cap;
  if (gy < 1) gy = 1;
  return launch_pdl(input_grad_kernel, dim3(ctiles, gy), dim3(kBwdThreads), smem, st, dx_shared, dxs, slot_row,
                    topk_idx, topk_gate, dy, ds, w_router, dx, d.T, d.d, d.K, rows, (long long)d.T * d.K, d.N + d.M,
                    d.C, status);
}

int launch_const_grad(const moe_dims_t& d, const int32_t* topk_idx, const float* topk_gate, const uint16_t* dy,
                      float* dconst, cudaStream_t st) {
  if (d.V == 0) return MOE_OK;
  const dim3 grid((d.d + kRwCols - 1) / kRwCols, d.V);
  return launch_pdl(const_grad_kernel, grid, dim3(kRwCols), 0, st, topk_idx, topk_gate, dy, dconst, d.T, d.d, d.K,
                    d.N + d.M + d.C);
}

}  // namespace moe
