// moe_combine: y[t] = E_shared(x_t) + sum over the token's real slots of
// g_{t,k} * E_e(x_t) (Kilian et al., "Improving MoE Compute Efficiency by
// Composing Weight and Data Sparsity", review page, section 三 / 核心公式).
// Null experts output zero, so null slots (slot_row = -1) are skipped.
// Written as a gather (each token reads its own rows of ys) so it is
// deterministic: fp32 accumulation in rank order, one bf16 rounding.
#include "moe_internal.cuh"

namespace moe {

constexpr int kCombineThreads = 256;

__global__ void __launch_bounds__(kCombineThreads)
combine_kernel(const uint16_t* __restrict__ ys, const uint16_t* __restrict__ sh,
               const float* __restrict__ gate, const int32_t* __restrict__ slot_row,
               uint16_t* __restrict__ y, int T, int d, int K, long long rcap, uint32_t* status) {
  const int lane = threadIdx.x & 31;
  const int wpb = kCombineThreads / 32;
  const int nch = d >> 3;
  for (int t = blockIdx.x * wpb + (threadIdx.x >> 5); t < T; t += gridDim.x * wpb) {
    int row = -1;
    float g = 0.f;
    if (lane < K) {
      row = __ldg(slot_row + (size_t)t * K + lane);
      g = __ldg(gate + (size_t)t * K + lane);
      if (row >= rcap) {
        if (status) atomicOr(status, kStatusBounds);
        row = -1;
      }
    }
    for (int c0 = 0; c0 < nch; c0 += 64) {  // two 16-byte chunks per lane per pass
      float acc[2][8];
      bool ok[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int c = c0 + 32 * h + lane;
        ok[h] = c < nch;
        const uint4 v = ok[h] ? __ldg(reinterpret_cast<const uint4*>(sh + (size_t)t * d) + c)
                              : make_uint4(0u, 0u, 0u, 0u);
        acc[h][0] = bf16lo(v.x); acc[h][1] = bf16hi(v.x); acc[h][2] = bf16lo(v.y); acc[h][3] = bf16hi(v.y);
        acc[h][4] = bf16lo(v.z); acc[h][5] = bf16hi(v.z); acc[h][6] = bf16lo(v.w); acc[h][7] = bf16hi(v.w);
      }
      // slots in rank order, four at a time: issue the real rows' loads before using any
      for (int k0 = 0; k0 < K; k0 += 4) {
        uint4 v[4][2];
        float gq[4];
        int rq[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int k = k0 + u;
          rq[u] = __shfl_sync(0xffffffffu, row, k & 31);
          gq[u] = __shfl_sync(0xffffffffu, g, k & 31);
          if (k >= K) rq[u] = -1;
#pragma unroll
          for (int h = 0; h < 2; ++h)
            v[u][h] = (rq[u] >= 0 && ok[h])
                          ? __ldg(reinterpret_cast<const uint4*>(ys + (size_t)rq[u] * d) + c0 + 32 * h + lane)
                          : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if (rq[u] >= 0) {
            const float gk = gq[u];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              acc[h][0] = fmaf(gk, bf16lo(v[u][h].x), acc[h][0]); acc[h][1] = fmaf(gk, bf16hi(v[u][h].x), acc[h][1]);
              acc[h][2] = fmaf(gk, bf16lo(v[u][h].y), acc[h][2]); acc[h][3] = fmaf(gk, bf16hi(v[u][h].y), acc[h][3]);
              acc[h][4] = fmaf(gk, bf16lo(v[u][h].z), acc[h][4]); acc[h][5] = fmaf(gk, bf16hi(v[u][h].z), acc[h][5]);
              acc[h][6] = fmaf(gk, bf16lo(v[u][h].w), acc[h][6]); acc[h][7] = fmaf(gk, bf16hi(v[u][h].w), acc[h][7]);
            }
          }
        }
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        if (ok[h]) {
          uint4 o;
          o.x = pack_bf16x2(acc[h][0], acc[h][1]);
          o.y = pack_bf16x2(acc[h][2], acc[h][3]);
          o.z = pack_bf16x2(acc[h][4], acc[h][5]);
          o.w = pack_bf16x2(acc[h][6], acc[h][7]);
          reinterpret_cast<uint4*>(y + (size_t)t * d)[c0 + 32 * h + lane] = o;
        }
      }
    }
  }
}

int launch_combine(const moe_dims_t& d, const uint16_t* ys, const uint16_t* shared_out,
                   const float* topk_gate, const int32_t* slot_row, uint16_t* y, cudaStream_t st) {
  // one wave of resident CTAs; each warp then loops over tokens
  static int per_sm[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  int occ = (dev >= 0 && dev < 64) ? per_sm[dev] : 0;
  if (occ == 0) {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, combine_kernel, kCombineThreads, 0) != cudaSuccess ||
        occ < 1)
      occ = 1;
    if (dev >= 0 && dev < 64) per_sm[dev] = occ;
  }
  const int wpb = kCombineThreads / 32;
  int grid = (d.T + wpb - 1) / wpb;
  const int cap = sm_count() * occ;
  if (grid > cap) grid = cap;
  combine_kernel<<<grid, kCombineThreads, 0, st>>>(ys, shared_out, topk_gate, slot_row, y, d.T, d.d, d.K,
                                                   (long long)d.T * d.K, nullptr);
  return cuda_status(cudaGetLastError());
}

}  // namespace moe
