// router.cu -- the Layer Router on sm_100a (gist.science summary "Flux
// Attention", section 2 "Methodology": "Layer Router" mean-pools the first
// and last 100 prompt tokens and runs a context-encoder MLP; "switch to hard
// routing" thresholds the soft weight into one 0/1 bit per layer at
// inference; "efficient deployment" does this once, at prefill).
//
// Two launches, no host sync:
//   pool_kernel   grid (Hd/256 column groups, 2 sides): each thread sums
//                 16-byte bf16 vectors of its rows, fixed-order shared-memory
//                 reduction -> pooled[2 Hd] (fp32).
//   mlp_kernel    four warps per hidden unit: u = relu(W1 p + b1) with W1 rows
//                 streamed by unrolled 128-bit loads; the last CTA (atomic
//                 ticket, no spin) computes z = W2 u + b2, r = sigmoid(z) and
//                 layer_mode = (r > thresh).
#include "common.cuh"
#include "kernels.h"

namespace flux {

namespace {

constexpr int kPoolThreads = 256;  // 32 column groups of 8 x 8 row groups
constexpr int kMlpWarps = 8;
constexpr int kWarpsPerRow = 4;
constexpr int kRowsPerCta = kMlpWarps / kWarpsPerRow;

__global__ void __launch_bounds__(kPoolThreads)
    pool_kernel(const uint16_t* __restrict__ hidden, int T, int Hd, int n_pool,
                float* __restrict__ pooled) {
  __shared__ float part[8][256];
  const int side = blockIdx.y;  // 0: first rows, 1: last rows
  const int n = min(n_pool, T);
  const int row0 = side == 0 ? 0 : T - n;
  const int cg = threadIdx.x & 31, rg = threadIdx.x >> 5;
  const int c0 = blockIdx.x * 256 + cg * 8;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  if (c0 + 8 <= Hd && (Hd & 7) == 0) {
    for (int t = rg; t < n; t += 8) {
      const uint4 w =
          *reinterpret_cast<const uint4*>(hidden + static_cast<size_t>(row0 + t) * Hd + c0);
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc[2 * e] += bf16lo_to_f32(ws[e]);
        acc[2 * e + 1] += bf16hi_to_f32(ws[e]);
      }
    }
  } else {
    for (int t = rg; t < n; t += 8)
      for (int e = 0; e < 8 && c0 + e < Hd; ++e)
        acc[e] += __uint_as_float(
            static_cast<uint32_t>(hidden[static_cast<size_t>(row0 + t) * Hd + c0 + e]) << 16);
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) part[rg][cg * 8 + e] = acc[e];
  __syncthreads();
  const int c = blockIdx.x * 256 + threadIdx.x;
  if (c < Hd) {
    float s = 0.f;
#pragma unroll
    for (int r = 0; r < 8; ++r) s += part[r][threadIdx.x];
    pooled[side * Hd + c] = s / static_cast<float>(n);
  }
}

__global__ void __launch_bounds__(kMlpWarps * 32)
    mlp_kernel(const float* __restrict__ pooled, int in_dim, const float* __restrict__ W1,
               const float* __restrict__ b1, int H1, const float* __restrict__ W2,
               const float* __restrict__ b2, int L, float thresh, float* __restrict__ hidden1,
               int* ticket, uint8_t* __restrict__ layer_mode, float* __restrict__ score) {
  __shared__ int last;
  __shared__ float part[kMlpWarps];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // kRowsPerCta hidden units per CTA, kWarpsPerRow warps share one unit's dot product.
  const int j = blockIdx.x * kRowsPerCta + warp / kWarpsPerRow;
  const int wr = warp % kWarpsPerRow;
  float acc = 0.f;
  if (j < H1) {
    const float* w = W1 + static_cast<size_t>(j) * in_dim;
    if ((in_dim & 3) == 0) {
      const int n4 = in_dim >> 2;
#pragma unroll 4
      for (int i4 = wr * 32 + lane; i4 < n4; i4 += 32 * kWarpsPerRow) {
        const float4 wv = __ldg(reinterpret_cast<const float4*>(w) + i4);
        const float4 pv = *(reinterpret_cast<const float4*>(pooled) + i4);
        acc = fmaf(wv.x, pv.x, acc);
        acc = fmaf(wv.y, pv.y, acc);
        acc = fmaf(wv.z, pv.z, acc);
        acc = fmaf(wv.w, pv.w, acc);
      }
    } else {
      for (int i = wr * 32 + lane; i < in_dim; i += 32 * kWarpsPerRow)
        acc = fmaf(__ldg(w + i), pooled[i], acc);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) part[warp] = acc;
  __syncthreads();
  if (threadIdx.x < kRowsPerCta) {
    const int jj = blockIdx.x * kRowsPerCta + threadIdx.x;
    if (jj < H1) {
      float t = 0.f;
      for (int q = 0; q < kWarpsPerRow; ++q) t += part[threadIdx.x * kWarpsPerRow + q];
      hidden1[jj] = fmaxf(t + b1[jj], 0.f);
    }
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) last = (atomicAdd(ticket, 1) == static_cast<int>(gridDim.x) - 1);
  __syncthreads();
  if (!last) return;
  __threadfence();
  for (int l = warp; l < L; l += kMlpWarps) {
    const float* w = W2 + static_cast<size_t>(l) * H1;
    float acc = 0.f;
    for (int i = lane; i < H1; i += 32) acc = fmaf(__ldg(w + i), __ldcg(hidden1 + i), acc);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) {
      const float z = acc + b2[l];
      const float r = 1.f / (1.f + expf(-z));
      layer_mode[l] = r > thresh ? 1 : 0;
      if (score) score[l] = r;
    }
  }
  if (threadIdx.x == 0) *ticket = 0;
}

}  // namespace

size_t route_workspace_bytes(int Hd, int H1) {
  return static_cast<size_t>(2 * Hd + H1) * sizeof(float) + 64;
}

cudaError_t launch_route(const RouteLaunch& p, cudaStream_t stream) {
  const dim3 pgrid((p.Hd + 255) / 256, 2);
  pool_kernel<<<pgrid, kPoolThreads, 0, stream>>>(p.hidden, p.T, p.Hd, p.n_pool, p.pooled);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int grid = (p.H1 + kRowsPerCta - 1) / kRowsPerCta;
  mlp_kernel<<<grid, kMlpWarps * 32, 0, stream>>>(p.pooled, 2 * p.Hd, p.W1, p.b1, p.H1, p.W2,
                                                  p.b2, p.L, p.thresh, p.hidden1, p.ticket,
                                                  p.layer_mode, p.score);
  return cudaGetLastError();
}

}  // namespace flux
