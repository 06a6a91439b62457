// router.cu -- the Layer Router on sm_100a (gist.science summary "Flux
// Attention", section 2 "Methodology": "Layer Router" mean-pools the first
// and last 100 prompt tokens and runs a context-encoder MLP; "switch to hard
// routing" thresholds the soft weight into one 0/1 bit per layer at
// inference; "efficient deployment" does this once, at prefill).
//
// Two launches, no host sync, overlapped by programmatic dependent launch:
//   pool_kernel   grid (Hd/256 column groups, 2 sides): each thread issues the
//                 16-byte bf16 loads of all its rows at once, then sums them;
//                 fixed-order shared-memory reduction -> pooled[2 Hd] (fp32).
//                 It lets the MLP launch at once.
//   mlp_kernel    four warps per hidden unit.  Each warp loads its slice of
//                 the unit's W1 row (128-bit loads) before waiting for the
//                 pool, so the weight stream -- nearly all of the router's
//                 bytes -- overlaps the pooling; then u = relu(W1 p + b1).  The
//                 last CTA (atomic ticket, no spin) computes z = W2 u + b2 with
//                 128-bit loads, r = sigmoid(z) and layer_mode = (r > thresh).
#include "common.cuh"
#include "kernels.h"

namespace flux {

namespace {

constexpr int kPoolThreads = 256;  // 32 column groups of 8 x 8 row groups
constexpr int kRowGroups = 8;
constexpr int kPoolRowsPerThread = 13;   // loads in flight per thread: n_pool <= 104
constexpr int kMlpWarps = 8;
constexpr int kWarpsPerRow = 4;
constexpr int kRowsPerCta = kMlpWarps / kWarpsPerRow;
constexpr int kW1Vec = 10;               // float4 of a W1 row per lane held ahead: in_dim <= 5120

__global__ void __launch_bounds__(kPoolThreads)
    pool_kernel(const uint16_t* __restrict__ hidden, int T, int Hd, int n_pool,
                float* __restrict__ pooled) {
  // The MLP's CTAs may start now: they load their weights and wait for this grid.
  griddep_launch_dependents();
  __shared__ float part[kRowGroups][256];
  const int side = blockIdx.y;  // 0: first rows, 1: last rows
  const int n = min(n_pool, T);
  const int row0 = side == 0 ? 0 : T - n;
  const int cg = threadIdx.x & 31, rg = threadIdx.x >> 5;
  const int c0 = blockIdx.x * 256 + cg * 8;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  if (c0 + 8 <= Hd && (Hd & 7) == 0 && n <= kRowGroups * kPoolRowsPerThread) {
    // Every load of the thread in flight at once (rows rg, rg + 8, ...).
    uint4 w[kPoolRowsPerThread];
#pragma unroll
    for (int k = 0; k < kPoolRowsPerThread; ++k) {
      const int t = rg + kRowGroups * k;
      w[k] = t < n ? *reinterpret_cast<const uint4*>(hidden + static_cast<size_t>(row0 + t) * Hd + c0)
                   : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int k = 0; k < kPoolRowsPerThread; ++k) {
      const uint32_t ws[4] = {w[k].x, w[k].y, w[k].z, w[k].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc[2 * e] += bf16lo_to_f32(ws[e]);
        acc[2 * e + 1] += bf16hi_to_f32(ws[e]);
      }
    }
  } else if (c0 + 8 <= Hd && (Hd & 7) == 0) {
    for (int t = rg; t < n; t += kRowGroups) {
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
    for (int t = rg; t < n; t += kRowGroups)
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
    for (int r = 0; r < kRowGroups; ++r) s += part[r][threadIdx.x];
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
  const bool vec = (in_dim & 3) == 0;
  const int n4 = in_dim >> 2;
  const bool held = vec && n4 <= kW1Vec * 32 * kWarpsPerRow;
  // The weights do not depend on the pool: this warp's slice of W1 row j is
  // loaded before the wait for the pool grid (launched programmatically).
  float4 wv[kW1Vec];
  if (held) {
    const float4* w = reinterpret_cast<const float4*>(W1 + static_cast<size_t>(j < H1 ? j : 0) * in_dim);
#pragma unroll
    for (int k = 0; k < kW1Vec; ++k) {
      const int i4 = wr * 32 + lane + k * 32 * kWarpsPerRow;
      wv[k] = (j < H1 && i4 < n4) ? __ldg(w + i4) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  griddep_wait();   // pooled[] is the previous grid's output
  float acc = 0.f;
  if (j < H1) {
    if (held) {
#pragma unroll
      for (int k = 0; k < kW1Vec; ++k) {
        const int i4 = wr * 32 + lane + k * 32 * kWarpsPerRow;
        if (i4 < n4) {
          const float4 pv = *(reinterpret_cast<const float4*>(pooled) + i4);
          acc = fmaf(wv[k].x, pv.x, acc);
          acc = fmaf(wv[k].y, pv.y, acc);
          acc = fmaf(wv[k].z, pv.z, acc);
          acc = fmaf(wv[k].w, pv.w, acc);
        }
      }
    } else if (vec) {
      const float* w = W1 + static_cast<size_t>(j) * in_dim;
#pragma unroll 4
      for (int i4 = wr * 32 + lane; i4 < n4; i4 += 32 * kWarpsPerRow) {
        const float4 wq = __ldg(reinterpret_cast<const float4*>(w) + i4);
        const float4 pv = *(reinterpret_cast<const float4*>(pooled) + i4);
        acc = fmaf(wq.x, pv.x, acc);
        acc = fmaf(wq.y, pv.y, acc);
        acc = fmaf(wq.z, pv.z, acc);
        acc = fmaf(wq.w, pv.w, acc);
      }
    } else {
      const float* w = W1 + static_cast<size_t>(j) * in_dim;
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
  const bool vec2 = (H1 & 3) == 0;
  for (int l = warp; l < L; l += kMlpWarps) {
    float acc2 = 0.f;
    if (vec2) {
      const float4* w = reinterpret_cast<const float4*>(W2 + static_cast<size_t>(l) * H1);
      const float4* u = reinterpret_cast<const float4*>(hidden1);
#pragma unroll 4
      for (int i4 = lane; i4 < (H1 >> 2); i4 += 32) {
        const float4 wq = __ldg(w + i4);
        const float4 uq = __ldcg(u + i4);
        acc2 = fmaf(wq.x, uq.x, acc2);
        acc2 = fmaf(wq.y, uq.y, acc2);
        acc2 = fmaf(wq.z, uq.z, acc2);
        acc2 = fmaf(wq.w, uq.w, acc2);
      }
    } else {
      const float* w = W2 + static_cast<size_t>(l) * H1;
      for (int i = lane; i < H1; i += 32) acc2 = fmaf(__ldg(w + i), __ldcg(hidden1 + i), acc2);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc2 += __shfl_xor_sync(0xffffffffu, acc2, o);
    if (lane == 0) {
      const float z = acc2 + b2[l];
      const float r = 1.f / (1.f + expf(-z));
      layer_mode[l] = r > thresh ? 1 : 0;
      if (score) score[l] = r;
    }
  }
  if (threadIdx.x == 0) *ticket = 0;
}

}  // namespace

// hidden1 starts on a 16-byte boundary after pooled[2 Hd]: the last CTA reads
// it as float4 whenever H1 % 4 == 0, and 2 Hd floats end 8 bytes short of one
// when Hd is odd.
size_t route_hidden1_offset(int Hd) { return static_cast<size_t>(2 * Hd + 3) & ~static_cast<size_t>(3); }

size_t route_workspace_bytes(int Hd, int H1) {
  return (route_hidden1_offset(Hd) + static_cast<size_t>(H1)) * sizeof(float) + 64;
}

cudaError_t launch_route(const RouteLaunch& p, cudaStream_t stream) {
  const dim3 pgrid((p.Hd + 255) / 256, 2);
  pool_kernel<<<pgrid, kPoolThreads, 0, stream>>>(p.hidden, p.T, p.Hd, p.n_pool, p.pooled);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // Programmatic stream serialisation: the MLP's CTAs start while the pool runs
  // and wait for it (griddep_wait) after loading their weights.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((p.H1 + kRowsPerCta - 1) / kRowsPerCta);
  cfg.blockDim = dim3(kMlpWarps * 32);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, mlp_kernel, static_cast<const float*>(p.pooled), 2 * p.Hd, p.W1,
                            p.b1, p.H1, p.W2, p.b2, p.L, p.thresh, p.hidden1, p.ticket,
                            p.layer_mode, p.score);
}

}  // namespace flux
