// block_select.cu -- dynamic SA block selection on sm_100a.
//
// The pages name a block-sparse selector for the SA side (the checkpoint
// page's repository name "full_xattn_Qwen3-4B"; XAttention among the sparse
// methods in the UniSparse abstract on the page list) but print no algorithm.
// This file implements a stated reading of that family's published idea --
// score key blocks by antidiagonal sums over strided positions, keep the
// fewest blocks whose score mass reaches a threshold:
//   z[r][c]   = scale * sum_{k<S} q[rS+k] . key[cS+S-1-k]   strided positions, c <= r
//   P_h[i][j] = the share of query block i's mass sum exp(z) that falls in
//               key block j (query head h of sequence b)
//   P[i][j]   = mean over (b, h) of P_h[i][j]
//   keep j < sink and j = i, then the largest P[i][j] while the kept sum is
//   below tau (fp32, forced blocks by ascending j, then as taken).
// Two kernels:
//   block_score_kernel: one CTA per (sequence, kv head, chunk of up to four
//     query heads, query block i), query blocks longest first.  TMA brings
//     the chunk's Q tiles once and the K tile of every key block j <= i
//     through a 2-stage ring, each tile as S strided boxes: box kk holds the
//     R rows kk, kk + S, ... (K: S-1-kk, 2S-1-kk, ...), so strided position r
//     is row r of every box and an ldmatrix over 8 positions touches 8
//     different swizzle phases (rows S apart in one box would all share one:
//     an 8-way bank conflict).  One warp per query head computes the R x R
//     strided logits of (i, j) as 16x8x16 warp MMAs and reduces them to the
//     block's log-sum-exp.
//     At the end each head's shares are summed over the chunk into a
//     per-chunk partial row.  Bound: the latency of each warp's dependent
//     ldmatrix -> mma chain, with four compute warps per SM (the Q tiles of
//     four heads fill most of shared memory); the K tiles come from L2, shared
//     by the heads of a kv group.
//   block_select_kernel: one CTA per query block: the partial rows summed in
//     a fixed order, a bitonic sort of the candidates (score descending, block
//     ascending) and one thread's sequential fp32 running sum decide the kept
//     blocks.  Deterministic: no atomics.
#include "common.cuh"
#include "kernels.h"

namespace flux {

namespace {

constexpr int kTile = 128;                 // query / key block, tokens
constexpr int kBox = 128 * 128;            // one 128-row x 64-channel swizzled box
constexpr int kMaxHeads = 4;               // query heads per score CTA
constexpr int kScoreThreads = 32 * (kMaxHeads + 1);
constexpr int kSelectThreads = 256;
// Stride of the strided positions: the TMA traversal stride, at most 8.
constexpr int kStride = 8;

struct ScoreArgs {
  int B, T, Hq, Hkv, G, hc;   // hc: query heads per CTA (divides G, <= kMaxHeads)
  int nr, nb;                 // strided positions, query / key blocks
  float scale_log2;
  float* partial;             // [B * Hkv * G / hc][nb][nb]
  DevStatus st;
};

template <int D>
struct ScoreSmem {
  static constexpr int CH = D / 64;
  // A tile (128 rows x D) = S strided boxes of R rows per 64-channel chunk,
  // [kk][chunk][R rows x 128 B]: CH * kBox bytes whatever the stride.
  static constexpr int Q = 0;                              // [kMaxHeads] tiles
  static constexpr int K = Q + kMaxHeads * CH * kBox;      // [2 stages] tiles
  static constexpr int LSE = K + 2 * CH * kBox;            // f32 [kMaxHeads][nb]
  static int total(int nb) { return LSE + kMaxHeads * nb * 4 + 8 * 8 + 1024; }
};

// Shared-memory address of channel chunk uu (16 bytes) of strided row r in
// box kk of a tile of strided boxes (R rows each, 128-byte swizzle).
template <int R, int CH>
__device__ __forceinline__ uint32_t swz(uint32_t tile, int kk, int r, int uu) {
  return tile + (kk * CH + (uu >> 3)) * (R * 128) + r * 128 + (((uu & 7) ^ (r & 7)) << 4);
}

template <int D>
__global__ void __launch_bounds__(kScoreThreads, 1)
    block_score_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k, const ScoreArgs a) {
  using L = ScoreSmem<D>;
  constexpr int CH = L::CH;
  constexpr int S = kStride;
  constexpr int R = kTile / S;               // strided positions per block: 16 = one m16 tile
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  float* lse = reinterpret_cast<float*>(smem + L::LSE);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::LSE + kMaxHeads * a.nb * 4);
  uint64_t* full = bars;         // [2]
  uint64_t* empty = bars + 2;    // [2]
  uint64_t* qbar = bars + 4;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nchunk = a.G / a.hc;
  const int per_i = a.B * a.Hkv * nchunk;
  const int i = a.nb - 1 - static_cast<int>(blockIdx.x) / per_i;
  const int rem = static_cast<int>(blockIdx.x) % per_i;
  const int b = rem / (a.Hkv * nchunk);
  const int g = (rem / nchunk) % a.Hkv;
  const int hc = rem % nchunk;
  const int head0 = g * a.G + hc * a.hc;

  if (threadIdx.x == 0) {
    mbar_init(&full[0], 1);
    mbar_init(&full[1], 1);
    mbar_init(&empty[0], a.hc);
    mbar_init(&empty[1], a.hc);
    mbar_init(qbar, 1);
    fence_barrier_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    mbar_arrive_expect_tx(qbar, a.hc * CH * kBox);
    for (int w = 0; w < a.hc; ++w)
      for (int kk = 0; kk < S; ++kk)
        for (int c = 0; c < CH; ++c)
          tma_load_4d(&tm_q, qbar, smem + L::Q + w * CH * kBox + (kk * CH + c) * (R * 128),
                      c * 64, head0 + w, i * kTile + kk, b);
  }
  __syncthreads();

  if (warp == kMaxHeads) {
    // ------------------------------------------------------------ K producer
    if (lane == 0) {
      int issued = 0;
      for (int j = 0; j <= i; ++j) {
        const int s = j & 1;
        if (j >= 2 && !mbar_wait(&empty[s], ((j >> 1) - 1) & 1, a.st)) break;
        mbar_arrive_expect_tx(&full[s], CH * kBox);
        for (int kk = 0; kk < S; ++kk)
          for (int c = 0; c < CH; ++c)
            tma_load_4d(&tm_k, &full[s], smem + L::K + s * CH * kBox + (kk * CH + c) * (R * 128),
                        c * 64, g, j * kTile + S - 1 - kk, b);
        issued = j + 1;
      }
      mbar_drain(qbar, 0);
      for (int j = issued - 2 < 0 ? 0 : issued - 2; j < issued; ++j)
        mbar_drain(&full[j & 1], (j >> 1) & 1);
    }
  } else if (warp < a.hc) {
    // ------------------------------------------------------------ one query head
    const int mi = lane >> 3, rr = lane & 7;     // ldmatrix: matrix, row within it
    const int gq = lane >> 2, tq = lane & 3;     // mma fragment: row group, column pair
    const uint32_t qbase = smem_u32(smem + L::Q + warp * CH * kBox);
    const int ra = ((mi & 1) << 3) + rr;         // A: strided row of this lane's matrix row
    const int cb = ((mi >> 1) << 3) + rr;        // B: strided column (two n-tiles of 8)
    float* my_lse = lse + warp * a.nb;
    bool ok = mbar_wait(qbar, 0, a.st);
    for (int j = 0; ok && j <= i; ++j) {
      const int s = j & 1;
      if (!mbar_wait(&full[s], (j >> 1) & 1, a.st)) { ok = false; break; }
      const uint32_t kbase = smem_u32(smem + L::K + s * CH * kBox);
      // Two partial sums per n-tile (even / odd channel steps) halve the
      // dependent MMA chains.
      float acc[2][2][4] = {};
#pragma unroll 1
      for (int kk = 0; kk < S; ++kk) {
#pragma unroll
        for (int dc = 0; dc < D / 16; ++dc) {
          uint32_t af[4], b00, b01, b10, b11;
          ldmatrix_x4(swz<R, CH>(qbase, kk, ra, dc * 2 + (mi >> 1)), af[0], af[1], af[2], af[3]);
          ldmatrix_x4(swz<R, CH>(kbase, kk, cb, dc * 2 + (mi & 1)), b00, b01, b10, b11);
          mma_bf16_16816(acc[0][dc & 1], af, b00, b01);
          mma_bf16_16816(acc[1][dc & 1], af, b10, b11);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      // Block log-sum-exp (log2 domain) over the valid strided pairs c <= r.
      float z[8];
      float m = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int r = gq + (e >> 1) * 8, c = nt * 8 + 2 * tq + (e & 1);
          const int rg = i * R + r, cg = j * R + c;
          const bool valid = cg <= rg && rg < a.nr && cg < a.nr;
          const float v = valid ? (acc[nt][0][e] + acc[nt][1][e]) * a.scale_log2 : -INFINITY;
          z[nt * 4 + e] = v;
          m = fmaxf(m, v);
        }
#pragma unroll
      for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      float sum = 0.f;
      if (m != -INFINITY) {
#pragma unroll
        for (int e = 0; e < 8; ++e) sum += ex2(z[e] - m);
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      if (lane == 0) my_lse[j] = m == -INFINITY ? -INFINITY : m + __log2f(sum);
    }
    __syncwarp();
    // This head's shares: P_h[j] = 2^(lse_j - lse_total), written over lse.
    float mx = -INFINITY;
    for (int j = lane; j <= i; j += 32) mx = fmaxf(mx, my_lse[j]);
#pragma unroll
    for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float tot = 0.f;
    for (int j = lane; j <= i; j += 32) tot += mx == -INFINITY ? 0.f : ex2(my_lse[j] - mx);
#pragma unroll
    for (int o = 16; o; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
    __syncwarp();
    for (int j = lane; j <= i; j += 32)
      my_lse[j] = (ok && tot > 0.f) ? ex2(my_lse[j] - mx) / tot : 0.f;
  }
  __syncthreads();
  // The chunk's heads summed in a fixed order.
  float* out = a.partial + (static_cast<size_t>((b * a.Hkv + g) * nchunk + hc) * a.nb + i) * a.nb;
  for (int j = threadIdx.x; j <= i; j += blockDim.x) {
    float s = 0.f;
    for (int w = 0; w < a.hc; ++w) s += lse[w * a.nb + j];
    out[j] = s;
  }
}

__global__ void __launch_bounds__(kSelectThreads)
    block_select_kernel(const float* __restrict__ partial, int np, int nb, float inv_heads,
                        float tau, int sink, uint8_t* __restrict__ mask, float* __restrict__ score) {
  extern __shared__ uint8_t smem_raw[];
  uint64_t* key = reinterpret_cast<uint64_t*>(smem_raw);                 // [n2]
  const int i = blockIdx.x, tid = threadIdx.x;
  int n2 = 1;
  while (n2 < i + 1) n2 <<= 1;
  float* P = reinterpret_cast<float*>(smem_raw + static_cast<size_t>(n2) * 8);   // [i+1]
  uint8_t* sel = reinterpret_cast<uint8_t*>(P + (i + 1));                       // [i+1]
  for (int j = tid; j <= i; j += blockDim.x) {
    float s = 0.f;
    for (int p = 0; p < np; ++p) s += partial[(static_cast<size_t>(p) * nb + i) * nb + j];
    P[j] = s * inv_heads;
    sel[j] = (j < sink || j == i) ? 1 : 0;
  }
  __syncthreads();
  // Candidates ordered by score descending, then block ascending: scores are
  // non-negative, so the complemented bits order them in reverse.
  for (int j = tid; j < n2; j += blockDim.x)
    key[j] = (j <= i && !sel[j])
                 ? (static_cast<uint64_t>(~__float_as_uint(P[j])) << 32) | static_cast<uint32_t>(j)
                 : ~0ull;
  __syncthreads();
  for (int k = 2; k <= n2; k <<= 1) {
    for (int jj = k >> 1; jj > 0; jj >>= 1) {
      for (int t = tid; t < n2; t += blockDim.x) {
        const int u = t ^ jj;
        if (u > t) {
          const uint64_t x = key[t], y = key[u];
          if ((x > y) == ((t & k) == 0)) {
            key[t] = y;
            key[u] = x;
          }
        }
      }
      __syncthreads();
    }
  }
  if (tid == 0) {
    float cum = 0.f;
    for (int j = 0; j <= i; ++j)
      if (sel[j]) cum += P[j];
    for (int t = 0; t < n2 && cum < tau; ++t) {
      const uint64_t x = key[t];
      if (x == ~0ull) break;
      const int j = static_cast<int>(x & 0xffffffffu);
      sel[j] = 1;
      cum += P[j];
    }
  }
  __syncthreads();
  for (int j = tid; j < nb; j += blockDim.x) {
    mask[static_cast<size_t>(i) * nb + j] = j <= i ? sel[j] : 0;
    if (score) score[static_cast<size_t>(i) * nb + j] = j <= i ? P[j] : 0.f;
  }
}

template <int D>
cudaError_t launch_scores_t(const CUtensorMap& tq, const CUtensorMap& tk, const ScoreArgs& a,
                            cudaStream_t stream) {
  const int smem = ScoreSmem<D>::total(a.nb);
  cudaFuncSetAttribute(block_score_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  const unsigned grid = static_cast<unsigned>(a.nb) * a.B * a.Hkv * (a.G / a.hc);
  block_score_kernel<D><<<grid, kScoreThreads, smem, stream>>>(tq, tk, a);
  return cudaGetLastError();
}

int heads_per_cta(int G) {
  for (int h = kMaxHeads; h > 1; --h)
    if (G % h == 0) return h;
  return 1;
}

}  // namespace

size_t block_select_workspace_bytes(int B, int T, int Hq, int Hkv, int stride) {
  const int G = Hq / Hkv;
  const int nr = (T + stride - 1) / stride, R = kTile / stride;
  const size_t nb = static_cast<size_t>((nr + R - 1) / R);
  return static_cast<size_t>(B) * Hkv * (G / heads_per_cta(G)) * nb * nb * sizeof(float);
}

cudaError_t launch_block_select(const CUtensorMap& tq, const CUtensorMap& tk,
                                const BlockSelectLaunch& p, cudaStream_t stream) {
  ScoreArgs a;
  a.B = p.B;
  a.T = p.T;
  a.Hq = p.Hq;
  a.Hkv = p.Hkv;
  a.G = p.Hq / p.Hkv;
  a.hc = heads_per_cta(a.G);
  a.nr = (p.T + p.stride - 1) / p.stride;
  const int R = kTile / p.stride;
  a.nb = (a.nr + R - 1) / R;
  a.scale_log2 = p.scale * 1.4426950408889634f;
  a.partial = p.workspace;
  a.st = p.st;
  if (p.stride != kStride) return cudaErrorInvalidValue;
  const cudaError_t e = p.d == 64 ? launch_scores_t<64>(tq, tk, a, stream)
                                  : launch_scores_t<128>(tq, tk, a, stream);
  if (e != cudaSuccess) return e;
  int n2 = 1;
  while (n2 < a.nb) n2 <<= 1;
  const int smem = n2 * 8 + a.nb * 4 + a.nb + 16;
  cudaFuncSetAttribute(block_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  block_select_kernel<<<a.nb, kSelectThreads, smem, stream>>>(
      a.partial, p.B * p.Hkv * (a.G / a.hc), a.nb, 1.f / (p.B * p.Hq), p.tau, p.sink_blocks,
      p.block_mask, p.block_score);
  return cudaGetLastError();
}

}  // namespace flux
