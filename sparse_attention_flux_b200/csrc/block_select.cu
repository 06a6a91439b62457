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
//     the chunk's Q once as strided boxes (traversal stride 8: box kk holds
//     the 16 rows kk, kk + 8, ... of block i), resident in shared memory as
//     the N = 64 operand (four heads x 16 strided rows).  The keys are the
//     M = 128 operand: 8 key blocks x 16 strided positions, boxes of rows
//     7-kk, 15-kk, ... so the antidiagonal pairing is the choice of box,
//     streamed as 16 KB chunks (one offset kk, 64 channels) through a 4-stage
//     ring; K = 8 d per tile.  The 128-lane x 64-column accumulator is
//     double-buffered in TMEM; four epilogue warps, one per lane quarter (two
//     key blocks each), reduce it to per-(head, key block) log-sum-exps while
//     the next tile's MMAs run, and at the end each head's shares are summed
//     over the chunk into a per-chunk partial row.  Bound: the K chunks'
//     stream from L2 (each key block once per query block and chunk of heads;
//     about 7 TB/s at T 32768).
//   block_select_kernel: one CTA per query block: the partial rows summed in
//     a fixed order, a bitonic sort of the candidates (score descending, block
//     ascending) and one thread's sequential fp32 running sum decide the kept
//     blocks.  Deterministic: no atomics.
#include "common.cuh"
#include "kernels.h"

namespace flux {

namespace {

constexpr int kTile = 128;                 // query / key block, tokens
constexpr int kMaxHeads = 4;               // query heads per score CTA
constexpr int kScoreThreads = 32 * 6;      // K producer, MMA issuer, four epilogue warps
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

constexpr int kGroup = 8;                  // key blocks per MMA tile: M = 128 strided keys
constexpr int kStages = 4;                 // K chunk ring
// The barrier area (16 slots of 8 bytes) holds full and empty per stage, dfull[2],
// dfree[2], qbar, drain and then the TMEM address slot.
static_assert(2 * kStages + 6 + 1 <= 16, "barrier area too small for the ring");

template <int D>
struct ScoreSmem {
  static constexpr int CH = D / 64;
  static constexpr int QROWS = kMaxHeads * 16;   // MMA N: four heads x 16 strided rows
  // Q (resident B operand): [kk][chunk][64 rows x 128 B].  K chunk (A operand, ring):
  // [128 rows x 128 B] = one antidiagonal offset kk and one 64-channel chunk of 8 key
  // blocks.  Both 128-byte swizzled, 8-row groups 1 KB apart.
  static constexpr int Q = 0;
  static constexpr int Q_BYTES = kStride * CH * QROWS * 128;   // CH * 64 KB
  static constexpr int KC = Q + Q_BYTES;
  static constexpr int KC_BYTES = kGroup * 16 * 128;           // 16 KB
  static constexpr int LSE = KC + kStages * KC_BYTES;          // f32 [kMaxHeads][nb]
  __host__ __device__ static int bars(int nb) { return LSE + kMaxHeads * nb * 4; }
  __host__ __device__ static int total(int nb) { return bars(nb) + 16 * 8 + 1024; }
};

template <int D>
__global__ void __launch_bounds__(kScoreThreads, 1)
    block_score_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k, const ScoreArgs a) {
  using L = ScoreSmem<D>;
  constexpr int CH = L::CH;
  constexpr int S = kStride;
  constexpr int R = kTile / S;               // 16 strided positions per block
  constexpr int NCHUNK = S * CH;             // K chunks per group (K = 8 d in 64-channel steps)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  float* lse = reinterpret_cast<float*>(smem + L::LSE);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::bars(a.nb));
  uint64_t* full = bars;                  // [kStages] K chunk landed
  uint64_t* empty = bars + kStages;       // [kStages] K chunk read by its MMAs
  uint64_t* dfull = bars + 2 * kStages;   // [2] accumulator tile written
  uint64_t* dfree = dfull + 2;            // [2] accumulator tile read by the epilogue warps
  uint64_t* qbar = dfull + 4;
  uint64_t* drain = dfull + 5;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(dfull + 6);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nchunk = a.G / a.hc;
  const int per_i = a.B * a.Hkv * nchunk;
  const int i = a.nb - 1 - static_cast<int>(blockIdx.x) / per_i;
  const int rem = static_cast<int>(blockIdx.x) % per_i;
  const int b = rem / (a.Hkv * nchunk);
  const int g = (rem / nchunk) % a.Hkv;
  const int hc = rem % nchunk;
  const int head0 = g * a.G + hc * a.hc;
  const int ngroups = i / kGroup + 1;        // key blocks 0..i in groups of 8

  // A chunk of fewer than four heads: the absent heads' rows of Q are zero.
  if (a.hc < kMaxHeads) {
    const int per_box = (kMaxHeads - a.hc) * 16 * 128 / 16;   // uint4 per (kk, chunk)
    for (int idx = threadIdx.x; idx < NCHUNK * per_box; idx += blockDim.x) {
      const int box = idx / per_box, off = idx % per_box;
      reinterpret_cast<uint4*>(smem + L::Q + box * (L::QROWS * 128) + a.hc * 16 * 128)[off] =
          make_uint4(0u, 0u, 0u, 0u);
    }
    fence_proxy_async_smem();
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&dfull[s], 1);
      mbar_init(&dfree[s], 4);
    }
    mbar_init(qbar, 1);
    mbar_init(drain, 1);
    fence_barrier_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    mbar_arrive_expect_tx(qbar, a.hc * NCHUNK * 16 * 128);
    for (int w = 0; w < a.hc; ++w)
      for (int kk = 0; kk < S; ++kk)
        for (int c = 0; c < CH; ++c)
          tma_load_4d(&tm_q, qbar, smem + L::Q + (kk * CH + c) * (L::QROWS * 128) + w * 16 * 128,
                      c * 64, head0 + w, i * kTile + kk, b);
  }
  if (warp == 1) tmem_alloc(tmem_slot, 128);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;

  if (warp == 0) {
    // ------------------------------------------------------------ K producer
    // Chunk t = (group, kk, channel chunk): 4 boxes of 32 strided rows, each
    // spanning two key blocks (rows 7-kk, 15-kk, ... of key blocks 2q, 2q+1).
    if (lane == 0) {
      const int total = ngroups * NCHUNK;
      int issued = 0;
      for (int t = 0; t < total; ++t) {
        const int st = t % kStages;
        if (t >= kStages && !mbar_wait(&empty[st], ((t / kStages) - 1) & 1, a.st)) break;
        const int gi = t / NCHUNK, kk = (t % NCHUNK) / CH, c = t % CH;
        mbar_arrive_expect_tx(&full[st], L::KC_BYTES);
        for (int q4 = 0; q4 < 4; ++q4)
          tma_load_4d(&tm_k, &full[st], smem + L::KC + st * L::KC_BYTES + q4 * 32 * 128, c * 64, g,
                      (gi * kGroup + 2 * q4) * kTile + S - 1 - kk, b);
        issued = t + 1;
      }
      mbar_drain(qbar, 0);
      for (int t = issued - kStages < 0 ? 0 : issued - kStages; t < issued; ++t)
        mbar_drain(&full[t % kStages], (t / kStages) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // D[128 keys x 64 query rows] = Kc[128 x 8d] Q[64 x 8d]^T per group of 8 key
    // blocks, double-buffered in TMEM columns [64 s, 64 s + 64): row = TMEM lane
    // = strided key position, column 16 h + r = strided row r of head h.
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16(kGroup * 16, L::QROWS, false, false);
      const uint32_t qbase = smem_u32(smem + L::Q);
      bool mok = mbar_wait(qbar, 0, a.st);
      for (int gi = 0; mok && gi < ngroups; ++gi) {
        const int gb = gi & 1;
        if (gi >= 2 && !mbar_wait(&dfree[gb], ((gi >> 1) - 1) & 1, a.st)) { mok = false; break; }
        for (int u = 0; u < NCHUNK; ++u) {
          const int t = gi * NCHUNK + u, st = t % kStages;
          if (!mbar_wait(&full[st], (t / kStages) & 1, a.st)) { mok = false; break; }
          tc_fence_after();
          const uint32_t kc = smem_u32(smem + L::KC + st * L::KC_BYTES);
          const uint32_t qc = qbase + u * (L::QROWS * 128);   // u = kk * CH + c
#pragma unroll
          for (int k16 = 0; k16 < 4; ++k16)
            umma_bf16_ss(tmem + gb * 64,
                         umma_smem_desc(kc + k16 * 32, 16, 1024, kSwizzle128B),
                         umma_smem_desc(qc + k16 * 32, 16, 1024, kSwizzle128B), idesc,
                         (u | k16) != 0);
          umma_commit(&empty[st]);
        }
        if (!mok) break;
        umma_commit(&dfull[gb]);
      }
      // Every MMA issued by this thread completes before TMEM is released.
      umma_commit(drain);
      mbar_drain(drain, 0);
    }
  } else {
    // ------------------------------------------------------------ epilogue: one lane quarter
    // Warp w reads TMEM lanes 32 q .. 32 q + 31 (q = w % 4): key blocks 2q + (lane >> 4)
    // of the group, strided key column lane & 15; 64 columns = 4 heads x 16 rows.
    const int q = warp & 3;
    const uint32_t tl = tmem + (static_cast<uint32_t>(q * 32) << 16);
    const int half = lane >> 4, cc = lane & 15;
    for (int gi = 0; gi < ngroups; ++gi) {
      const int gb = gi & 1;
      if (!mbar_wait(&dfull[gb], (gi >> 1) & 1, a.st)) { ok = false; break; }
      tc_fence_after();
      uint32_t v[2][32];
      tmem_ld32(tl + gb * 64, v[0]);
      tmem_ld32(tl + gb * 64 + 32, v[1]);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&dfree[gb]);
      const int j = gi * kGroup + 2 * q + half;   // this lane's key block
      const int cg = j * R + cc;
#pragma unroll
      for (int h = 0; h < kMaxHeads; ++h) {
        float z[16];
        float m = -INFINITY;
#pragma unroll
        for (int r = 0; r < 16; ++r) {
          const int rg = i * R + r;
          const bool valid = j <= i && cg <= rg && rg < a.nr && cg < a.nr;
          z[r] = valid ? __uint_as_float(v[h >> 1][(h & 1) * 16 + r]) * a.scale_log2 : -INFINITY;
          m = fmaxf(m, z[r]);
        }
        // over the 16 lanes of this key block (xor within a half-warp)
#pragma unroll
        for (int o = 8; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float sum = 0.f;
        if (m != -INFINITY) {
#pragma unroll
          for (int r = 0; r < 16; ++r) sum += ex2(z[r] - m);
        }
#pragma unroll
        for (int o = 8; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        if (cc == 0 && j <= i) lse[h * a.nb + j] = m == -INFINITY ? -INFINITY : m + __log2f(sum);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp >= 2) {
    // This head's shares: P_h[j] = 2^(lse_j - lse_total), written over lse.
    float* my_lse = lse + (warp & 3) * a.nb;
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
    float sacc = 0.f;
    for (int w = 0; w < a.hc; ++w) sacc += lse[w * a.nb + j];
    out[j] = sacc;
  }
  if (warp == 1) tmem_dealloc(tmem, 128);
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
