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
//   block_score_kernel: a cluster of two CTAs (one per SM) per (sequence, kv
//     head, chunk of up to four query heads, pair of query blocks iA = i,
//     iB = i - 1), pairs longest first.  Each CTA holds its own query block's Q
//     resident, loaded once by TMA as strided boxes (traversal stride 8: box kk
//     holds the 16 rows kk, kk + 8, ... of the block): four heads x 16 strided
//     rows, 64 rows of the N = 128 operand of a two-SM tcgen05 MMA (CTA 0's
//     block in columns 0-63, CTA 1's in 64-127).  The keys are the M = 256
//     operand: per pair tile, CTA c streams key group 2 t + c -- 8 key blocks x
//     16 strided positions, boxes of rows 7-kk, 15-kk, ... so the antidiagonal
//     pairing is the choice of box -- as 16 KB chunks (one offset kk, 64
//     channels) through a 4-stage ring whose loads complete on CTA 0's
//     barriers; K = 8 d per tile.  CTA 0's thread issues the MMAs; each CTA's
//     TMEM receives its 128 keys x both blocks' 128 columns, double-buffered.
//     Each key tile thus serves two query blocks: the key stream from L2 --
//     what bounds the one-block form -- is halved.  Four epilogue warps per CTA,
//     one per TMEM lane quarter (two key blocks), reduce the tile to per-(query
//     block, head, key block) log-sum-exps while the next tile's MMAs run, each
//     written into the shared memory of the CTA that owns the query block
//     (the peer's by a distributed shared-memory store); after a cluster
//     barrier each CTA turns its block's log-sum-exps into shares and sums them
//     over the chunk's heads into a per-chunk partial row.
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

// ---- two-SM pair primitives (a cluster of two CTAs, one per SM)
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
               ::: "memory");
}
// The address of this CTA's shared location `saddr` in CTA `rank`'s window.
__device__ __forceinline__ uint32_t in_cta(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ void arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}
__device__ __forceinline__ void st_cluster_f32(uint32_t cluster_addr, float v) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(cluster_addr), "f"(v) : "memory");
}
__device__ __forceinline__ bool try_wait_cl(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait (cluster scope): the time limit or the error word ends it.
__device__ __forceinline__ bool wait_cl(uint64_t* bar, uint32_t parity, const DevStatus& st) {
  if (try_wait_cl(bar, parity)) return true;
  const long long t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (try_wait_cl(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (globaltimer_ns() - t0 > st.spin_ns || *reinterpret_cast<volatile int*>(st.err) != 0) {
        raise_error(st.err, DEV_ERR_TIMEOUT);
        return false;
      }
    }
  }
}
// Wait for the pair's own copies and MMAs: bounded by time alone.
__device__ __forceinline__ bool drain_cl(uint64_t* bar, uint32_t parity,
                                         long long limit_ns = 100000000) {
  if (try_wait_cl(bar, parity)) return true;
  const long long t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (try_wait_cl(bar, parity)) return true;
    if ((it & 63u) == 0 && globaltimer_ns() - t0 > limit_ns) return false;
  }
}
// Tiled load into this CTA's shared memory completing on CTA 0's barrier
// (`bar` in the cluster window).  No multicast: each CTA reads its own tile.
__device__ __forceinline__ void tma_load_4d_pair(const CUtensorMap* map, uint32_t bar, void* smem,
                                                 int c0, int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(smem)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}
// D[256 x N] (+)= A[256 x 16] B[N x 16]^T over the pair: each CTA supplies the A
// rows of its 128-row half and N/2 rows of B from its shared memory at the same
// offsets; each CTA's TMEM receives its 128 rows at full N.
__device__ __forceinline__ void umma_ss_pair(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                             uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
// Arrive on the barrier at this offset in both CTAs once the issued MMAs are done.
__device__ __forceinline__ void umma_commit_pair(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(smem_u32(bar)), "h"(static_cast<uint16_t>(0x3))
      : "memory");
}

template <int D>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kScoreThreads, 1)
    block_score_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k, const ScoreArgs a) {
  using L = ScoreSmem<D>;
  constexpr int CH = L::CH;
  constexpr int S = kStride;
  constexpr int R = kTile / S;               // 16 strided positions per block
  constexpr int NCHUNK = S * CH;             // K chunks per key group (K = 8 d in 64-channel steps)
  constexpr int QBOX = L::QROWS * 128;       // one (kk, chunk) box of the resident Q
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  float* lse = reinterpret_cast<float*>(smem + L::LSE);   // [kMaxHeads][nb]: this CTA's query block
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::bars(a.nb));
  uint64_t* full = bars;                  // [kStages] both CTAs' K chunks landed (CTA 0)
  uint64_t* empty = bars + kStages;       // [kStages] K chunk read by its MMAs (both CTAs)
  uint64_t* dfull = bars + 2 * kStages;   // [2] accumulator tile written (both CTAs)
  uint64_t* dfree = dfull + 2;            // [2] accumulator tile read by both CTAs' epilogues (CTA 0)
  uint64_t* qbar = dfull + 4;             // both CTAs' Q landed (CTA 0)
  uint64_t* drain = dfull + 5;            // every MMA of the pair done (both CTAs)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(dfull + 6);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int nchunk = a.G / a.hc;
  const int per_p = a.B * a.Hkv * nchunk;
  const int pair = static_cast<int>(blockIdx.x >> 1) / per_p;   // query-block pairs, longest first
  const int rem = static_cast<int>(blockIdx.x >> 1) % per_p;
  const int b = rem / (a.Hkv * nchunk);
  const int g = (rem / nchunk) % a.Hkv;
  const int hc = rem % nchunk;
  const int head0 = g * a.G + hc * a.hc;
  const int iA = a.nb - 1 - 2 * pair;        // CTA 0's query block
  const int iB = iA - 1;                     // CTA 1's query block (none when negative)
  const int i_me = rank == 0 ? iA : iB;
  const int npt = iA / (2 * kGroup) + 1;     // pair tiles of 16 key blocks: CTA c takes group 2 t + c
  const int q_bytes = a.hc * NCHUNK * 16 * 128;

  // Q rows the CTA does not load are zero: heads past the chunk, or no query block.
  {
    const int h_lo = i_me >= 0 ? a.hc : 0;
    if (h_lo < kMaxHeads) {
      const int per_box = (kMaxHeads - h_lo) * 16 * 128 / 16;   // uint4 per (kk, chunk)
      for (int idx = threadIdx.x; idx < NCHUNK * per_box; idx += blockDim.x) {
        const int box = idx / per_box, off = idx % per_box;
        reinterpret_cast<uint4*>(smem + L::Q + box * QBOX + h_lo * 16 * 128)[off] =
            make_uint4(0u, 0u, 0u, 0u);
      }
      fence_proxy_async_smem();
    }
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&dfull[s], 1);
      mbar_init(&dfree[s], 8);            // four epilogue warps of each CTA
    }
    mbar_init(qbar, 1);
    mbar_init(drain, 1);
    fence_barrier_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)), "r"(256u) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  // Both CTAs' barriers are initialised, and TMEM allocated, before anything
  // signals across the pair.
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t bars0 = in_cta(smem_u32(bars), 0);   // CTA 0's barriers, cluster window
  bool ok = true;
  bool aborted = false;

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    // Pair tile t, chunk (kk, channel chunk): this CTA's 8 key blocks of group
    // 2 t + rank as 4 strided boxes of 32 rows (rows 7-kk, 15-kk, ... of two
    // key blocks each), completing on CTA 0's barrier of the stage.
    if (lane == 0) {
      if (rank == 0) mbar_arrive_expect_tx(qbar, q_bytes * (iB >= 0 ? 2 : 1));
      if (i_me >= 0)
        for (int w = 0; w < a.hc; ++w)
          for (int kk = 0; kk < S; ++kk)
            for (int c = 0; c < CH; ++c)
              tma_load_4d_pair(&tm_q, bars0 + 8u * (qbar - bars), smem + L::Q + (kk * CH + c) * QBOX + w * 16 * 128,
                               c * 64, head0 + w, i_me * kTile + kk, b);
      const int total = npt * NCHUNK;
      int issued = 0;
      for (int t = 0; t < total; ++t) {
        const int st = t % kStages;
        if (t >= kStages && !wait_cl(&empty[st], ((t / kStages) - 1) & 1, a.st)) { aborted = true; break; }
        const int pt = t / NCHUNK, kk = (t % NCHUNK) / CH, c = t % CH;
        const int grp = 2 * pt + static_cast<int>(rank);
        if (rank == 0) mbar_arrive_expect_tx(&full[st], 2 * L::KC_BYTES);
        for (int q4 = 0; q4 < 4; ++q4)
          tma_load_4d_pair(&tm_k, bars0 + 8u * (full + st - bars),
                           smem + L::KC + st * L::KC_BYTES + q4 * 32 * 128, c * 64, g,
                           (grp * kGroup + 2 * q4) * kTile + S - 1 - kk, b);
        issued = t + 1;
      }
      if (rank == 0) {
        // CTA 0's barriers count both CTAs' bytes: once they complete, every copy
        // of the pair has landed.
        drain_cl(qbar, 0);
        for (int t = issued - kStages < 0 ? 0 : issued - kStages; t < issued; ++t)
          drain_cl(&full[t % kStages], (t / kStages) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (CTA 0)
    // D[256 keys x 128 columns] per pair tile: rows = this CTA's strided key
    // positions (TMEM lane), columns 16 h + r of CTA 0's query block and 64 + 16 h + r
    // of CTA 1's; double-buffered in TMEM columns [128 s, 128 s + 128).
    if (rank == 0 && lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16(2 * kGroup * 16, 2 * L::QROWS, false, false);
      const uint32_t qbase = smem_u32(smem + L::Q);
      bool mok = wait_cl(qbar, 0, a.st);
      for (int pt = 0; mok && pt < npt; ++pt) {
        const int gb = pt & 1;
        if (pt >= 2 && !wait_cl(&dfree[gb], ((pt >> 1) - 1) & 1, a.st)) { mok = false; break; }
        for (int u = 0; u < NCHUNK; ++u) {
          const int t = pt * NCHUNK + u, st = t % kStages;
          if (!wait_cl(&full[st], (t / kStages) & 1, a.st)) { mok = false; break; }
          tc_fence_after();
          const uint32_t kc = smem_u32(smem + L::KC + st * L::KC_BYTES);
          const uint32_t qc = qbase + u * QBOX;   // u = kk * CH + c
#pragma unroll
          for (int k16 = 0; k16 < 4; ++k16)
            umma_ss_pair(tmem + gb * 128,
                         umma_smem_desc(kc + k16 * 32, 16, 1024, kSwizzle128B),
                         umma_smem_desc(qc + k16 * 32, 16, 1024, kSwizzle128B), idesc,
                         (u | k16) != 0);
          umma_commit_pair(&empty[st]);
        }
        if (!mok) break;
        umma_commit_pair(&dfull[gb]);
      }
      // Every MMA of the pair completes before TMEM is released (in both CTAs).
      umma_commit_pair(drain);
      mbar_drain(drain, 0);
    } else if (rank == 1 && lane == 0) {
      drain_cl(drain, 0);
    }
  } else {
    // ------------------------------------------------------------ epilogue: one lane quarter
    // Warp w reads TMEM lanes 32 q .. 32 q + 31 (q = w % 4): key blocks 2q + (lane >> 4)
    // of this CTA's group, strided key column lane & 15; 128 columns = the two query
    // blocks' four heads x 16 rows.  Each (query block, head, key block) log-sum-exp
    // goes to the shared memory of the CTA that owns the query block.
    const int q = warp & 3;
    const uint32_t tl = tmem + (static_cast<uint32_t>(q * 32) << 16);
    const int half = lane >> 4, cc = lane & 15;
    const uint32_t lse_peer = in_cta(smem_u32(lse), rank ^ 1u);
    for (int pt = 0; pt < npt; ++pt) {
      const int gb = pt & 1;
      if (!wait_cl(&dfull[gb], (pt >> 1) & 1, a.st)) { ok = false; break; }
      tc_fence_after();
      uint32_t v[4][32];
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) tmem_ld32(tl + gb * 128 + c4 * 32, v[c4]);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (rank == 0) mbar_arrive(&dfree[gb]);
        else arrive_cluster(bars0 + 8u * (dfree + gb - bars));
      }
      const int j = (2 * pt + static_cast<int>(rank)) * kGroup + 2 * q + half;   // this lane's key block
      const int cg = j * R + cc;
#pragma unroll
      for (int qb = 0; qb < 2; ++qb) {
        const int iq = qb == 0 ? iA : iB;
#pragma unroll
        for (int h = 0; h < kMaxHeads; ++h) {
          float z[16];
          float m = -INFINITY;
#pragma unroll
          for (int r = 0; r < 16; ++r) {
            const int rg = iq * R + r;
            const bool valid = iq >= 0 && j <= iq && cg <= rg && rg < a.nr && cg < a.nr;
            z[r] = valid ? __uint_as_float(v[qb * 2 + (h >> 1)][(h & 1) * 16 + r]) * a.scale_log2
                         : -INFINITY;
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
          if (cc == 0 && iq >= 0 && j <= iq) {
            const float val = m == -INFINITY ? -INFINITY : m + __log2f(sum);
            if (qb == static_cast<int>(rank)) lse[h * a.nb + j] = val;
            else st_cluster_f32(lse_peer + 4u * static_cast<uint32_t>(h * a.nb + j), val);
          }
        }
      }
    }
  }
  // A CTA 1 whose producer gave up may still have copies in flight that complete on
  // CTA 0's barriers only: give them time to land before its memory goes away.
  if (warp == 0 && lane == 0 && aborted && rank == 1) {
    const long long t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 200000) {
    }
  }
  // Every log-sum-exp of this CTA's query block -- written here or by the peer --
  // is in place once both CTAs pass the cluster barrier.
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  if (warp >= 2 && i_me >= 0) {
    // This head's shares: P_h[j] = 2^(lse_j - lse_total), written over lse.
    float* my_lse = lse + (warp & 3) * a.nb;
    float mx = -INFINITY;
    for (int j = lane; j <= i_me; j += 32) mx = fmaxf(mx, my_lse[j]);
#pragma unroll
    for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float tot = 0.f;
    for (int j = lane; j <= i_me; j += 32) tot += mx == -INFINITY ? 0.f : ex2(my_lse[j] - mx);
#pragma unroll
    for (int o = 16; o; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
    __syncwarp();
    for (int j = lane; j <= i_me; j += 32)
      my_lse[j] = (ok && tot > 0.f) ? ex2(my_lse[j] - mx) / tot : 0.f;
  }
  __syncthreads();
  if (i_me >= 0) {
    // The chunk's heads summed in a fixed order.
    float* out = a.partial + (static_cast<size_t>((b * a.Hkv + g) * nchunk + hc) * a.nb + i_me) * a.nb;
    for (int j = threadIdx.x; j <= i_me; j += blockDim.x) {
      float sacc = 0.f;
      for (int w = 0; w < a.hc; ++w) sacc += lse[w * a.nb + j];
      out[j] = sacc;
    }
  }
  // Both CTAs leave together: no commit or remote access targets a CTA that has left.
  __syncwarp();
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  if (warp == 1)
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(256u)
                 : "memory");
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
    // The candidates in order, each taken while the running sum is below tau.
    // A key carries its score's bits, so the loop needs one shared-memory read
    // per candidate, issued eight at a time; the sum is the same sequential
    // fp32 sum in the same order.
    bool more = true;
    for (int t0 = 0; more && t0 < n2; t0 += 8) {
      uint64_t xs[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) xs[k] = t0 + k < n2 ? key[t0 + k] : ~0ull;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        if (!more || !(cum < tau) || xs[k] == ~0ull) {
          more = false;
          continue;
        }
        sel[static_cast<int>(xs[k] & 0xffffffffu)] = 1;
        cum += __uint_as_float(~static_cast<uint32_t>(xs[k] >> 32));
      }
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
  // Clusters of two CTAs, one per pair of query blocks (an odd count leaves the
  // last pair's second CTA without a query block).
  const unsigned npairs = static_cast<unsigned>(a.nb + 1) / 2;
  const unsigned grid = 2u * npairs * a.B * a.Hkv * (a.G / a.hc);
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
