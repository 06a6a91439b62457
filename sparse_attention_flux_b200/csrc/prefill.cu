// prefill.cu -- FA / SA prefill attention for one layer on sm_100a.
//
// Flux Attention routes each layer to Full Attention (exact causal softmax
// attention) or to block-sparse Sparse Attention (arXiv abstract; model card
// "Flux Attention: Qwen3-4B", "Sample Usage").  One kernel serves both: a
// CTA owns two 128-row query tiles Q0, Q1 that read the same keys and walks a
// list of 128-column key tiles: every tile up to the diagonal for FA, the
// tiles named by the compressed block-index list for SA (built once per CTA
// into shared memory), so skipped blocks are never loaded.  Each K/V tile is
// loaded once and used by both query tiles.  The two tiles are either
//   a head pair (GQA with an even group size): the same 128 rows of two query
//     heads that share a KV head.  Both tiles need exactly the same key tiles,
//     so no MMA or softmax is spent on a tile that only one of them sees; or
//   a row pair (odd group size, or per-head routing): rows [256u, 256u + 256)
//     of one query head, walking the union of the two tiles' lists.
// CTAs are ordered per sequence, in chunks of kv groups whose K/V fit in 48 MB
// of L2, longest unit first within a chunk.
//
// Per CTA (384 threads, warp-specialised):
//   warp 0      TMA producer (Q0, Q1 once; K/V tiles into a 2-stage ring, K
//               and V slots released separately) and, for SA, the builder of
//               the CTA's key-tile list.
//   warp 1      TMEM owner (all 512 columns) and UMMA issuer:
//                 S_i = Q_i K^T             (A, B from shared memory)
//                 O_i += P_i V              (A = P_i from TMEM, B from smem)
//               issued in the order S0 S1 | PV0 S0' PV1 S1' | ... so that the
//               tensor core works on one tile while the other's softmax runs;
//               the issue queue is shallow, so the thread's barrier waits and
//               slot releases sit outside the back-to-back MMA groups.
//   warps 2, 3  idle.
//   warps 4-7   softmax of Q0, warps 8-11 softmax of Q1: one query row per
//               thread (= one TMEM lane); online softmax in the log2 domain;
//               P_i written back over S_i's columns as packed bf16 for the
//               TMEM-A MMA.  After a row's first tile the exponentials use
//               the running max without the tile's row max (any max is exact
//               as long as the final division uses it); the tile's row sum
//               bounds every P, and only a sum above 2^20 sends the warp to
//               the row max, a lazy rescale of l and O (growth above 2^8) and
//               a redo of the tile.  The epilogue stages O_i / l as bf16 in
//               Q_i's freed shared memory and stores it by TMA.
// TMEM columns: S0 [0,128)  S1 [128,256)  O0 [256,256+D)  O1 [384,384+D).
#include "common.cuh"
#include "kernels.h"

namespace flux {

namespace {

constexpr int kBM = 128;                  // query rows per tile (TMEM lanes)
constexpr int kBN = 128;                  // key columns per tile
constexpr int kChunkBytes = 128 * 128;    // 128 rows x 64 bf16: one swizzle-128B box
constexpr int kThreads = 384;
constexpr float kRescaleLog2 = 8.f;       // lazy rescale threshold, log2 units
constexpr float kRedoSum = 1048576.f;     // 2^20: a tile row sum above it is redone

struct PrefillArgs {
  int B, T, Hq, Hkv, G;
  int head_pair;     // 1: a CTA = one 128-row tile of two heads; 0: 256 rows of one head
  int nunit;         // CTA units along T: 128-row tiles (head pair) or 256-row pairs
  int gchunk;        // kv groups whose units are scheduled together (divides Hkv)
  int nkt;           // 128-column key tiles along T
  int block;         // mask block: 64 or a multiple of 128
  int nqb;           // rows of the CSR
  int nkb;           // kv blocks along T (valid CSR column range)
  float scale_log2;  // scale * log2(e)
  const uint8_t* layer_mode;
  int layer;
  const int32_t* row_ptr;
  const int32_t* col;
  uint16_t* o;
  float* lse;
  int force_mode;            // -1: read layer_mode; 0: SA; 1: FA
  const uint8_t* head_mode;  // per-query-head routing [Hq] (overrides layer_mode), or null
  const float* blend_score;  // soft routing: o = r * o(previous) + (1 - r) * this, r = score[layer]
  DevStatus st;
};

// K and V slots are released separately: K(j) once S1(j) has read it, V(j)
// once PV1(j) has, so the load of K(j+2) starts about a tile-step earlier
// than it could if both waited for PV1(j).
enum { B_Q = 0, B_KF = 1, B_VF = 3, B_KE = 5, B_VE = 7, B_SF = 9, B_PF = 11, B_OD = 13,
       B_DRAIN = 14, B_COUNT = 15 };

template <int D>
struct Smem {
  static constexpr int CH = D / 64;
  static constexpr int Q = 0;                                  // [2 tiles][CH chunks]
  static constexpr int K = Q + 2 * CH * kChunkBytes;           // [2 stages][CH]
  static constexpr int V = K + 2 * CH * kChunkBytes;           // [2 stages][CH]
  static constexpr int MAP = V + 2 * CH * kChunkBytes;         // u32 [kPrefillMaxKvTiles]
  static constexpr int LIST = MAP + 4 * kPrefillMaxKvTiles;    // u32 [kPrefillMaxKvTiles]
  static constexpr int BARS = LIST + 4 * kPrefillMaxKvTiles;
  static constexpr int TMEM_SLOT = BARS + B_COUNT * 8;
  static constexpr int NLIST = TMEM_SLOT + 4;
  static constexpr int TOTAL = NLIST + 12;
  static constexpr int ALLOC = TOTAL + 1024;  // room to align the base to 1024
};

// Inclusive warp prefix sum.
__device__ __forceinline__ int warp_inclusive_sum(int x) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  return x;
}

// SA: the CTA's key tiles and, per tile, which (64-row query sub-block,
// 64-column key sub-block) pairs the block mask keeps: bit (qs * 2 + ks).
// One warp builds it; returns the list length.  Tiles past the last tile index
// `last` (the diagonal) are dropped (causal).  A CSR row out of range, an entry
// out of range or a row whose columns are not strictly ascending raises
// DEV_ERR_CSR and empties the list, so the unit's rows are written as zero.
//   Direct path -- blocks are whole key tiles (block a multiple of 128) and the
//   unit's rows all lie in one CSR row (e.g. a head-pair unit at block 128):
//   the row's ascending columns are the list, every tile with all bits set.
//   Two dependent global-read rounds (the row range and nnz, then the columns).
//   Map path otherwise: OR every kept block of the CSR rows of the nsub 64-row
//   sub-blocks (from row0) into a per-tile map, then compact it in ascending
//   tile order; the columns of each distinct CSR row are read once.
__device__ int build_tile_list(const PrefillArgs& a, int row0, int nsub, int last, uint32_t* map,
                               uint32_t* list) {
  const int lane = threadIdx.x & 31;
  const int r_last = min(row0 + nsub * 64, a.T) - 1;
  if (a.block % kBN == 0 && row0 / a.block == r_last / a.block) {
    const int qb = row0 / a.block;
    if (qb >= a.nqb) {
      if (lane == 0) raise_error(a.st.err, DEV_ERR_CSR);
      return 0;
    }
    const int lo = a.row_ptr[qb], hi = a.row_ptr[qb + 1], nnz = a.row_ptr[a.nqb];
    if (lo < 0 || hi < lo || hi > nnz) {
      if (lane == 0) raise_error(a.st.err, DEV_ERR_CSR);
      return 0;
    }
    const int tpb = a.block / kBN;                          // key tiles per block
    const uint32_t full = ((1u << (2 * nsub)) - 1u) << 24;  // every (qs, ks) bit
    int n = 0, prev = -1;
    for (int base = lo; base < hi; base += 32) {
      const int e = base + lane;
      const int j = e < hi ? a.col[e] : 0;
      const int jp = __shfl_up_sync(0xffffffffu, j, 1);
      const int before = lane == 0 ? prev : jp;
      const bool ok = e < hi && j >= 0 && j < a.nkb && j > before;
      if (__any_sync(0xffffffffu, e < hi && !ok)) {
        if (lane == 0) raise_error(a.st.err, DEV_ERR_CSR);
        return 0;
      }
      const int cnt = ok ? max(0, min(tpb, last - j * tpb + 1)) : 0;
      const int incl = warp_inclusive_sum(cnt);
      for (int t = 0; t < cnt; ++t)
        list[n + incl - cnt + t] = static_cast<uint32_t>(j * tpb + t) | full;
      n += __shfl_sync(0xffffffffu, incl, 31);
      prev = __shfl_sync(0xffffffffu, j, min(31, hi - 1 - base));
    }
    return n;
  }
  for (int J = lane; J <= last; J += 32) map[J] = 0;
  int qb_l = -1, lo_l = 0, hi_l = 0;
  if (lane < nsub && row0 + lane * 64 < a.T) {
    qb_l = (row0 + lane * 64) / a.block;
    if (qb_l < a.nqb) {
      lo_l = a.row_ptr[qb_l];
      hi_l = a.row_ptr[qb_l + 1];
    } else {
      qb_l = -2;   // row out of range
    }
  }
  const int nnz = a.row_ptr[a.nqb];
  if (qb_l >= 0 && (lo_l < 0 || hi_l < lo_l || hi_l > nnz)) qb_l = -2;
  bool bad = __any_sync(0xffffffffu, qb_l == -2);
  __syncwarp();
  for (int qs = 0; qs < nsub; ++qs) {
    const int qb = __shfl_sync(0xffffffffu, qb_l, qs);
    if (qb < 0 || (qs > 0 && __shfl_sync(0xffffffffu, qb_l, qs - 1) == qb)) continue;
    // Key sub-block bits of every query sub-block that reads CSR row qb.
    uint32_t bits_even = 0;
    for (int q2 = qs; q2 < nsub; ++q2)
      if (__shfl_sync(0xffffffffu, qb_l, q2) == qb) bits_even |= 1u << (q2 * 2);
    const int lo = __shfl_sync(0xffffffffu, lo_l, qs), hi = __shfl_sync(0xffffffffu, hi_l, qs);
    int prev = -1;
    for (int base = lo; base < hi; base += 32) {
      const int e = base + lane;
      const int j = e < hi ? a.col[e] : 0;
      const int jp = __shfl_up_sync(0xffffffffu, j, 1);
      const int before = lane == 0 ? prev : jp;
      prev = __shfl_sync(0xffffffffu, j, min(31, hi - 1 - base));
      if (e >= hi) continue;
      if (j < 0 || j >= a.nkb || j <= before) {
        bad = true;
        continue;
      }
      const int k0 = j * a.block, k1 = min((j + 1) * a.block, a.T);   // key range of block j
      for (int ks = k0 >> 6; ks < (k1 + 63) >> 6; ++ks) {                 // 64-column sub-blocks
        const int J = ks >> 1;
        if (J > last) break;
        atomicOr(&map[J], bits_even << (ks & 1));
      }
    }
  }
  if (__any_sync(0xffffffffu, bad)) {
    if (lane == 0) raise_error(a.st.err, DEV_ERR_CSR);
    return 0;
  }
  __syncwarp();
  int n = 0;
  for (int base = 0; base <= last; base += 32) {
    const int J = base + lane;
    const uint32_t m = J <= last ? map[J] : 0u;
    const unsigned bal = __ballot_sync(0xffffffffu, m != 0);
    if (m != 0) list[n + __popc(bal & ((1u << lane) - 1u))] = static_cast<uint32_t>(J) | (m << 24);
    n += __popc(bal);
  }
  return n;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tm_q,
                   const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v,
                   const __grid_constant__ CUtensorMap tm_o, const PrefillArgs a) {
  using L = Smem<D>;
  constexpr int CH = L::CH;
  constexpr uint32_t kTmemCols = 512;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem + L::Q;
  uint8_t* sK = smem + L::K;
  uint8_t* sV = smem + L::V;
  uint32_t* map = reinterpret_cast<uint32_t*>(smem + L::MAP);
  uint32_t* list = reinterpret_cast<uint32_t*>(smem + L::LIST);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::BARS);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::TMEM_SLOT);
  int* nlist = reinterpret_cast<int*>(smem + L::NLIST);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Order: sequence, then chunks of gchunk kv groups, then units longest
  // first (the last query rows carry the most causal work), then the chunk's
  // head units.  The CTAs in flight then read the K/V of gchunk groups only,
  // which stays in L2 instead of being re-read from DRAM.  Tile i (0, 1)
  // holds rows [row0 + i * row_step, +128) of query head head0 + i * head_step.
  const int hpu = a.head_pair ? a.Hq / 2 : a.Hq;   // head units per sequence
  const int cu = hpu / a.Hkv * a.gchunk;           // head units per chunk
  const int per_chunk = cu * a.nunit;
  const int per_seq = per_chunk * (a.Hkv / a.gchunk);
  const int b = static_cast<int>(blockIdx.x) / per_seq;
  const int rs_ = static_cast<int>(blockIdx.x) % per_seq;
  const int chunk = rs_ / per_chunk, rc = rs_ % per_chunk;
  const int unit = a.nunit - 1 - rc / cu;
  const int hu = chunk * cu + rc % cu;
  const int row0 = unit * (a.head_pair ? kBM : 2 * kBM);          // first row of the unit
  const int nrow = a.head_pair ? kBM : 2 * kBM;                    // rows of the unit
  const int head0 = a.head_pair ? 2 * hu : hu, head_step = a.head_pair ? 1 : 0;
  const int row_step = a.head_pair ? 0 : kBM;
  const int g = head0 / a.G;
  const bool fa = a.force_mode >= 0 ? a.force_mode == 1
                 : a.head_mode     ? a.head_mode[hu] != 0
                                   : (a.layer_mode == nullptr || a.layer_mode[a.layer] != 0);
  const int last_tile = min((row0 + nrow - 1) / kBN, a.nkt - 1);

  if (threadIdx.x == 0) {
    mbar_init(&bars[B_Q], 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars[B_KF + s], 1);
      mbar_init(&bars[B_VF + s], 1);
      mbar_init(&bars[B_KE + s], 1);
      mbar_init(&bars[B_VE + s], 1);
      mbar_init(&bars[B_SF + s], 1);
      mbar_init(&bars[B_PF + s], 128);
    }
    mbar_init(&bars[B_OD], 1);
    mbar_init(&bars[B_DRAIN], 1);
    fence_barrier_init();
    fence_proxy_async_smem();
    // Q does not depend on the key-tile list: start it now, so that its
    // latency overlaps the list build (two dependent global reads).
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    mbar_arrive_expect_tx(&bars[B_Q], 2 * CH * kChunkBytes);
    for (int i = 0; i < 2; ++i)
      for (int c = 0; c < CH; ++c)
        tma_load_4d(&tm_q, &bars[B_Q], sQ + (i * CH + c) * kChunkBytes, c * 64,
                    head0 + i * head_step, row0 + i * row_step, b);
  }
  if (warp == 0) {
    const int n = fa ? last_tile + 1 : build_tile_list(a, row0, nrow / 64, last_tile, map, list);
    if (lane == 0) *nlist = n;
  }
  if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int n = *nlist;
  auto tile_of = [&](int j, uint32_t& mask) -> int {
    if (fa) {
      mask = 0xFFu;
      return j;
    }
    const uint32_t e = list[j];
    mask = e >> 24;
    return static_cast<int>(e & 0xFFFFFFu);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int issued = 0;
      bool ok = true;
      for (int j = 0; j < n; ++j) {
        const int s = j & 1;
        uint32_t mask;
        const int J = tile_of(j, mask);
        if (j >= 2 && !mbar_wait(&bars[B_KE + s], ((j >> 1) - 1) & 1, a.st)) { ok = false; break; }
        mbar_arrive_expect_tx(&bars[B_KF + s], CH * kChunkBytes);
        for (int c = 0; c < CH; ++c)
          tma_load_4d(&tm_k, &bars[B_KF + s], sK + (s * CH + c) * kChunkBytes, c * 64, g,
                      J * kBN, b);
        if (j >= 2 && !mbar_wait(&bars[B_VE + s], ((j >> 1) - 1) & 1, a.st)) {
          // K(j) is in flight; V(j) is not: drain only what was issued.
          mbar_drain(&bars[B_KF + s], (j >> 1) & 1);
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&bars[B_VF + s], CH * kChunkBytes);
        for (int c = 0; c < CH; ++c)
          tma_load_4d(&tm_v, &bars[B_VF + s], sV + (s * CH + c) * kChunkBytes, c * 64, g,
                      J * kBN, b);
        issued = j + 1;
      }
      // Every copy issued lands before the CTA's smem goes away, also when a
      // consumer gave up early (loads before the last two were consumed).
      mbar_drain(&bars[B_Q], 0);
      for (int j = issued - 2 < 0 ? 0 : issued - 2; j < issued; ++j) {
        mbar_drain(&bars[B_KF + (j & 1)], (j >> 1) & 1);
        mbar_drain(&bars[B_VF + (j & 1)], (j >> 1) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && n > 0) {
      constexpr uint32_t idesc_s = umma_idesc_bf16(kBM, kBN, false, false);
      constexpr uint32_t idesc_o = umma_idesc_bf16(kBM, D, false, true);
      // Base descriptors are built once; a k-step or a ring slot adds its byte
      // offset / 16 to the 14-bit start-address field (shared memory is below
      // 256 KB, so the field never carries).  The MMA issue path then does one
      // 64-bit add per operand, which shortens both the issuing thread's loop
      // and the PV / next-S MMAs on the softmax's round trip.
      const uint64_t dq0 = umma_smem_desc(smem_u32(sQ), 16, 1024, kSwizzle128B);
      const uint64_t dk0 = umma_smem_desc(smem_u32(sK), 16, 1024, kSwizzle128B);
      const uint64_t dv0 = umma_smem_desc(smem_u32(sV), kChunkBytes, 1024, kSwizzle128B);
      constexpr uint64_t kSlot = static_cast<uint64_t>((CH * kChunkBytes) >> 4);
      auto issue_s = [&](int i, int s) {
        const uint64_t a0 = dq0 + (i ? kSlot : 0), b0 = dk0 + (s ? kSlot : 0);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint64_t off = static_cast<uint64_t>(((ks >> 2) * kChunkBytes + (ks & 3) * 32) >> 4);
          umma_bf16_ss(tmem + i * 128, a0 + off, b0 + off, idesc_s, ks > 0);
        }
      };
      auto issue_pv = [&](int i, int s, bool acc) {
        const uint64_t b0 = dv0 + (s ? kSlot : 0);
#pragma unroll
        for (int ks = 0; ks < kBN / 16; ++ks)
          umma_bf16_ts(tmem + 256 + i * 128, tmem + i * 128 + ks * 8,
                       b0 + static_cast<uint64_t>((ks * 16 * 128) >> 4), idesc_o,
                       (acc || ks > 0) ? 1u : 0u);
      };
      bool ok = mbar_wait(&bars[B_Q], 0, a.st) && mbar_wait(&bars[B_KF], 0, a.st);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        umma_commit(&bars[B_SF + 0]);
        issue_s(1, 0);
        umma_commit(&bars[B_SF + 1]);
        umma_commit(&bars[B_KE + 0]);
      }
      // The issue queue is shallow: this thread blocks in tcgen05.mma until
      // about the previous MMA starts, so anything it does between two groups
      // (even a wait that is already satisfied) idles the tensor core.  The
      // operand waits therefore come first, where the thread waits for P0
      // anyway, and the slot releases after the last group of the step.
      for (int j = 0; ok && j < n; ++j) {
        const int s = j & 1, sn = (j + 1) & 1;
        const bool more = j + 1 < n;
        if (!mbar_wait(&bars[B_VF + s], (j >> 1) & 1, a.st) ||
            (more && !mbar_wait(&bars[B_KF + sn], ((j + 1) >> 1) & 1, a.st)) ||
            !mbar_wait(&bars[B_PF + 0], j & 1, a.st)) { ok = false; break; }
        tc_fence_after();
        issue_pv(0, s, j > 0);
        if (more) {
          issue_s(0, sn);
          umma_commit(&bars[B_SF + 0]);
        }
        if (!mbar_wait(&bars[B_PF + 1], j & 1, a.st)) { ok = false; break; }
        tc_fence_after();
        issue_pv(1, s, j > 0);
        if (more) {
          issue_s(1, sn);
          umma_commit(&bars[B_SF + 1]);
        }
        umma_commit(&bars[B_VE + s]);
        if (more) umma_commit(&bars[B_KE + sn]);
      }
      if (ok) umma_commit(&bars[B_OD]);
      // Every MMA issued by this thread is complete before TMEM is released.
      umma_commit(&bars[B_DRAIN]);
      mbar_drain(&bars[B_DRAIN], 0);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax
    const int i = (warp - 4) >> 2;           // query tile 0 or 1
    const int quarter = warp & 3;            // TMEM lanes 32*quarter .. +31
    const int r = quarter * 32 + lane;       // row within the tile
    const int t_row = row0 + i * row_step + r;
    const int h = head0 + i * head_step;
    const int qs = (t_row - row0) >> 6;      // 64-row sub-block within the unit
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_off + i * 128;
    const uint32_t tO = tmem + lane_off + 256 + i * 128;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      uint32_t mask;
      const int J = tile_of(j, mask);
      if (!mbar_wait(&bars[B_SF + i], j & 1, a.st)) { ok = false; break; }
      tc_fence_after();
      float x[kBN];
      {
        uint32_t v[kBN / 32][32];
#pragma unroll
        for (int c = 0; c < kBN / 32; ++c) tmem_ld32(tS + c * 32, v[c]);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < kBN / 32; ++c)
#pragma unroll
          for (int e = 0; e < 32; ++e) x[c * 32 + e] = __uint_as_float(v[c][e]);
      }
      const uint32_t sub = (mask >> (qs * 2)) & 3u;
      const bool need_mask = J * kBN + kBN - 1 > t_row || sub != 3u;
      if (need_mask) {
#pragma unroll
        for (int c = 0; c < kBN; ++c)
          if (J * kBN + c > t_row || !((sub >> (c >> 6)) & 1u)) x[c] = -INFINITY;
      }
      // P = 2^(x scale - m) is exact for any m as long as the final division
      // (and the LSE) use the same m and nothing overflows, so after a row's
      // first visible tile the exponentials are taken against the running max
      // m_run without the tile's row max: the row sum, computed anyway, bounds
      // every P of the tile.  Only if some lane's sum passes kRedoSum (or is
      // not finite) -- its scores grew by more than about 20 in log2 units, as
      // at a planted needle -- does the warp take the row max, rescale l and O
      // lazily (growth above 2^8) and redo the tile.  P <= 2^20 per tile keeps
      // l and O far from fp32 overflow over any T this kernel takes.
      float rs[4] = {0.f, 0.f, 0.f, 0.f};   // independent partial row sums
      // xv(i) reads score i; unrolled, every index is a compile-time constant.
      auto exp_pass = [&](float m_use, auto&& xv) {
#pragma unroll
        for (int c = 0; c < kBN / 32; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float p0 = ex2(fmaf(xv(c * 32 + 2 * e), a.scale_log2, -m_use));
            const float p1 = ex2(fmaf(xv(c * 32 + 2 * e + 1), a.scale_log2, -m_use));
            rs[e & 3] += p0 + p1;
            pk[e] = pack_bf16x2(p0, p1);
          }
          tmem_st16(tS + c * 16, pk);   // P_i over S_i's first 64 columns
        }
      };
      bool redo = m_run == -INFINITY;
      if (!__any_sync(0xffffffffu, redo)) {
        exp_pass(m_run, [&](int i) { return x[i]; });
        redo = !((rs[0] + rs[1]) + (rs[2] + rs[3]) <= kRedoSum);
      }
      if (__any_sync(0xffffffffu, redo)) {
        // P overwrote columns 0-63 only: scores 64-127 are read back from TMEM,
        // 0-63 are still in registers.
        float xh[kBN / 2];
        {
          uint32_t v[2][32];
          tmem_ld32(tS + 64, v[0]);
          tmem_ld32(tS + 96, v[1]);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            xh[e] = __uint_as_float(v[0][e]);
            xh[32 + e] = __uint_as_float(v[1][e]);
          }
          if (need_mask) {
#pragma unroll
            for (int c = kBN / 2; c < kBN; ++c)
              if (J * kBN + c > t_row || !((sub >> (c >> 6)) & 1u)) xh[c - kBN / 2] = -INFINITY;
          }
        }
        auto xr = [&](int i) { return i < kBN / 2 ? x[i] : xh[i - kBN / 2]; };
        // Row max with 8 independent accumulators (a 127-deep chain otherwise).
        float mx[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) mx[e] = xr(e);
#pragma unroll
        for (int c = 8; c < kBN; ++c) mx[c & 7] = fmaxf(mx[c & 7], xr(c));
        const float mt = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                               fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
        const float m_tile = mt * a.scale_log2;
        const bool grow = m_tile > m_run + kRescaleLog2;
        float alpha = 1.f;
        if (grow) {
          alpha = ex2(m_run - m_tile);
          l_run *= alpha;
          m_run = m_tile;
        }
        rs[0] = rs[1] = rs[2] = rs[3] = 0.f;
        tmem_wait_st();   // the first pass's P stores land before these replace them
        exp_pass(m_run == -INFINITY ? 0.f : m_run, xr);
        if (j > 0 && __any_sync(0xffffffffu, grow)) {
          // O_i is stable: S_i(j) completing implies PV_i(j-1) completed, and
          // PV_i(j) waits for this warpgroup's arrival below.
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t v[32];
            tmem_ld32(tO + c * 32, v);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
            tmem_st32(tO + c * 32, v);
          }
        }
      }
      l_run += (rs[0] + rs[1]) + (rs[2] + rs[3]);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars[B_PF + i]);
    }

    // ------------------------------------------------------------ epilogue
    const size_t row_elem = ((static_cast<size_t>(b) * a.T + t_row) * a.Hq + h) * D;
    const bool valid = t_row < a.T;
    // One decision per warpgroup (a named barrier below needs all 128 threads).
    // Barrier instructions are warp-aligned and lanes may have left the tile
    // loop apart (a wait that gave up), so the warp reconverges first.
    const bool mine = n > 0 && ok && mbar_wait(&bars[B_OD], 0, a.st);
    __syncwarp();
    const bool have_o = named_bar_and(1 + i, 128, mine);
    if (have_o && !a.blend_score) {
      // O_i / l -> bf16 rows staged in Q_i's (now free: every MMA has completed)
      // shared memory in the 128-byte swizzled box layout, then stored by TMA:
      // one 16-byte chunk per st.shared, conflict-free, no strided global stores.
      tc_fence_after();
      const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
      const uint32_t stage = smem_u32(sQ) + i * CH * kChunkBytes + r * 128;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tO + c * 32, v);
        tmem_wait_ld();
        const uint32_t box = stage + (c >> 1) * kChunkBytes;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint32_t k16 = static_cast<uint32_t>((c & 1) * 4 + u);
          st_shared_v4(box + ((k16 ^ static_cast<uint32_t>(r & 7)) << 4),
                       pack_bf16x2(__uint_as_float(v[u * 8 + 0]) * inv, __uint_as_float(v[u * 8 + 1]) * inv),
                       pack_bf16x2(__uint_as_float(v[u * 8 + 2]) * inv, __uint_as_float(v[u * 8 + 3]) * inv),
                       pack_bf16x2(__uint_as_float(v[u * 8 + 4]) * inv, __uint_as_float(v[u * 8 + 5]) * inv),
                       pack_bf16x2(__uint_as_float(v[u * 8 + 6]) * inv, __uint_as_float(v[u * 8 + 7]) * inv));
        }
      }
      if (valid && a.lse) {
        a.lse[(static_cast<size_t>(b) * a.Hq + h) * a.T + t_row] =
            l_run > 0.f ? (m_run + __log2f(l_run)) * 0.69314718055994531f : -INFINITY;
      }
      fence_proxy_async_smem();
      named_bar_sync(1 + i, 128);
      const int tile_row = row0 + i * row_step;
      if (r == 0 && tile_row < a.T) {
        // Rows past T are clipped by the tensor map; the CTA's smem stays valid
        // until the copy has read it.
#pragma unroll
        for (int c = 0; c < CH; ++c)
          tma_store_4d(&tm_o, sQ + (i * CH + c) * kChunkBytes, c * 64, h, tile_row, b);
        bulk_commit_group();
        bulk_wait_read0();
      }
    } else if (have_o) {
      // Soft routing: blend with the row already in o (the other path's output).
      tc_fence_after();
      const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
      const float rb = a.blend_score[a.layer];
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tO + c * 32, v);
        tmem_wait_ld();
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(a.o + row_elem + c * 32);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const uint4 prev = dst[u];
            const uint32_t pw[4] = {prev.x, prev.y, prev.z, prev.w};
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
              w[e] = pack_bf16x2(
                  fmaf(rb, bf16lo_to_f32(pw[e]), (1.f - rb) * __uint_as_float(v[u * 8 + 2 * e]) * inv),
                  fmaf(rb, bf16hi_to_f32(pw[e]),
                       (1.f - rb) * __uint_as_float(v[u * 8 + 2 * e + 1]) * inv));
            dst[u] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
      if (valid && a.lse) {
        a.lse[(static_cast<size_t>(b) * a.Hq + h) * a.T + t_row] =
            l_run > 0.f ? (m_run + __log2f(l_run)) * 0.69314718055994531f : -INFINITY;
      }
    } else if (valid) {
      // No visible key (or an aborted tile): this pass contributes zero.
      uint4* dst = reinterpret_cast<uint4*>(a.o + row_elem);
      const float rb = a.blend_score ? a.blend_score[a.layer] : 0.f;
      for (int u = 0; u < D / 8; ++u) {
        uint4 w = make_uint4(0, 0, 0, 0);
        if (a.blend_score) {
          const uint4 prev = dst[u];
          w.x = pack_bf16x2(rb * bf16lo_to_f32(prev.x), rb * bf16hi_to_f32(prev.x));
          w.y = pack_bf16x2(rb * bf16lo_to_f32(prev.y), rb * bf16hi_to_f32(prev.y));
          w.z = pack_bf16x2(rb * bf16lo_to_f32(prev.z), rb * bf16hi_to_f32(prev.z));
          w.w = pack_bf16x2(rb * bf16lo_to_f32(prev.w), rb * bf16hi_to_f32(prev.w));
        }
        dst[u] = w;
      }
      if (a.lse) a.lse[(static_cast<size_t>(b) * a.Hq + h) * a.T + t_row] = -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

int prefill_smem_bytes(int d) { return d == 64 ? Smem<64>::ALLOC : Smem<128>::ALLOC; }

cudaError_t launch_prefill(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                           const CUtensorMap& to, const PrefillLaunch& p, cudaStream_t stream) {
  PrefillArgs a;
  a.B = p.B;
  a.T = p.T;
  a.Hq = p.Hq;
  a.Hkv = p.Hkv;
  a.G = p.Hq / p.Hkv;
  // Head pairs need both heads of a pair in one KV group and on one path.
  a.head_pair = (a.G % 2 == 0 && p.head_mode == nullptr) ? 1 : 0;
  a.nunit = a.head_pair ? (p.T + kBM - 1) / kBM : (p.T + 2 * kBM - 1) / (2 * kBM);
  a.nkt = (p.T + kBN - 1) / kBN;
  // As many kv groups per chunk (a divisor of Hkv) as keep their K and V
  // within 48 MB, inside L2 beside the Q and O streams, so that the CTAs in
  // flight re-read K and V from L2 rather than DRAM (measured at T 65536 in a
  // power-capped run of FA layers: the same time as a 72 MB chunk, which let
  // DRAM reads reach about 1.9x the algorithmic bytes).
  {
    const long long kv_bytes = 4LL * p.T * p.d;   // K + V of one group, bf16
    a.gchunk = 1;
    for (int gcand = p.Hkv; gcand > 1; --gcand)
      if (p.Hkv % gcand == 0 && gcand * kv_bytes <= (48LL << 20)) { a.gchunk = gcand; break; }
  }
  a.block = p.block;
  a.nqb = p.nqb;
  a.nkb = (p.T + p.block - 1) / p.block;
  a.scale_log2 = p.scale * 1.4426950408889634f;
  a.layer_mode = p.layer_mode;
  a.layer = p.layer;
  a.row_ptr = p.row_ptr;
  a.col = p.col;
  a.o = p.o;
  a.lse = p.lse;
  a.force_mode = p.force_mode;
  a.head_mode = p.head_mode;
  a.blend_score = p.blend_score;
  a.st = p.st;
  const dim3 grid(static_cast<unsigned>(a.nunit) * (a.head_pair ? p.Hq / 2 : p.Hq) * p.B);
  if (p.d == 64) {
    const int smem = Smem<64>::ALLOC;
    cudaFuncSetAttribute(prefill_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    prefill_kernel<64><<<grid, kThreads, smem, stream>>>(tq, tk, tv, to, a);
  } else {
    const int smem = Smem<128>::ALLOC;
    cudaFuncSetAttribute(prefill_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    prefill_kernel<128><<<grid, kThreads, smem, stream>>>(tq, tk, tv, to, a);
  }
  return cudaGetLastError();
}

}  // namespace flux
