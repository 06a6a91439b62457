// decode.cu -- split-KV decode attention for one layer on sm_100a.
//
// One new query token per sequence attends the KV cache (gist.science
// summary "Flux Attention", section 2, "efficient deployment": the routing
// bit chosen at prefill is reused at every decode step; SA layers read only
// the sink blocks and the most recent W blocks, never the history between).
// Decode is bound by HBM bandwidth (section 1 of the same summary), so the
// kernel is built around the KV stream:
//   * grid (kv head, sequence, split), split slowest; each CTA streams one chunk of one
//     (sequence, kv head) and serves all G = Hq/Hkv query heads of the group
//     from that single read;
//   * a producer warp moves 64-token K and V tiles by TMA (128-byte swizzle)
//     into a 3-stage ring; four compute warps each own a 16-token slice of
//     every tile, so the loop has no block barrier: a stage is released by an
//     mbarrier that counts the four warps;
//   * per warp, the group's scores S[G x 16] = Q K^T and values O += P V are
//     16x8x16 warp MMAs (bf16 in, fp32 accumulate) fed by ldmatrix straight
//     from the swizzled tiles -- the G <= 8 query heads fill rows 0..G-1 of the
//     16-row operand (G is a launch argument, not a template parameter); online
//     softmax in the log2 domain on the accumulator fragments, O rescaled only
//     when a row max grows by more than 2^8;
//   * the four warps' partials are merged in shared memory, then the last
//     active CTA of each (sequence, kv head) -- found by an atomic ticket, no
//     spin -- merges the partial (o, m, l) of every active split; splits past
//     the active range (most of an SA layer's grid) exit at entry;
//   * the cache is either full (row = position) or, for an SA layer, the
//     compact ring of its sink blocks and last W blocks (block j >= sink in
//     slot j mod W); with the step's new K/V rows passed in, the split that
//     reads token s - 1 writes them into the cache before loading its tiles
//     (the KV append fused into the decode launch).
// About 160 registers (d 128) and 97 KB of shared memory: two CTAs per SM.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace flux {

namespace {

constexpr int kTok = 64;        // tokens per tile (4 warps x 16)
constexpr int kStages = 3;
constexpr int kComputeWarps = 4;
constexpr int kThreads = 32 * (kComputeWarps + 1);
constexpr float kRescaleLog2 = 8.f;
constexpr int kMaxGroup = kDecodeMaxGroup;   // query heads per kv head: operand rows 0..7

template <int D>
struct DSmem {
  static constexpr int CH = D / 64;                // 64-channel swizzle boxes per row
  static constexpr int BOX = kTok * 128;           // one box: 64 tokens x 128 bytes
  static constexpr int KT = CH * BOX;              // K tile bytes
  static constexpr int STAGE = 2 * KT;             // K + V
  static constexpr int BARS = kStages * STAGE;     // full[kStages], empty[kStages]
  static constexpr int FLAG = BARS + 2 * kStages * 8;
  static constexpr int TOTAL = FLAG + 16;
  static constexpr int ALLOC = TOTAL + 1024;
  // After the stream: per-warp partials m, l [warp][kMaxGroup] and o[warp][kMaxGroup][D].
  static constexpr int CM = 0, CL = CM + kComputeWarps * kMaxGroup * 4;
  static constexpr int CO = CL + kComputeWarps * kMaxGroup * 4;
  static_assert(CO + kComputeWarps * kMaxGroup * D * 4 <= BARS, "combine area must fit in the ring");
};

// A split's 64-token tiles.  FA: a contiguous token range.  SA: the sink
// segment [0, n_sink) and the window segment [win_start, s) are tiled
// separately and their tiles numbered consecutively (sink tiles first); split i
// takes tiles [i * tiles_sa, (i + 1) * tiles_sa), so one split may hold sink
// tiles followed by window tiles.
struct Range {
  bool fa;
  int start, end;    // FA: tokens [start, end)
  int v0, v1;        // SA: virtual tiles [v0, v1)
  int t_sink;        // SA: tiles of the sink segment
  int n_sink;        // SA: tokens of the sink segment
  int win_start, s;  // SA: window segment [win_start, s)
  int ntiles;
  int n_active;      // active splits of this (sequence, kv head)
  // Does this split read token u?
  __device__ __forceinline__ bool holds(int u) const {
    if (ntiles == 0 || u < 0) return false;
    if (fa) return start <= u && u < end;
    int vt;
    if (u < n_sink) vt = u / 64;
    else if (u >= win_start && u < s) vt = t_sink + (u - win_start) / 64;
    else return false;
    return v0 <= vt && vt < v1;
  }
  // Tile k of this split: tokens [*t0, *t1).
  __device__ __forceinline__ void tile(int k, int* t0, int* t1) const {
    if (fa) {
      *t0 = start + k * 64;
      *t1 = end;
    } else {
      const int vt = v0 + k;
      if (vt < t_sink) {
        *t0 = vt * 64;
        *t1 = n_sink;
      } else {
        *t0 = win_start + (vt - t_sink) * 64;
        *t1 = s;
      }
    }
  }
};

__device__ __forceinline__ Range split_range(const DecodeLaunch& a, bool fa, int s, int i) {
  Range r{};
  r.fa = fa;
  if (s <= 0) return r;
  if (fa) {
    r.n_active = (s + a.chunk_fa - 1) / a.chunk_fa;
    r.start = i * a.chunk_fa;
    r.end = min(r.start + a.chunk_fa, s);
    r.ntiles = r.end > r.start ? (r.end - r.start + kTok - 1) / kTok : 0;
  } else {
    const int blk = a.block;
    r.s = s;
    r.n_sink = min(a.sink_blocks * blk, s);
    const int nbs = (s + blk - 1) / blk;
    r.win_start = max(r.n_sink, max(0, nbs - a.window_blocks) * blk);
    r.t_sink = (r.n_sink + kTok - 1) / kTok;
    const int total = r.t_sink + (s - r.win_start + kTok - 1) / kTok;
    r.n_active = (total + a.tiles_sa - 1) / a.tiles_sa;
    r.v0 = i * a.tiles_sa;
    r.v1 = min(r.v0 + a.tiles_sa, total);
    r.ntiles = r.v1 > r.v0 ? r.v1 - r.v0 : 0;
  }
  if (i >= r.n_active) r.ntiles = 0;
  return r;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 2)
    decode_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                  const DecodeLaunch a) {
  using L = DSmem<D>;
  constexpr int KS = D / 16;        // k-steps of the score MMA
  constexpr int NT = D / 8;         // n-tiles of the value MMA
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::BARS);
  uint64_t* empty = full + kStages;
  int* flag = reinterpret_cast<int*>(smem + L::FLAG);

  // Split-major grid: every group's split 0 is dispatched first, so the active
  // CTAs of an SA layer (low splits) run in the first wave and the splits it
  // leaves idle (launched for the FA range) only exit after them.
  const int i = blockIdx.z, g = blockIdx.x, b = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // Launched with programmatic stream serialisation: the next decode launch may
  // be dispatched as soon as every CTA of this one has started, and this CTA
  // starts before the previous kernel has finished.  Everything below reads or
  // writes memory that kernel may touch (routing bits, lengths, q, the cache,
  // the split partials and merge tickets of a shared workspace), so it waits
  // for that kernel first; what overlaps is the launch and the CTA dispatch.
  griddep_launch_dependents();
  // This CTA's own barriers and the tensor-map descriptors (launch parameters)
  // owe nothing to the previous kernel: they are set up while it finishes.
  if (tid == 0) {
    for (int st = 0; st < kStages; ++st) {
      mbar_init(&full[st], 1);
      mbar_init(&empty[st], kComputeWarps);
    }
    fence_barrier_init();
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  griddep_wait();
  const int G = a.Hq / a.Hkv;   // 1..kMaxGroup, checked on the host
  // Per-head routing: the group reads the FA range if any of its heads is FA;
  // its SA heads then mask every token outside the sink + window blocks.
  const uint8_t* hm = a.head_mode ? a.head_mode + g * G : nullptr;
  bool fa;
  if (hm) {
    fa = false;
    for (int hh = 0; hh < G; ++hh) fa |= hm[hh] != 0;
  } else {
    fa = !a.compact && (a.layer_mode == nullptr || a.layer_mode[a.layer] != 0);
  }
  int s = a.seqlens[b];
  if (s < 0 || (!a.compact && s > a.S_max) || (a.k_new && s < 1)) {
    if (i == 0 && g == 0 && tid == 0) raise_error(a.st.err, DEV_ERR_SEQLEN);
    s = 0;
  }
  const Range rg = split_range(a, fa, s, i);
  const int ntiles = rg.ntiles;
  const size_t grp = static_cast<size_t>(b) * a.Hq + g * G;  // first query head of the group
  if (ntiles == 0) {
    // Splits past the active range exit at once (SA layers use only a few);
    // with no visible token at all, split 0 writes the zero output.
    if (i == 0 && rg.n_active == 0) {
      for (int idx = tid; idx < G * D; idx += kThreads) {
        reinterpret_cast<__nv_bfloat16*>(a.o)[grp * D + idx] = __float2bfloat16_rn(0.f);
        if (idx % D == 0 && a.lse) a.lse[grp + idx / D] = -INFINITY;
      }
    }
    return;
  }

  __syncthreads();   // the barriers initialised above are visible to every warp

  const int gq = lane >> 2, tq = lane & 3;   // fragment row (head) and column pair
  float m_run = -INFINITY, l_part = 0.f;
  float oacc[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n) oacc[n][0] = oacc[n][1] = oacc[n][2] = oacc[n][3] = 0.f;
  bool ok = true;

  if (warp == kComputeWarps) {
    // ------------------------------------------------------------ producer
    if (a.k_new && rg.holds(s - 1)) {
      // Fused append: this split reads token s - 1, so it writes the new K/V
      // rows into the cache (the ring slot of the token's block when compact)
      // before any of its tiles is loaded; no other CTA reads that row.
      const int u = s - 1;
      int row = u;
      if (a.compact && u >= a.sink_blocks * a.block) {
        const int j = u / a.block;
        row = (a.sink_blocks + j % a.window_blocks) * a.block + u % a.block;
      }
      const size_t dst = ((static_cast<size_t>(b) * a.S_max + row) * a.Hkv + g) * D;
      const size_t src = (static_cast<size_t>(b) * a.Hkv + g) * D;
      if (lane < D / 8) {
        reinterpret_cast<uint4*>(a.k_cache + dst)[lane] =
            reinterpret_cast<const uint4*>(a.k_new + src)[lane];
        reinterpret_cast<uint4*>(a.v_cache + dst)[lane] =
            reinterpret_cast<const uint4*>(a.v_new + src)[lane];
      }
      fence_proxy_async_global();
      __syncwarp();
    }
    if (lane == 0 && ntiles > 0) {
      int issued = 0;
      for (int k = 0; k < ntiles; ++k) {
        const int st = k % kStages;
        if (k >= kStages && !mbar_wait(&empty[st], ((k / kStages) - 1) & 1, a.st)) {
          ok = false;
          break;
        }
        uint8_t* kb = smem + st * L::STAGE;
        uint8_t* vb = kb + L::KT;
        mbar_arrive_expect_tx(&full[st], 2 * L::KT);
        int row, t_end;
        rg.tile(k, &row, &t_end);
        if (a.compact && row >= a.sink_blocks * a.block) {
          // Ring slot of the token's block (a 64-token tile never straddles blocks).
          const int j = row / a.block;
          row = (a.sink_blocks + j % a.window_blocks) * a.block + row % a.block;
        }
        for (int c = 0; c < L::CH; ++c) {
          tma_load_4d(&tm_k, &full[st], kb + c * L::BOX, c * 64, g, row, b);
          tma_load_4d(&tm_v, &full[st], vb + c * L::BOX, c * 64, g, row, b);
        }
        issued = k + 1;
      }
      // Every copy issued lands before the ring is reused for the merge, also
      // when the compute warps gave up early.
      for (int k = max(0, issued - kStages); k < issued; ++k)
        mbar_drain(&full[k % kStages], (k / kStages) & 1);
    }
  } else if (ntiles > 0) {
    // ------------------------------------------------------------ compute warps
    // Q fragments (rows = the group's G heads, zero beyond), A of the score MMA.
    uint32_t qa[KS][4];
    {
      const uint32_t* qrow = reinterpret_cast<const uint32_t*>(
          a.q + (static_cast<size_t>(b) * a.Hq + g * G + (gq < G ? gq : 0)) * D);
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        qa[ks][0] = gq < G ? qrow[ks * 8 + tq] : 0u;
        qa[ks][2] = gq < G ? qrow[ks * 8 + 4 + tq] : 0u;
        qa[ks][1] = qa[ks][3] = 0u;
      }
    }
    const float sl2 = a.scale * 1.4426950408889634f;
    const int mrow = lane & 7, msel = lane >> 3;     // ldmatrix row and matrix index
    const bool row_sa = fa && hm != nullptr && gq < G && hm[gq] == 0;
    const int nbs = (s + a.block - 1) / a.block;
    const int wtok = warp * 16;
    for (int k = 0; k < ntiles; ++k) {
      const int st = k % kStages;
      if (!mbar_wait(&full[st], (k / kStages) & 1, a.st)) { ok = false; break; }
      const uint32_t kb = smem_u32(smem + st * L::STAGE);
      const uint32_t vb = kb + L::KT;
      // ---- scores: S[head][token] for this warp's 16 tokens (two n-tiles of 8)
      float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      {
        const int tok = wtok + (msel >> 1) * 8 + mrow;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          const int uu = 2 * ks + (msel & 1);
          const uint32_t addr = kb + (uu >> 3) * L::BOX + tok * 128 + (((uu & 7) ^ (tok & 7)) << 4);
          uint32_t b00, b01, b10, b11;
          ldmatrix_x4(addr, b00, b01, b10, b11);
          mma_bf16_16816(sc[0], qa[ks], b00, b01);
          mma_bf16_16816(sc[1], qa[ks], b10, b11);
        }
      }
      // ---- online softmax on the fragment: row gq, tokens 8n + 2tq + e
      int t_begin, t_end;
      rg.tile(k, &t_begin, &t_end);
      const int tok0 = t_begin + wtok + 2 * tq;
      float x[4];
#pragma unroll
      for (int n = 0; n < 2; ++n)
#pragma unroll
        for (int e = 0; e < 2; ++e)
        {
          const int u = tok0 + 8 * n + e;
          const bool keep = gq < G && u < t_end &&
                            (!row_sa || u / a.block < a.sink_blocks ||
                             u / a.block >= nbs - a.window_blocks);
          x[n * 2 + e] = keep ? sc[n][e] : -INFINITY;
        }
      float mt = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
      mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 1));
      mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 2));
      const float m_tile = mt * sl2;
      const bool grow = m_tile > m_run + kRescaleLog2;
      float alpha = 1.f;
      if (grow) {
        alpha = ex2(m_run - m_tile);
        l_part *= alpha;
        m_run = m_tile;
      }
      if (__any_sync(0xffffffffu, grow)) {
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          oacc[n][0] *= alpha;
          oacc[n][1] *= alpha;
        }
      }
      const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
      float p[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        p[e] = ex2(fmaf(x[e], sl2, -m_use));
        l_part += p[e];
      }
      const uint32_t pa[4] = {pack_bf16x2(p[0], p[1]), 0u, pack_bf16x2(p[2], p[3]), 0u};
      // ---- values: O[head][d] += P[head][16 tokens] V[16 tokens][d]
      {
        const int tok = wtok + (msel & 1) * 8 + mrow;
#pragma unroll
        for (int np = 0; np < NT / 2; ++np) {
          const int uu = 2 * np + (msel >> 1);
          const uint32_t addr = vb + (uu >> 3) * L::BOX + tok * 128 + (((uu & 7) ^ (tok & 7)) << 4);
          uint32_t b0a, b1a, b0b, b1b;
          ldmatrix_x4_trans(addr, b0a, b1a, b0b, b1b);
          mma_bf16_16816(oacc[2 * np], pa, b0a, b1a);
          mma_bf16_16816(oacc[2 * np + 1], pa, b0b, b1b);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
    }
  }
  __syncthreads();

  // ---- merge the four warps' partials in shared memory (the ring is free now)
  float* cm = reinterpret_cast<float*>(smem + L::CM);
  float* cl = reinterpret_cast<float*>(smem + L::CL);
  float* co = reinterpret_cast<float*>(smem + L::CO);
  if (warp < kComputeWarps) {
    float lq = l_part;
    lq += __shfl_xor_sync(0xffffffffu, lq, 1);
    lq += __shfl_xor_sync(0xffffffffu, lq, 2);
    if (gq < G) {
      if (tq == 0) {
        cm[warp * kMaxGroup + gq] = (ntiles > 0) ? m_run : -INFINITY;
        cl[warp * kMaxGroup + gq] = (ntiles > 0) ? lq : 0.f;
      }
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        co[(warp * kMaxGroup + gq) * D + 8 * n + 2 * tq] = oacc[n][0];
        co[(warp * kMaxGroup + gq) * D + 8 * n + 2 * tq + 1] = oacc[n][1];
      }
    }
  }
  __syncthreads();
  {
    for (int idx = tid; idx < G * D; idx += kThreads) {
      const int hh = idx / D, c = idx % D;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kComputeWarps; ++w) M = fmaxf(M, cm[w * kMaxGroup + hh]);
      float O = 0.f, Lsum = 0.f;
      if (M != -INFINITY) {
#pragma unroll
        for (int w = 0; w < kComputeWarps; ++w) {
          const float wt = ex2(cm[w * kMaxGroup + hh] - M);
          O += wt * co[(w * kMaxGroup + hh) * D + c];
          Lsum += wt * cl[w * kMaxGroup + hh];
        }
      }
      a.part_o[((grp + hh) * a.nsplit + i) * D + c] = O;
      if (c == 0) {
        a.part_ml[((grp + hh) * a.nsplit + i) * 2 + 0] = M;
        a.part_ml[((grp + hh) * a.nsplit + i) * 2 + 1] = Lsum;
      }
    }
  }

  // ---- ticket: the last CTA of this (sequence, kv head) merges the splits
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const int old = atomicAdd(&a.tickets[b * a.Hkv + g], 1);
    *flag = (old == rg.n_active - 1);
  }
  __syncthreads();
  if (!*flag) return;
  __threadfence();
  const int na = rg.n_active;
  for (int idx = tid; idx < G * D; idx += kThreads) {
    const int hh = idx / D, c = idx % D;
    const size_t base = (grp + hh) * a.nsplit;
    float M = -INFINITY;
    for (int sp = 0; sp < na; ++sp) M = fmaxf(M, __ldcg(&a.part_ml[(base + sp) * 2]));
    float Lsum = 0.f, O = 0.f;
    if (M != -INFINITY) {
      for (int sp = 0; sp < na; ++sp) {
        const float w = ex2(__ldcg(&a.part_ml[(base + sp) * 2]) - M);
        Lsum += w * __ldcg(&a.part_ml[(base + sp) * 2 + 1]);
        O += w * __ldcg(&a.part_o[(base + sp) * D + c]);
      }
    }
    const float out = Lsum > 0.f ? O / Lsum : 0.f;
    reinterpret_cast<__nv_bfloat16*>(a.o)[(grp + hh) * D + c] = __float2bfloat16_rn(out);
    if (c == 0 && a.lse)
      a.lse[grp + hh] = Lsum > 0.f ? (M + __log2f(Lsum)) * 0.69314718055994531f : -INFINITY;
  }
  if (tid == 0) a.tickets[b * a.Hkv + g] = 0;
}

template <int D>
cudaError_t launch_t(const CUtensorMap& tk, const CUtensorMap& tv, const DecodeLaunch& p,
                     cudaStream_t stream) {
  const int smem = DSmem<D>::ALLOC;
  cudaFuncSetAttribute(decode_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  // Programmatic stream serialisation: consecutive decode launches (one per
  // layer) overlap the next launch's dispatch with this one's tail.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.Hkv, p.B, p.nsplit);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_kernel<D>, tk, tv, p);
}

}  // namespace

void decode_plan(int B, int Hkv, int S_max, int sink_blocks, int window_blocks, int block,
                 int num_sms, int* nsplit, int* chunk_fa, int* tiles_sa) {
  const long long groups = static_cast<long long>(B) * Hkv;
  const long long slots = 2LL * num_sms;   // two CTAs per SM
  // FA: few, long splits -- about 1.75 waves of CTAs in all (the tail wave
  // still holds enough streams to keep HBM busy; fewer splits mean fewer CTA
  // ramps and partials to merge, and fewer CTAs left idle when the layer
  // turns out to be SA).  Measured on one GPU at 131072 tokens: batch 16 (128
  // groups) 1.186 ms with 4 splits against 1.248 ms with 64 (2048-token
  // chunks); batch 4: 325-332 us for 2-18 splits against 353 us with 64.
  int ns = static_cast<int>((7 * slots + 2 * groups) / (4 * groups));   // round(1.75 slots / groups)
  const int max_ns = (S_max + kTok - 1) / kTok;
  if (ns > max_ns) ns = max_ns;
  if (ns < 1) ns = 1;
  // SA: the sink and window tiles of a sequence, split as little as possible
  // (every CTA pays a fixed ramp -- first loads, q, the merge -- worth several
  // tiles) while the active CTAs still fill at least half of the resident
  // slots, and within one wave where the groups allow it.  At batch 16, 8 kv
  // heads (128 groups, 296 slots) this is 2 splits of 17 tiles: measured on
  // one GPU, 33.6 us against 39.3 us for 3 splits of 12 (1.3 waves) and far
  // slower for 1-tile splits.
  const long long sa_tiles = (static_cast<long long>(sink_blocks) * block + kTok - 1) / kTok +
                             (static_cast<long long>(window_blocks) * block + kTok - 1) / kTok;
  long long sa_splits = (slots + 2 * groups - 1) / (2 * groups);   // fill half the slots
  const long long one_wave = std::max<long long>(1, slots / groups);
  sa_splits = std::max<long long>(1, std::min(sa_splits, one_wave));
  if (sa_splits > sa_tiles) sa_splits = std::max<long long>(1, sa_tiles);
  long long tsa = sa_tiles > 0 ? (sa_tiles + sa_splits - 1) / sa_splits : 1;
  const long long need_sa = (sa_tiles + tsa - 1) / tsa;
  ns = static_cast<int>(std::max<long long>(ns, need_sa));
  if (ns > 65535) {   // grid z limit (not reached: both plans stay within a wave or two)
    ns = 65535;       // the FA chunks and the SA tiles per split grow instead
    tsa = std::max<long long>(tsa, (sa_tiles + ns - 1) / ns);
  }
  int cfa = (S_max + ns - 1) / ns;
  cfa = ((cfa + kTok - 1) / kTok) * kTok;
  if (cfa < kTok) cfa = kTok;
  *nsplit = ns;
  *chunk_fa = cfa;
  *tiles_sa = static_cast<int>(tsa);
}

int decode_sa_splits(int sink_blocks, int window_blocks, int block, int tiles_sa) {
  const long long sa_tiles = (static_cast<long long>(sink_blocks) * block + kTok - 1) / kTok +
                             (static_cast<long long>(window_blocks) * block + kTok - 1) / kTok;
  const long long t = tiles_sa > 0 ? tiles_sa : 1;
  return static_cast<int>(std::max<long long>(1, (sa_tiles + t - 1) / t));
}

size_t decode_workspace_bytes(int B, int Hq, int Hkv, int d, int nsplit) {
  const size_t rows = static_cast<size_t>(B) * Hq * nsplit;
  size_t bytes = rows * d * sizeof(float);
  bytes = (bytes + 255) & ~size_t(255);
  bytes += ((rows * 2 * sizeof(float)) + 255) & ~size_t(255);
  bytes += ((static_cast<size_t>(B) * Hkv * sizeof(int)) + 255) & ~size_t(255);
  return bytes;
}

cudaError_t launch_decode(const CUtensorMap& tk, const CUtensorMap& tv, const DecodeLaunch& p,
                          cudaStream_t stream) {
  if (p.Hkv < 1 || p.Hq % p.Hkv != 0 || p.Hq / p.Hkv > kMaxGroup || (p.d != 64 && p.d != 128))
    return cudaErrorInvalidValue;
  return p.d == 64 ? launch_t<64>(tk, tv, p, stream) : launch_t<128>(tk, tv, p, stream);
}

}  // namespace flux
