// decode.cu -- split-KV decode attention for one layer on sm_100a.
//
// One new query token per sequence attends the KV cache (gist.science
// summary "Flux Attention", section 2, "efficient deployment": the routing
// bit chosen at prefill is reused at every decode step; SA layers read only
// the sink blocks and the most recent W blocks, never the history between).
// Decode is bound by HBM bandwidth (section 1 of the same summary), so the
// kernel is built around the KV stream:
//   * grid (split, kv head, sequence); each CTA streams one chunk of one
//     (sequence, kv head) and serves all G = Hq/Hkv query heads of that group
//     from the single read;
//   * 64-token K and V tiles arrive by TMA (128-byte swizzle, so that the
//     per-token and per-channel shared-memory reads are conflict-free) into a
//     4-stage ring guarded by mbarriers;
//   * scores: 4 threads per token, fp32 FMAs on bf16 data widened in
//     registers, a 2-step shuffle to combine the quarters, online softmax in
//     the log2 domain;
//   * values: each thread owns 8 channels of all G heads for a subset of the
//     tile's tokens; the subsets are combined once per CTA;
//   * the last CTA of each (sequence, kv head) -- found by an atomic ticket,
//     no spin -- merges the partial (o, m, l) of every active split.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace flux {

namespace {

constexpr int kTok = 64;        // tokens per tile
constexpr int kStages = 4;
constexpr int kThreads = 256;

template <int D>
struct DSmem {
  static constexpr int CH = D / 64;                // 64-channel swizzle boxes per row
  static constexpr int BOX = kTok * 128;           // one box: 64 tokens x 128 bytes
  static constexpr int KT = CH * BOX;              // K tile bytes
  static constexpr int STAGE = 2 * KT;             // K + V
  static constexpr int P = kStages * STAGE;        // p[64][4] fp32
  static constexpr int RED = P + kTok * 16;        // [8 warps][4] fp32
  static constexpr int BARS = RED + 8 * 4 * 4;
  static constexpr int FLAG = BARS + kStages * 8;
  static constexpr int TOTAL = FLAG + 16;
  static constexpr int ALLOC = TOTAL + 1024;
};

struct Range {
  int start, end;  // tokens [start, end) of this split
  int n_active;    // active splits of this (sequence, kv head)
};

__device__ __forceinline__ Range split_range(const DecodeLaunch& a, bool fa, int s, int i) {
  Range r{0, 0, 0};
  if (s <= 0) return r;
  if (fa) {
    r.n_active = (s + a.chunk_fa - 1) / a.chunk_fa;
    r.start = i * a.chunk_fa;
    r.end = min(r.start + a.chunk_fa, s);
  } else {
    const int blk = a.block;
    const int n_sink = min(a.sink_blocks * blk, s);
    const int nbs = (s + blk - 1) / blk;
    const int win_start = max(n_sink, max(0, nbs - a.window_blocks) * blk);
    const int n_win = s - win_start;
    const int sp_sink = (n_sink + a.chunk_sa - 1) / a.chunk_sa;
    const int sp_win = (n_win + a.chunk_sa - 1) / a.chunk_sa;
    r.n_active = sp_sink + sp_win;
    if (i < sp_sink) {
      r.start = i * a.chunk_sa;
      r.end = min(r.start + a.chunk_sa, n_sink);
    } else if (i < r.n_active) {
      r.start = win_start + (i - sp_sink) * a.chunk_sa;
      r.end = min(r.start + a.chunk_sa, s);
    }
  }
  if (i >= r.n_active) r.start = r.end = 0;
  return r;
}

template <int D, int G>
__global__ void __launch_bounds__(kThreads, 1)
    decode_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                  const DecodeLaunch a) {
  using L = DSmem<D>;
  constexpr int QW = D / 4;          // channels per quarter-thread in the score phase
  constexpr int NCH = D / 8;         // 8-channel units per row
  constexpr int NSUB = kThreads / NCH;   // token subsets in the value phase
  constexpr int TPS = kTok / NSUB;       // tokens per thread per tile in the value phase
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  float* p_s = reinterpret_cast<float*>(smem + L::P);
  float* red = reinterpret_cast<float*>(smem + L::RED);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::BARS);
  int* flag = reinterpret_cast<int*>(smem + L::FLAG);

  const int i = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool fa = a.layer_mode == nullptr || a.layer_mode[a.layer] != 0;
  int s = a.seqlens[b];
  if (s < 0 || s > a.S_max) {
    if (i == 0 && g == 0 && tid == 0) raise_error(a.st.err, DEV_ERR_SEQLEN);
    s = 0;
  }
  const Range rg = split_range(a, fa, s, i);
  const int ntiles = (rg.end - rg.start + kTok - 1) / kTok;

  if (tid == 0) {
    for (int st = 0; st < kStages; ++st) mbar_init(&full[st], 1);
    fence_barrier_init();
  }
  __syncthreads();

  auto issue = [&](int k) {
    const int st = k % kStages;
    uint8_t* kb = smem + st * L::STAGE;
    uint8_t* vb = kb + L::KT;
    mbar_arrive_expect_tx(&full[st], 2 * L::KT);
    const int tok = rg.start + k * kTok;
    for (int c = 0; c < L::CH; ++c) {
      tma_load_4d(&tm_k, &full[st], kb + c * L::BOX, c * 64, g, tok, b);
      tma_load_4d(&tm_v, &full[st], vb + c * L::BOX, c * 64, g, tok, b);
    }
  };
  if (tid == 0 && ntiles > 0) {
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    for (int k = 0; k < kStages && k < ntiles; ++k) issue(k);
  }

  // Query registers for the score phase: G heads x QW channels, pre-scaled
  // into the log2 domain.
  const int tj = tid >> 2, qd = tid & 3;
  float qr[G][QW];
  {
    const float sl2 = a.scale * 1.4426950408889634f;
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
      const uint4* src = reinterpret_cast<const uint4*>(
          a.q + (static_cast<size_t>(b) * a.Hq + g * G + hh) * D + qd * QW);
#pragma unroll
      for (int u = 0; u < QW / 8; ++u) {
        const uint4 w = src[u];
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          qr[hh][u * 8 + 2 * e] = bf16lo_to_f32(ws[e]) * sl2;
          qr[hh][u * 8 + 2 * e + 1] = bf16hi_to_f32(ws[e]) * sl2;
        }
      }
    }
  }

  float m_run[G], acc[G][8];
  float l_part = 0.f;
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
    m_run[hh] = -INFINITY;
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[hh][e] = 0.f;
  }
  const int vch = tid % NCH, vsub = tid / NCH;
  bool ok = true;
  int consumed = 0;

  for (int k = 0; k < ntiles; ++k) {
    const int st = k % kStages;
    if (!mbar_wait(&full[st], (k / kStages) & 1, a.st)) { ok = false; break; }
    const uint32_t kb = smem_u32(smem + st * L::STAGE);
    const uint32_t vb = kb + L::KT;
    const int tok0 = rg.start + k * kTok;

    // ---- scores: token tj, channel quarter qd
    float dot[G];
#pragma unroll
    for (int hh = 0; hh < G; ++hh) dot[hh] = 0.f;
#pragma unroll
    for (int u = 0; u < QW / 8; ++u) {
      const int unit = qd * (QW / 8) + u;         // 16-byte unit along the row (0 .. D/8-1)
      const int box = unit >> 3, uu = unit & 7;
      const uint4 w = ld_shared_v4(kb + box * L::BOX + tj * 128 + ((uu ^ (tj & 7)) << 4));
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float k0 = bf16lo_to_f32(ws[e]), k1 = bf16hi_to_f32(ws[e]);
#pragma unroll
        for (int hh = 0; hh < G; ++hh) {
          dot[hh] = fmaf(qr[hh][u * 8 + 2 * e], k0, dot[hh]);
          dot[hh] = fmaf(qr[hh][u * 8 + 2 * e + 1], k1, dot[hh]);
        }
      }
    }
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
      dot[hh] += __shfl_xor_sync(0xffffffffu, dot[hh], 1);
      dot[hh] += __shfl_xor_sync(0xffffffffu, dot[hh], 2);
    }
    const bool valid = (tok0 + tj < rg.end) && (qd < G);
    float sc = -INFINITY;
#pragma unroll
    for (int hh = 0; hh < G; ++hh)
      if (hh == qd && valid) sc = dot[hh];
    float mx = sc;
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
    if (lane < 4) red[warp * 4 + lane] = mx;
    __syncthreads();
    float alpha[G], m_use[G];
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
      float t = red[hh];
#pragma unroll
      for (int w = 1; w < 8; ++w) t = fmaxf(t, red[w * 4 + hh]);
      const float m_new = fmaxf(m_run[hh], t);
      m_use[hh] = (m_new == -INFINITY) ? 0.f : m_new;
      alpha[hh] = ex2(m_run[hh] - m_use[hh]);
      m_run[hh] = m_new;
    }
    float my_m = 0.f, my_alpha = 1.f;
#pragma unroll
    for (int hh = 0; hh < G; ++hh)
      if (hh == qd) { my_m = m_use[hh]; my_alpha = alpha[hh]; }
    const float p = valid ? ex2(sc - my_m) : 0.f;
    l_part = l_part * my_alpha + p;
    p_s[tj * 4 + qd] = p;
    __syncthreads();

    // ---- values: channels 8*vch .. +7, tokens vsub + NSUB*n
#pragma unroll
    for (int hh = 0; hh < G; ++hh)
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[hh][e] *= alpha[hh];
#pragma unroll
    for (int n = 0; n < TPS; ++n) {
      const int j = vsub + NSUB * n;
      const int box = vch >> 3, uu = vch & 7;
      const uint4 w = ld_shared_v4(vb + box * L::BOX + j * 128 + ((uu ^ (j & 7)) << 4));
      const float4 pj = *reinterpret_cast<const float4*>(p_s + j * 4);
      const float pv[4] = {pj.x, pj.y, pj.z, pj.w};
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float v0 = bf16lo_to_f32(ws[e]), v1 = bf16hi_to_f32(ws[e]);
#pragma unroll
        for (int hh = 0; hh < G; ++hh) {
          acc[hh][2 * e] = fmaf(pv[hh], v0, acc[hh][2 * e]);
          acc[hh][2 * e + 1] = fmaf(pv[hh], v1, acc[hh][2 * e + 1]);
        }
      }
    }
    __syncthreads();  // stage st and p_s are free again
    consumed = k + 1;
    if (tid == 0 && k + kStages < ntiles) issue(k + kStages);
  }
  if (!ok && tid == 0) {
    // Let the copies still in flight land before the CTA's smem goes away.
    DevStatus drain = a.st;
    drain.spin_ns = 100000000;
    const int last = min(ntiles, consumed + kStages);
    for (int k = consumed; k < last; ++k) mbar_wait(&full[k % kStages], (k / kStages) & 1, drain);
  }
  __syncthreads();

  // ---- combine within the CTA: l per head, acc over the NSUB token subsets
  float* comb = reinterpret_cast<float*>(smem);  // [NSUB][G][D], reuses the stage ring
  {
    float lp = l_part;
    lp += __shfl_xor_sync(0xffffffffu, lp, 4);
    lp += __shfl_xor_sync(0xffffffffu, lp, 8);
    lp += __shfl_xor_sync(0xffffffffu, lp, 16);
    if (lane < 4) red[warp * 4 + lane] = lp;
#pragma unroll
    for (int hh = 0; hh < G; ++hh)
#pragma unroll
      for (int e = 0; e < 8; ++e) comb[(vsub * G + hh) * D + vch * 8 + e] = acc[hh][e];
  }
  __syncthreads();
  const size_t grp = static_cast<size_t>(b) * a.Hq + g * G;  // first query head of the group
  if (rg.end > rg.start) {
    for (int idx = tid; idx < G * D; idx += kThreads) {
      const int hh = idx / D, c = idx % D;
      float t = 0.f;
      for (int sidx = 0; sidx < NSUB; ++sidx) t += comb[(sidx * G + hh) * D + c];
      a.part_o[((grp + hh) * a.nsplit + i) * D + c] = t;
    }
    if (tid < G) {
      float l = 0.f;
      for (int w = 0; w < 8; ++w) l += red[w * 4 + tid];
      a.part_ml[((grp + tid) * a.nsplit + i) * 2 + 0] = m_run[tid];
      a.part_ml[((grp + tid) * a.nsplit + i) * 2 + 1] = l;
    }
  }

  // ---- ticket: the last CTA of this (sequence, kv head) merges
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const int old = atomicAdd(&a.tickets[b * a.Hkv + g], 1);
    *flag = (old == static_cast<int>(gridDim.x) - 1);
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

template <int D, int G>
cudaError_t launch_t(const CUtensorMap& tk, const CUtensorMap& tv, const DecodeLaunch& p,
                     cudaStream_t stream) {
  const int smem = DSmem<D>::ALLOC;
  cudaFuncSetAttribute(decode_kernel<D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  const dim3 grid(p.nsplit, p.Hkv, p.B);
  decode_kernel<D, G><<<grid, kThreads, smem, stream>>>(tk, tv, p);
  return cudaGetLastError();
}

}  // namespace

void decode_plan(int B, int Hkv, int S_max, int sink_blocks, int window_blocks, int block,
                 int num_sms, int* nsplit, int* chunk_fa, int* chunk_sa) {
  // FA: chunks of about 2048 tokens (1 MiB of K+V per CTA at d=128), but at
  // least ~4 CTAs per SM in total; never below one 64-token tile.
  const long long groups = static_cast<long long>(B) * Hkv;
  int ns = (S_max + 2047) / 2048;
  const int want = static_cast<int>((4LL * num_sms + groups - 1) / groups);
  if (ns < want) ns = want;
  const int max_ns = (S_max + kTok - 1) / kTok;
  if (ns > max_ns) ns = max_ns;
  if (ns < 1) ns = 1;
  int cfa = (S_max + ns - 1) / ns;
  cfa = ((cfa + kTok - 1) / kTok) * kTok;
  // SA: the sink + window tokens, in chunks of at least one tile, spread over
  // about 8 splits.
  const long long sa_tokens = static_cast<long long>(sink_blocks + window_blocks) * block;
  long long csa = (sa_tokens + 7) / 8;
  csa = ((csa + kTok - 1) / kTok) * kTok;
  if (csa < kTok) csa = kTok;
  if (csa < cfa / 64) csa = ((cfa / 64 + kTok - 1) / kTok) * kTok;
  // The split count must cover both modes for any seqlen <= S_max.
  const long long need_sa = (static_cast<long long>(sink_blocks) * block + csa - 1) / csa +
                            (static_cast<long long>(window_blocks) * block + csa - 1) / csa;
  ns = static_cast<int>(std::max<long long>(ns, need_sa));
  cfa = (S_max + ns - 1) / ns;
  cfa = ((cfa + kTok - 1) / kTok) * kTok;
  if (cfa < kTok) cfa = kTok;
  *nsplit = ns;
  *chunk_fa = cfa;
  *chunk_sa = static_cast<int>(csa);
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
  const int G = p.Hq / p.Hkv;
  if (p.d == 64) {
    if (G == 1) return launch_t<64, 1>(tk, tv, p, stream);
    if (G == 2) return launch_t<64, 2>(tk, tv, p, stream);
    return launch_t<64, 4>(tk, tv, p, stream);
  }
  if (G == 1) return launch_t<128, 1>(tk, tv, p, stream);
  if (G == 2) return launch_t<128, 2>(tk, tv, p, stream);
  return launch_t<128, 4>(tk, tv, p, stream);
}

}  // namespace flux
