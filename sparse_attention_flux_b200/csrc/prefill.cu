// prefill.cu -- FA / SA prefill attention for one layer on sm_100a.
//
// Flux Attention routes each layer to Full Attention (exact causal softmax
// attention) or to block-sparse Sparse Attention (arXiv abstract; model card
// "Flux Attention: Qwen3-4B", "Sample Usage").  One kernel serves both: a
// CTA owns one 128-row query tile of one (batch, query head) and walks a list
// of 128-column key tiles -- every tile up to the diagonal for FA, the tiles
// named by the compressed block-index list for SA -- so skipped blocks are
// never loaded.
//
// Per CTA (192 threads, warp-specialised):
//   warp 0      TMA producer: Q once, then K/V tiles into a 2-stage ring.
//   warp 1      TMEM owner and UMMA issuer: S = Q K^T into TMEM (fp32), then
//               O += P V into TMEM, tcgen05.commit onto mbarriers.
//   warps 2..5  softmax: one query row per thread (= one TMEM lane), online
//               softmax in the log2 domain, P written to shared memory as
//               bf16 in the 128-byte-swizzled K-major layout UMMA reads,
//               lazy O rescale, and the epilogue O / l -> bf16.
// The S MMA of tile j+1 overlaps the exponentials of tile j.
#include "common.cuh"
#include "kernels.h"

namespace flux {

namespace {

constexpr int kBM = 128;            // query rows per CTA (TMEM lanes)
constexpr int kBN = 128;            // key columns per tile
constexpr int kChunkBytes = 128 * 128;  // 128 rows x 64 bf16 (one swizzle-128B box)
constexpr int kThreads = 192;

struct PrefillArgs {
  int B, T, Hq, Hkv, G;
  int nqt;           // number of 128-row tiles along T
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
  DevStatus st;
};

// The sequence of key tiles a query tile visits, identical in every role.
// sub-mask bit (r * 2 + c): query half r (rows 64r..64r+63) may see key half
// c (columns 64c..64c+63); only a 64-token mask block makes it partial.
struct TileIter {
  int fa, I, m;      // m = block / 128 (>= 1), or 0 for block == 64
  int J;             // FA cursor
  int p0, e0, p1, e1, sub;
  const int32_t* col;
  int nkb;
  int* err;

  __device__ void init(const PrefillArgs& a, int qt, bool is_fa) {
    fa = is_fa;
    I = qt;
    J = 0;
    sub = 0;
    col = a.col;
    nkb = a.nkb;
    err = a.st.err;
    p0 = e0 = p1 = e1 = 0;
    m = a.block >= 128 ? a.block / 128 : 0;
    if (fa) return;
    const int nnz = a.row_ptr[a.nqb];
    auto row = [&](int qb, int& p, int& e) {
      p = e = 0;
      if (qb >= a.nqb) return;
      int lo = a.row_ptr[qb], hi = a.row_ptr[qb + 1];
      if (lo < 0 || hi < lo || hi > nnz) {
        raise_error(err, DEV_ERR_CSR);
        return;
      }
      p = lo;
      e = hi;
    };
    if (m >= 1) {
      row(qt / m, p0, e0);
    } else {
      row(2 * qt, p0, e0);
      row(2 * qt + 1, p1, e1);
    }
  }

  __device__ int entry(int p) {
    int j = col[p];
    if (j < 0 || j >= nkb) {
      raise_error(err, DEV_ERR_CSR);
      return -1;
    }
    return j;
  }

  __device__ bool next(int& Jo, uint32_t& sm) {
    if (fa) {
      if (J > I) return false;
      Jo = J++;
      sm = 0xFu;
      return true;
    }
    if (m >= 1) {
      while (p0 < e0) {
        int j = entry(p0);
        if (j < 0) { ++p0; sub = 0; continue; }
        int t = j * m + sub;
        if (t > I) { p0 = e0; return false; }   // ascending list: nothing further is causal
        if (++sub == m) { sub = 0; ++p0; }
        Jo = t;
        sm = 0xFu;
        return true;
      }
      return false;
    }
    // block == 64: merge the lists of query blocks 2I and 2I+1 by key tile j/2.
    for (;;) {
      int j0 = -1, j1 = -1;
      while (p0 < e0 && (j0 = entry(p0)) < 0) ++p0;
      while (p1 < e1 && (j1 = entry(p1)) < 0) ++p1;
      if (p0 >= e0) j0 = -1;
      if (p1 >= e1) j1 = -1;
      if (j0 < 0 && j1 < 0) return false;
      int t0 = j0 >= 0 ? (j0 >> 1) : 0x7fffffff;
      int t1 = j1 >= 0 ? (j1 >> 1) : 0x7fffffff;
      int t = t0 < t1 ? t0 : t1;
      if (t > I) { p0 = e0; p1 = e1; return false; }
      uint32_t bits = 0;
      while (p0 < e0) {
        int j = entry(p0);
        if (j >= 0 && (j >> 1) != t) break;
        if (j >= 0) bits |= 1u << (0 * 2 + (j & 1));
        ++p0;
      }
      while (p1 < e1) {
        int j = entry(p1);
        if (j >= 0 && (j >> 1) != t) break;
        if (j >= 0) bits |= 1u << (1 * 2 + (j & 1));
        ++p1;
      }
      if (bits == 0) continue;
      Jo = t;
      sm = bits;
      return true;
    }
  }
};

// Bars: 0 q_full | 1,2 k_full | 3,4 v_full | 5,6 kv_empty | 7 s_full | 8 s_free
//       9 p_full | 10 o_done | 11 drain
enum { B_Q = 0, B_KF = 1, B_VF = 3, B_KE = 5, B_SF = 7, B_SFREE = 8, B_PF = 9, B_OD = 10,
       B_DRAIN = 11, B_COUNT = 12 };

template <int D>
struct Smem {
  static constexpr int CH = D / 64;
  static constexpr int Q = 0;
  static constexpr int K = Q + CH * kChunkBytes;
  static constexpr int V = K + 2 * CH * kChunkBytes;
  static constexpr int P = V + 2 * CH * kChunkBytes;
  static constexpr int BARS = P + 2 * kChunkBytes;
  static constexpr int TMEM_SLOT = BARS + B_COUNT * 8;
  static constexpr int TOTAL = TMEM_SLOT + 16;
  static constexpr int ALLOC = TOTAL + 1024;  // room to align the base to 1024
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tm_q,
                   const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const PrefillArgs a) {
  using L = Smem<D>;
  constexpr int CH = L::CH;
  constexpr uint32_t kTmemCols = 256;  // S: 128 columns, O: D columns
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem + L::Q;
  uint8_t* sK = smem + L::K;
  uint8_t* sV = smem + L::V;
  uint8_t* sP = smem + L::P;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::BARS);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::TMEM_SLOT);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Longest-first order: the last query tiles carry the most causal work.
  const int per_tile = a.Hq * a.B;
  const int qt = a.nqt - 1 - static_cast<int>(blockIdx.x) / per_tile;
  const int rem = static_cast<int>(blockIdx.x) % per_tile;
  const int b = rem / a.Hq, h = rem % a.Hq, g = h / a.G;
  const bool fa = a.layer_mode == nullptr || a.layer_mode[a.layer] != 0;

  TileIter it_count;
  it_count.init(a, qt, fa);
  int n = 0;
  {
    int J;
    uint32_t sm;
    while (it_count.next(J, sm)) ++n;
  }

  if (threadIdx.x == 0) {
    mbar_init(&bars[B_Q], 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars[B_KF + s], 1);
      mbar_init(&bars[B_VF + s], 1);
      mbar_init(&bars[B_KE + s], 1);
    }
    mbar_init(&bars[B_SF], 1);
    mbar_init(&bars[B_SFREE], 128);
    mbar_init(&bars[B_PF], 128);
    mbar_init(&bars[B_OD], 1);
    mbar_init(&bars[B_DRAIN], 1);
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem;         // columns [0, 128)
  const uint32_t tO = tmem + 128;   // columns [128, 128 + D)

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && n > 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      mbar_arrive_expect_tx(&bars[B_Q], CH * kChunkBytes);
      for (int c = 0; c < CH; ++c)
        tma_load_4d(&tm_q, &bars[B_Q], sQ + c * kChunkBytes, c * 64, h, qt * kBM, b);
      TileIter iter;
      iter.init(a, qt, fa);
      int J;
      uint32_t sm;
      int issued = 0;
      bool ok = true;
      for (int it = 0; it < n && iter.next(J, sm); ++it) {
        const int s = it & 1;
        if (it >= 2 && !mbar_wait(&bars[B_KE + s], ((it >> 1) - 1) & 1, a.st)) { ok = false; break; }
        mbar_arrive_expect_tx(&bars[B_KF + s], CH * kChunkBytes);
        for (int c = 0; c < CH; ++c)
          tma_load_4d(&tm_k, &bars[B_KF + s], sK + (s * CH + c) * kChunkBytes, c * 64, g,
                      J * kBN, b);
        mbar_arrive_expect_tx(&bars[B_VF + s], CH * kChunkBytes);
        for (int c = 0; c < CH; ++c)
          tma_load_4d(&tm_v, &bars[B_VF + s], sV + (s * CH + c) * kChunkBytes, c * 64, g,
                      J * kBN, b);
        issued = it + 1;
      }
      if (!ok) {
        // Let the copies already issued land before the CTA's smem goes away.
        DevStatus drain = a.st;
        drain.spin_ns = 100000000;  // 100 ms
        for (int it = issued - 2 < 0 ? 0 : issued - 2; it < issued; ++it) {
          mbar_wait(&bars[B_KF + (it & 1)], (it >> 1) & 1, drain);
          mbar_wait(&bars[B_VF + (it & 1)], (it >> 1) & 1, drain);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && n > 0) {
      constexpr uint32_t idesc_s = umma_idesc_bf16(kBM, kBN, false, false);
      constexpr uint32_t idesc_o = umma_idesc_bf16(kBM, D, false, true);
      const uint32_t q_addr = smem_u32(sQ), k_addr = smem_u32(sK), v_addr = smem_u32(sV);
      const uint32_t p_addr = smem_u32(sP);
      bool ok = mbar_wait(&bars[B_Q], 0, a.st);
      for (int it = 0; ok && it <= n; ++it) {
        if (it < n) {
          const int s = it & 1;
          if (!mbar_wait(&bars[B_KF + s], (it >> 1) & 1, a.st)) { ok = false; break; }
          if (it >= 1 && !mbar_wait(&bars[B_SFREE], (it - 1) & 1, a.st)) { ok = false; break; }
          tc_fence_after();
          const uint32_t kb = k_addr + s * CH * kChunkBytes;
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const uint32_t off = (ks >> 2) * kChunkBytes + (ks & 3) * 32;
            umma_bf16_ss(tS, umma_smem_desc(q_addr + off, 16, 1024, kSwizzle128B),
                         umma_smem_desc(kb + off, 16, 1024, kSwizzle128B), idesc_s, ks > 0);
          }
          umma_commit(&bars[B_SF]);
        }
        if (it >= 1) {
          const int j = it - 1, sj = j & 1;
          if (!mbar_wait(&bars[B_PF], j & 1, a.st)) { ok = false; break; }
          if (!mbar_wait(&bars[B_VF + sj], (j >> 1) & 1, a.st)) { ok = false; break; }
          tc_fence_after();
          const uint32_t vb = v_addr + sj * CH * kChunkBytes;
#pragma unroll
          for (int ks = 0; ks < kBN / 16; ++ks) {
            const uint32_t poff = (ks >> 2) * kChunkBytes + (ks & 3) * 32;
            umma_bf16_ss(tO, umma_smem_desc(p_addr + poff, 16, 1024, kSwizzle128B),
                         umma_smem_desc(vb + ks * 16 * 128, kChunkBytes, 1024, kSwizzle128B),
                         idesc_o, (j > 0 || ks > 0) ? 1u : 0u);
          }
          umma_commit(&bars[B_OD]);
          umma_commit(&bars[B_KE + sj]);
        }
      }
      // Every MMA issued by this thread is complete before TMEM is released.
      umma_commit(&bars[B_DRAIN]);
      DevStatus drain = a.st;
      drain.spin_ns = 100000000;
      mbar_wait(&bars[B_DRAIN], 0, drain);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int quarter = warp & 3;            // TMEM lanes 32*quarter .. +31
    const int r = quarter * 32 + lane;       // row within the tile
    const int t_row = qt * kBM + r;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t p_addr = smem_u32(sP);
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    TileIter iter;
    iter.init(a, qt, fa);
    int J;
    uint32_t sm;
    for (int it = 0; it < n && iter.next(J, sm); ++it) {
      if (!mbar_wait(&bars[B_SF], it & 1, a.st)) { ok = false; break; }
      tc_fence_after();
      float x[kBN];
#pragma unroll
      for (int c = 0; c < kBN / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tS + lane_off + c * 32, v);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) x[c * 32 + e] = __uint_as_float(v[e]) * a.scale_log2;
      }
      tc_fence_before();
      mbar_arrive(&bars[B_SFREE]);

      const bool diag = (J == qt);
      if (diag || sm != 0xFu) {
        const int qhalf = r >> 6;
#pragma unroll
        for (int c = 0; c < kBN; ++c) {
          const bool causal_ok = !diag || (J * kBN + c <= t_row);
          const bool blk_ok = (sm >> (qhalf * 2 + (c >> 6))) & 1u;
          if (!(causal_ok && blk_ok)) x[c] = -INFINITY;
        }
      }
      float mt = x[0];
#pragma unroll
      for (int c = 1; c < kBN; ++c) mt = fmaxf(mt, x[c]);
      const float m_new = fmaxf(m_run, mt);
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      const float alpha = ex2(m_run - m_use);
      float rs = 0.f;
#pragma unroll
      for (int c = 0; c < kBN; ++c) {
        x[c] = ex2(x[c] - m_use);
        rs += x[c];
      }
      l_run = l_run * alpha + rs;
      m_run = m_new;

      if (it >= 1 && !mbar_wait(&bars[B_OD], (it - 1) & 1, a.st)) { ok = false; break; }
      // P row -> shared memory, bf16, 128-byte swizzle (16-byte unit u ^ (row & 7)).
#pragma unroll
      for (int u = 0; u < kBN / 8; ++u) {
        const uint32_t w0 = pack_bf16x2(x[u * 8 + 0], x[u * 8 + 1]);
        const uint32_t w1 = pack_bf16x2(x[u * 8 + 2], x[u * 8 + 3]);
        const uint32_t w2 = pack_bf16x2(x[u * 8 + 4], x[u * 8 + 5]);
        const uint32_t w3 = pack_bf16x2(x[u * 8 + 6], x[u * 8 + 7]);
        const uint32_t addr = p_addr + (u >> 3) * kChunkBytes + r * 128 +
                              ((((u & 7) ^ (r & 7))) << 4);
        st_shared_v4(addr, w0, w1, w2, w3);
      }
      fence_proxy_async_smem();
      if (it >= 1) {
        tc_fence_after();
        if (!__all_sync(0xffffffffu, alpha == 1.f)) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t v[32];
            tmem_ld32(tO + lane_off + c * 32, v);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
            tmem_st32(tO + lane_off + c * 32, v);
          }
          tmem_wait_st();
        }
      }
      tc_fence_before();
      mbar_arrive(&bars[B_PF]);
    }

    // ------------------------------------------------------------ epilogue
    const size_t row_elem = ((static_cast<size_t>(b) * a.T + t_row) * a.Hq + h) * D;
    const bool valid = t_row < a.T;
    if (n > 0 && ok && mbar_wait(&bars[B_OD], (n - 1) & 1, a.st)) {
      tc_fence_after();
      const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tO + lane_off + c * 32, v);
        tmem_wait_ld();
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(a.o + row_elem + c * 32);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(v[u * 8 + 0]) * inv, __uint_as_float(v[u * 8 + 1]) * inv);
            w.y = pack_bf16x2(__uint_as_float(v[u * 8 + 2]) * inv, __uint_as_float(v[u * 8 + 3]) * inv);
            w.z = pack_bf16x2(__uint_as_float(v[u * 8 + 4]) * inv, __uint_as_float(v[u * 8 + 5]) * inv);
            w.w = pack_bf16x2(__uint_as_float(v[u * 8 + 6]) * inv, __uint_as_float(v[u * 8 + 7]) * inv);
            dst[u] = w;
          }
        }
      }
      if (valid && a.lse) {
        a.lse[(static_cast<size_t>(b) * a.Hq + h) * a.T + t_row] =
            l_run > 0.f ? (m_run + __log2f(l_run)) * 0.69314718055994531f : -INFINITY;
      }
    } else if (valid) {
      // No visible key (or an aborted tile): the row's output is zero.
      uint4* dst = reinterpret_cast<uint4*>(a.o + row_elem);
      for (int u = 0; u < D / 8; ++u) dst[u] = make_uint4(0, 0, 0, 0);
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
                           const PrefillLaunch& p, cudaStream_t stream) {
  PrefillArgs a;
  a.B = p.B;
  a.T = p.T;
  a.Hq = p.Hq;
  a.Hkv = p.Hkv;
  a.G = p.Hq / p.Hkv;
  a.nqt = (p.T + kBM - 1) / kBM;
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
  a.st = p.st;
  const dim3 grid(static_cast<unsigned>(a.nqt) * p.Hq * p.B);
  if (p.d == 64) {
    const int smem = Smem<64>::ALLOC;
    cudaFuncSetAttribute(prefill_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    prefill_kernel<64><<<grid, kThreads, smem, stream>>>(tq, tk, tv, a);
  } else {
    const int smem = Smem<128>::ALLOC;
    cudaFuncSetAttribute(prefill_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    prefill_kernel<128><<<grid, kThreads, smem, stream>>>(tq, tk, tv, a);
  }
  return cudaGetLastError();
}

}  // namespace flux
