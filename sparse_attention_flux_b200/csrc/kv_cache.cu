// kv_cache.cu -- the compact KV cache of SA layers.
//
// SA layers keep only the minimal KV cache -- the attention-sink blocks and
// the most recent W blocks -- and never read the history between (gist.science
// summary "Flux Attention", section 2, "efficient deployment").  Layout per
// (sequence, kv head): rows [0, sink*block) hold the sink tokens; block j >=
// sink lives in ring slot j mod W at rows [(sink + j mod W) * block, ...).
// The live window blocks ceil(s/block) - W .. ceil(s/block) - 1 always have
// distinct slots, and a new block overwrites exactly the block that has just
// left the window.
//
// ring_write_kernel copies the tokens at positions [s - n, s) (s = seqlens[b]
// after the write) of a [B, n, Hkv, d] source into the ring -- the whole
// prompt after prefill (n = T), or one new token per decode step (n = 1).
// Only tokens that are still live at length s are written, so no two threads
// write the same ring row.  With window == 0 it writes a full cache instead
// (row = position; `block` is then the cache capacity): the FA layers' append.
// 16 bytes per thread, coalesced along (head, d).
#include "common.cuh"
#include "kernels.h"

namespace flux {

namespace {

__global__ void ring_write_kernel(const uint4* __restrict__ k_src, const uint4* __restrict__ v_src,
                                  int n, const int32_t* __restrict__ seqlens, int Hkv, int d,
                                  uint4* __restrict__ k_ring, uint4* __restrict__ v_ring,
                                  int sink, int window, int block, int* err) {
  const int b = blockIdx.y;
  const int vec_per_tok = Hkv * d / 8;
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<long long>(n) * vec_per_tok) return;
  const int i = static_cast<int>(idx / vec_per_tok), e = static_cast<int>(idx % vec_per_tok);
  const int s = seqlens[b];
  if (s < n) {
    if (idx == 0) raise_error(err, DEV_ERR_SEQLEN);
    return;
  }
  const int u = s - n + i;                 // token position
  int row;
  if (window == 0) {
    // Full cache: row = position, capacity `block` rows.
    if (s > block) {
      if (idx == 0) raise_error(err, DEV_ERR_SEQLEN);
      return;
    }
    row = u;
  } else {
    const int j = u / block;
    const int nbs = (s + block - 1) / block;
    if (j < sink) {
      row = u;
    } else if (j >= nbs - window) {
      row = (sink + j % window) * block + u % block;
    } else {
      return;                              // already outside the window at length s
    }
  }
  const int ring_rows = window == 0 ? block : (sink + window) * block;
  const size_t src = (static_cast<size_t>(b) * n + i) * vec_per_tok + e;
  const size_t dst = (static_cast<size_t>(b) * ring_rows + row) * vec_per_tok + e;
  k_ring[dst] = k_src[src];
  v_ring[dst] = v_src[src];
}

}  // namespace

cudaError_t launch_ring_write(const uint16_t* k_src, const uint16_t* v_src, int n,
                              const int32_t* seqlens, int B, int Hkv, int d, uint16_t* k_ring,
                              uint16_t* v_ring, int sink, int window, int block, int* err,
                              cudaStream_t stream) {
  const long long total = static_cast<long long>(n) * Hkv * d / 8;
  const dim3 grid(static_cast<unsigned>((total + 255) / 256), B);
  ring_write_kernel<<<grid, 256, 0, stream>>>(
      reinterpret_cast<const uint4*>(k_src), reinterpret_cast<const uint4*>(v_src), n, seqlens,
      Hkv, d, reinterpret_cast<uint4*>(k_ring), reinterpret_cast<uint4*>(v_ring), sink, window,
      block, err);
  return cudaGetLastError();
}

}  // namespace flux
