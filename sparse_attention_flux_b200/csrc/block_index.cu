// block_index.cu -- the SA block mask and its compressed block-index list.
//
// SA layers run block-sparse attention (model card "Flux Attention:
// Qwen3-4B", "Sample Usage") over attention sinks plus a window of recent
// blocks (SA keeps only the minimal KV: gist.science summary, section 2).
// The prefill kernel walks the CSR form so that skipped blocks are never
// loaded.  Everything here is integer work and bit-exact:
//   mask_kernel    mask[i][j] = (j <= i) && (j < sink || j >= i - W + 1)
//   count_kernel   one CTA per q-block row: number of kept blocks
//   scan_kernel    one CTA: exclusive scan of the counts -> row_ptr, nnz,
//                  capacity check
//   fill_kernel    one CTA per row: order-preserving compaction into col[]
#include "common.cuh"
#include "kernels.h"

namespace flux {

namespace {

constexpr int kT = 256;

__global__ void mask_kernel(int nqb, int nkb, int sink, int window, uint8_t* __restrict__ mask) {
  const size_t total = static_cast<size_t>(nqb) * nkb;
  for (size_t idx = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int i = static_cast<int>(idx / nkb), j = static_cast<int>(idx % nkb);
    mask[idx] = static_cast<uint8_t>((j <= i) && (j < sink || j >= i - window + 1));
  }
}

__global__ void __launch_bounds__(kT)
    count_kernel(const uint8_t* __restrict__ mask, int nkb, int32_t* __restrict__ counts) {
  const uint8_t* row = mask + static_cast<size_t>(blockIdx.x) * nkb;
  int c = 0;
  for (int j = threadIdx.x; j < nkb; j += kT) c += row[j] != 0;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
  __shared__ int ws[kT / 32];
  if ((threadIdx.x & 31) == 0) ws[threadIdx.x >> 5] = c;
  __syncthreads();
  if (threadIdx.x == 0) {
    int t = 0;
    for (int w = 0; w < kT / 32; ++w) t += ws[w];
    counts[blockIdx.x] = t;
  }
}

__global__ void __launch_bounds__(kT)
    scan_kernel(const int32_t* __restrict__ counts, int nqb, int32_t* __restrict__ row_ptr,
                int cap, int* err) {
  __shared__ int32_t carry;
  __shared__ int32_t wsum[kT / 32];
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int base = 0; base < nqb; base += kT) {
    const int i = base + threadIdx.x;
    const int32_t v = i < nqb ? counts[i] : 0;
    int32_t x = v;  // inclusive warp scan
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) wsum[warp] = x;
    __syncthreads();
    int32_t wofs = 0;
    for (int w = 0; w < warp; ++w) wofs += wsum[w];
    const int32_t excl = carry + wofs + x - v;
    if (i < nqb) row_ptr[i] = excl;
    __syncthreads();
    if (threadIdx.x == kT - 1) carry = excl + v;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    row_ptr[nqb] = carry;
    if (carry > cap) raise_error(err, DEV_ERR_CAPACITY);
  }
}

__global__ void __launch_bounds__(kT)
    fill_kernel(const uint8_t* __restrict__ mask, int nkb, const int32_t* __restrict__ row_ptr,
                int32_t* __restrict__ col, int cap) {
  __shared__ int32_t wsum[kT / 32];
  __shared__ int32_t carry;
  const uint8_t* row = mask + static_cast<size_t>(blockIdx.x) * nkb;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) carry = row_ptr[blockIdx.x];
  __syncthreads();
  for (int base = 0; base < nkb; base += kT) {
    const int j = base + threadIdx.x;
    const bool keep = j < nkb && row[j] != 0;
    const unsigned bal = __ballot_sync(0xffffffffu, keep);
    const int before = __popc(bal & ((1u << lane) - 1u));
    if (lane == 0) wsum[warp] = __popc(bal);
    __syncthreads();
    int32_t wofs = 0;
    for (int w = 0; w < warp; ++w) wofs += wsum[w];
    const int32_t pos = carry + wofs + before;
    if (keep && pos < cap) col[pos] = j;
    __syncthreads();
    if (threadIdx.x == 0) {
      int32_t t = 0;
      for (int w = 0; w < kT / 32; ++w) t += wsum[w];
      carry += t;
    }
    __syncthreads();
  }
}

}  // namespace

cudaError_t launch_streaming_mask(int nqb, int nkb, int sink, int window, uint8_t* mask,
                                  cudaStream_t stream) {
  const size_t total = static_cast<size_t>(nqb) * nkb;
  size_t blocks = (total + 255) / 256;
  if (blocks > 4096) blocks = 4096;
  mask_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(nqb, nkb, sink, window, mask);
  return cudaGetLastError();
}

cudaError_t launch_block_index(const uint8_t* mask, int nqb, int nkb, int32_t* row_ptr,
                               int32_t* col, int cap, int32_t* counts, int* err,
                               cudaStream_t stream) {
  count_kernel<<<nqb, kT, 0, stream>>>(mask, nkb, counts);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  scan_kernel<<<1, kT, 0, stream>>>(counts, nqb, row_ptr, cap, err);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  fill_kernel<<<nqb, kT, 0, stream>>>(mask, nkb, row_ptr, col, cap);
  return cudaGetLastError();
}

}  // namespace flux
