// kernels.h -- internal launcher interfaces between the C ABI (api.cu) and
// the kernel translation units.  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "common.cuh"

namespace flux {

// A routed (block-index) prefill keeps its key-tile list in shared memory:
// at most this many 128-column key tiles, i.e. T <= 262144.
constexpr int kPrefillMaxKvTiles = 2048;

// Decode serves a kv head's whole query group from one read of its keys: the
// group fills rows of a 16-row warp-MMA operand, at most this many query heads.
constexpr int kDecodeMaxGroup = 8;

struct PrefillLaunch {
  int B, T, Hq, Hkv, d;
  int block, nqb;
  float scale;
  const uint8_t* layer_mode;
  int layer;
  const int32_t* row_ptr;
  const int32_t* col;
  uint16_t* o;
  float* lse;
  int force_mode;            // -1: layer_mode decides; 0: SA; 1: FA
  const uint8_t* head_mode;  // per-query-head routing [Hq], overrides layer_mode
  const float* blend_score;  // non-null: o = r * o + (1 - r) * this pass, r = blend_score[layer]
  DevStatus st;
};
int prefill_smem_bytes(int d);
cudaError_t launch_prefill(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                           const CUtensorMap& to, const PrefillLaunch& p, cudaStream_t stream);

struct DecodeLaunch {
  int B, Hq, Hkv, d, S_max;
  const uint16_t* q;
  const int32_t* seqlens;
  uint16_t* o;
  float* lse;
  const uint8_t* layer_mode;
  int layer;
  int sink_blocks, window_blocks, block;
  float scale;
  int nsplit, chunk_fa, tiles_sa;   // FA tokens per split; SA 64-token tiles per split
  int compact;      // SA over the compact ring cache (sink + window blocks), S_max = ring rows
  const uint8_t* head_mode;  // per-query-head routing [Hq] (overrides layer_mode), or null
  float* part_o;    // [B, Hq, nsplit, d]
  float* part_ml;   // [B, Hq, nsplit, 2]
  int* tickets;     // [B, Hkv], zero between calls
  DevStatus st;
  // Fused append (null = none): the new token's K/V rows k_new/v_new [B, Hkv, d]
  // are written into k_cache/v_cache (the tensors behind the maps) at token
  // seqlens[b] - 1 -- its ring slot when compact -- by the CTA that reads it.
  const uint16_t* k_new = nullptr;
  const uint16_t* v_new = nullptr;
  uint16_t* k_cache = nullptr;
  uint16_t* v_cache = nullptr;
};
// Split plan for a shape (host only): number of splits and chunk lengths.
void decode_plan(int B, int Hkv, int S_max, int sink_blocks, int window_blocks, int block,
                 int num_sms, int* nsplit, int* chunk_fa, int* tiles_sa);
// Active splits of an SA-only (compact ring) launch: its grid needs no FA splits.
int decode_sa_splits(int sink_blocks, int window_blocks, int block, int tiles_sa);
size_t decode_workspace_bytes(int B, int Hq, int Hkv, int d, int nsplit);
cudaError_t launch_decode(const CUtensorMap& tk, const CUtensorMap& tv, const DecodeLaunch& p,
                          cudaStream_t stream);

struct RouteLaunch {
  const uint16_t* hidden;
  int T, Hd, n_pool;
  const float* W1;
  const float* b1;
  int H1;
  const float* W2;
  const float* b2;
  int L;
  float thresh;
  uint8_t* layer_mode;
  float* score;
  float* pooled;   // workspace [2 Hd]
  float* hidden1;  // workspace [H1]
  int* ticket;     // workspace, zero between calls
};
size_t route_hidden1_offset(int Hd);   // in floats from pooled
size_t route_workspace_bytes(int Hd, int H1);
cudaError_t launch_route(const RouteLaunch& p, cudaStream_t stream);

// Dynamic SA block selection (strided antidiagonal scores, threshold selection).
constexpr int kSelectMaxBlocks = 1024;   // query / key blocks of 128 tokens: T <= 131072
struct BlockSelectLaunch {
  int B, T, Hq, Hkv, d;
  int stride;                // 8 (block 128)
  float scale, tau;
  int sink_blocks;
  uint8_t* block_mask;       // [nb][nb] out
  float* block_score;        // [nb][nb] out, optional
  float* workspace;          // block_select_workspace_bytes()
  DevStatus st;
};
size_t block_select_workspace_bytes(int B, int T, int Hq, int Hkv, int stride);
cudaError_t launch_block_select(const CUtensorMap& tq, const CUtensorMap& tk,
                                const BlockSelectLaunch& p, cudaStream_t stream);

cudaError_t launch_ring_write(const uint16_t* k_src, const uint16_t* v_src, int n,
                              const int32_t* seqlens, int B, int Hkv, int d, uint16_t* k_ring,
                              uint16_t* v_ring, int sink, int window, int block, int* err,
                              cudaStream_t stream);

// One thread waits on an mbarrier that is never arrived at (bounded wait test).
cudaError_t launch_selftest_wait(DevStatus st, int* waited_us, cudaStream_t stream);

cudaError_t launch_streaming_mask(int nqb, int nkb, int sink, int window, uint8_t* mask,
                                  cudaStream_t stream);
cudaError_t launch_block_index(const uint8_t* mask, int nqb, int nkb, int32_t* row_ptr,
                               int32_t* col, int cap, int32_t* counts, int* err,
                               cudaStream_t stream);

}  // namespace flux
