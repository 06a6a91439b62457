/*
 * flux.h -- C ABI of the B200 (sm_100a) routed-attention library (libflux.so).
 *
 * Flux Attention ("Flux Attention: Context-Aware Hybrid Attention for
 * Efficient LLMs Inference", arXiv 2604.07394) puts a small Layer Router in
 * front of a frozen LLM.  The router looks at the prompt once, at prefill,
 * and sends every layer either to Full Attention (FA: exact causal softmax
 * attention) or to Sparse Attention (SA: block-sparse attention over a sink +
 * local-window block mask).  The decision is reused for every decode step,
 * and SA layers read only the minimal KV.  This header exposes that hot path:
 *
 *   flux_route                 pool + MLP + hard threshold  -> layer_mode[L]
 *   flux_build_streaming_mask  sink + window block mask     -> mask[nqb][nkb]
 *   flux_select_blocks         dynamic block mask from Q, K -> mask[nb][nb]
 *   flux_build_block_index     block mask                   -> CSR row_ptr/col
 *   flux_attn_prefill          one layer, FA or SA per layer_mode[layer]
 *   flux_attn_prefill_soft     r FA + (1 - r) SA, the training-time soft routing
 *   flux_attn_decode           one layer, one new token per sequence
 *   flux_kv_write              append / fill a full cache or an SA layer's ring
 *   flux_attn_decode_sa_compact  SA decode over the ring (sink + last W blocks)
 *   flux_attn_decode_append    append the step's token + decode, one launch
 *
 * Conventions shared by every entry point
 *   - Every tensor pointer is a DEVICE pointer owned by the caller; the
 *     library never frees or keeps it beyond the call's stream work.
 *   - bf16 tensors are passed as uint16_t bit patterns (IEEE bfloat16).
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the
 *     legacy default stream) and returns an int status.  Host-side argument
 *     checks happen before any launch; on failure nothing is launched.
 *   - Stream order holds as usual.  The decode calls and the router's second
 *     kernel are launched with programmatic stream serialisation: their CTAs
 *     may be dispatched while the previous kernel on the stream finishes, but
 *     they read and write no memory until that kernel has completed and its
 *     writes are visible, so the caller sees ordinary stream semantics.
 *   - Device-side checks (seqlens beyond capacity, CSR entries out of range,
 *     a bounded wait that ran out) set the context's device error word and
 *     zero the affected outputs; flux_ctx_check() reports it.
 *   - The routing bit is read ON THE DEVICE (layer_mode[layer]; 1 = FA,
 *     0 = SA), so routing and attention chain on one stream with no host sync.
 *   - A flux_ctx owns the only memory the library allocates (a workspace for
 *     split-KV decode partials and router intermediates, and the error word).
 *     Calls that share a ctx must not overlap in time on different streams.
 *   - flux_last_error() describes the last failure of the calling thread.
 */
#ifndef FLUX_H
#define FLUX_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define FLUX_ABI_VERSION 1

/* Status codes. */
#define FLUX_OK                0
#define FLUX_ERR_INVALID_ARG  -1  /* null pointer, negative size, bad threshold ...        */
#define FLUX_ERR_SHAPE        -2  /* sizes inconsistent or beyond capacity / workspace      */
#define FLUX_ERR_UNSUPPORTED  -3  /* e.g. head_dim not 64/128, Hq % Hkv != 0, block size   */
#define FLUX_ERR_CUDA         -4  /* a CUDA runtime call failed (launch, memcpy, ...)       */
#define FLUX_ERR_TIMEOUT      -5  /* a bounded device-side wait ran out (device error word) */
#define FLUX_ERR_DEVICE_CHECK -6  /* a device-side range check failed (device error word)   */

typedef struct flux_ctx flux_ctx;
typedef void* flux_stream_t; /* cudaStream_t */

/* ABI version (FLUX_ABI_VERSION). */
int flux_version(void);

/* Message for the calling thread's last failed call ("" if none). */
const char* flux_last_error(void);

/* Create a context on CUDA device `device`, allocating `workspace_bytes` of
 * device workspace (0 = a default of 64 MiB) plus the device error word.
 * The workspace holds split-KV decode partials and router intermediates; use
 * flux_decode_workspace_bytes() to size it for a decode shape.  The ctx is
 * bound to `device`; calls through it must run with that device current. */
int flux_ctx_create(flux_ctx** ctx, int device, size_t workspace_bytes);

/* Free the context's device memory.  Pending work on any stream that used the
 * ctx must be complete. */
int flux_ctx_destroy(flux_ctx* ctx);

/* Synchronize `stream`, read and clear the device error word.  Returns
 * FLUX_OK, FLUX_ERR_TIMEOUT, FLUX_ERR_DEVICE_CHECK or FLUX_ERR_CUDA. */
int flux_ctx_check(flux_ctx* ctx, flux_stream_t stream);

/* Spin limit of every bounded device-side wait, in milliseconds (default
 * 2000).  A wait that runs out sets the error word and makes the kernel
 * release its resources and return. */
int flux_ctx_set_spin_limit_ms(flux_ctx* ctx, int ms);

/* Self-test of the failure path every pipeline kernel relies on: launches one
 * thread that waits on an mbarrier nothing ever arrives at, through the same
 * bounded wait (here limited to spin_limit_ms, 1..10000).  The wait gives up,
 * records the timeout in the device error word and the kernel returns; a
 * following flux_ctx_check returns FLUX_ERR_TIMEOUT and clears the word, and
 * the context stays usable.  waited_us (device int, optional) receives the
 * time the wait took, in microseconds.  No fault and no hang is involved. */
int flux_selftest_bounded_wait(flux_ctx* ctx, int spin_limit_ms, int* waited_us,
                               flux_stream_t stream);

/* --------------------------------------------------------------------------
 * Layer Router (gist.science summary "Flux Attention", section 2
 * "Methodology": "Layer Router" pools the first and last 100 prompt tokens
 * and runs a context-encoder MLP; "switch to hard routing" thresholds the
 * soft weight to 0/1 at inference; "efficient deployment" routes once, at
 * prefill).
 *   hidden     [T, Hd] bf16, row-major: the prompt's hidden states.
 *   n_pool     rows pooled on each side (100 on the pages); each side uses
 *              n = min(n_pool, T) rows, so the windows overlap when T < 2 n.
 *   p          = [mean(hidden[0:n]), mean(hidden[T-n:T])]      (2*Hd, fp32)
 *   W1 [H1, 2*Hd], b1 [H1], W2 [L, H1], b2 [L]: fp32, row-major.
 *   z          = W2 relu(W1 p + b1) + b2;  r = sigmoid(z)
 *   layer_mode [L] uint8 out: 1 (FA) iff r > thresh, else 0 (SA); a tie is SA.
 *   score      [L] fp32 out (optional, may be NULL): r.
 *   hidden, W1 and W2 start on 16-byte boundaries (they are read in 16-byte
 *   vectors); b1 and b2 need only fp32 alignment.
 * Uses 4 * (round_up(2*Hd, 4) + H1) + 64 bytes of the ctx workspace.
 * Errors: INVALID_ARG for null required pointers, sizes <= 0, thresh not
 * finite, hidden, W1 or W2 not 16-byte aligned; SHAPE if the workspace is
 * too small. */
int flux_route(flux_ctx* ctx, const uint16_t* hidden, int T, int Hd, int n_pool,
               const float* W1, const float* b1, int H1,
               const float* W2, const float* b2, int L,
               float thresh, uint8_t* layer_mode, float* score, flux_stream_t stream);

/* --------------------------------------------------------------------------
 * SA block mask: attention sinks plus a local window of recent blocks (the
 * block-sparse SA of the model card "Flux Attention: Qwen3-4B", "Sample
 * Usage"; SA keeps only the minimal KV, gist.science summary section 2).
 *   block_mask [nqb, nkb] uint8 out, row-major:
 *     mask[i][j] = (j <= i) && (j < sink_blocks || j >= i - window_blocks + 1)
 *   The window counts the diagonal block.  sink_blocks >= 0, window_blocks >= 1. */
int flux_build_streaming_mask(int nqb, int nkb, int sink_blocks, int window_blocks,
                              uint8_t* block_mask, flux_stream_t stream);

/* Dynamic SA block selection: a block mask chosen from the layer's own Q and
 * K.  The pages name a block-sparse selector for the SA side (the checkpoint
 * page's repository name "full_xattn_Qwen3-4B"; XAttention among the sparse
 * methods in the UniSparse abstract on the page list) but give no algorithm;
 * this call implements a stated reading of that family's published idea
 * (antidiagonal scores over strided positions, then the fewest blocks whose
 * score mass reaches tau).  Parity against the pages is therefore unpinned;
 * the definition below is the contract.  With S = stride, R = block / S,
 * nr = ceil(T / S) strided positions and nb = ceil(T / block) blocks:
 *   z[r][c]   = scale * sum_{k<S} q[rS+k] . key[cS+S-1-k] for c <= r < nr, per
 *               (sequence b, query head h, kv head h / (Hq/Hkv)); rows >= T
 *               read as zero;
 *   P_h[i][j] = sum of exp(z) over strided rows r in [iR, iR+R) and columns c
 *               in [jR, jR+R), c <= r, divided by that sum over all j <= i;
 *   P[i][j]   = mean over (b, h) of P_h[i][j]  (block_score, fp32);
 *   block_mask[i][j] = 1 for j < sink_blocks (j <= i) and j = i, and for the
 *               other j <= i taken by decreasing P (ties: smaller j first)
 *               while the fp32 sum of the kept blocks' P (forced blocks by
 *               ascending j, then in the order taken) is below tau.
 * One mask for the layer (all sequences and heads), the input of
 * flux_build_block_index and of an SA prefill with the same block.
 *   q [B, T, Hq, d], k [B, T, Hkv, d] bf16 in (16-byte aligned, contiguous).
 *   block_mask [nb, nb] uint8 out; block_score [nb, nb] fp32 out (optional,
 *   zero above the diagonal).
 * Supported: d 64 or 128, block 128, stride 8, T <= 131072.  Uses
 * flux_select_blocks_workspace_bytes() bytes of the ctx workspace (that query
 * returns 0 for a shape this call does not support).
 * Errors: INVALID_ARG (null pointers, scale not finite and positive, tau
 * negative or not finite, sink_blocks < 0, misaligned q/k), UNSUPPORTED
 * (d, block, stride, T, Hq % Hkv), SHAPE (sizes, workspace too small). */
size_t flux_select_blocks_workspace_bytes(int B, int T, int Hq, int Hkv, int stride);
int flux_select_blocks(flux_ctx* ctx, const uint16_t* q, const uint16_t* k, int B, int T,
                       int Hq, int Hkv, int d, int block, int stride, float scale, float tau,
                       int sink_blocks, uint8_t* block_mask, float* block_score,
                       flux_stream_t stream);

/* Compressed block-index list of a block mask (the form the prefill kernel
 * walks, so that skipped blocks cost no memory traffic).
 *   block_mask [nqb, nkb] uint8 in (nonzero = keep).
 *   row_ptr [nqb + 1] int32 out; row_ptr[nqb] = nnz.
 *   col [cap] int32 out: for each q-block i, the ascending kept kv blocks in
 *   col[row_ptr[i] .. row_ptr[i+1]).
 * If nnz > cap, nothing beyond cap is written and the device error word is
 * set (flux_ctx_check -> FLUX_ERR_DEVICE_CHECK).  Uses 4 * nqb bytes of the
 * ctx workspace. */
int flux_build_block_index(flux_ctx* ctx, const uint8_t* block_mask, int nqb, int nkb,
                           int32_t* row_ptr, int32_t* col, int cap, flux_stream_t stream);

/* --------------------------------------------------------------------------
 * Prefill attention for one layer (arXiv abstract: FA = exact causal full
 * attention; SA = sparse attention; routing is per layer).
 *   q [B, T, Hq, d], k and v [B, T, Hkv, d]: bf16, contiguous.
 *   o [B, T, Hq, d] bf16 out.  lse [B, Hq, T] fp32 out (optional): natural-log
 *   sum of exp of the scaled scores; -inf for a row with no visible key.
 *   Query head h reads kv head h / (Hq / Hkv).
 *   layer_mode: device uint8 array; layer_mode[layer] = 1 -> FA (every key
 *   u <= t), 0 -> SA (u <= t and the block pair (t / block, u / block) is in
 *   the CSR list).  layer_mode == NULL means FA.
 *   row_ptr/col: the CSR list from flux_build_block_index over nqb >=
 *   ceil(T / block) q-blocks; required unless layer_mode == NULL.  Each row's
 *   columns must be strictly ascending and < ceil(T / block), as
 *   flux_build_block_index writes them.  A row range or an entry out of range,
 *   or a row out of order, is a device-checked error (FLUX_ERR_DEVICE_CHECK from
 *   flux_ctx_check): the query rows whose key list reads that CSR row (that
 *   q-block's rows, up to the 256-row unit holding them) are written as zero,
 *   lse -inf.
 *   block: 64 or a multiple of 128.  d: 64 or 128.  With layer_mode given,
 *   T <= 262144 (the CTA's key-tile list lives in shared memory).  scale: score scale
 *   (1/sqrt(d) for the models on the pages).
 * Runs the tcgen05/TMEM/TMA flash-attention kernel; skipped blocks are never
 * loaded.  Errors: UNSUPPORTED for other d or block, or Hq % Hkv != 0; SHAPE
 * for T < 1, nqb too small, or sizes whose tensor maps cannot be encoded. */
int flux_attn_prefill(flux_ctx* ctx, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                      uint16_t* o, float* lse, int B, int T, int Hq, int Hkv, int d,
                      const uint8_t* layer_mode, int layer,
                      const int32_t* row_ptr, const int32_t* col, int nqb, int block,
                      float scale, flux_stream_t stream);

/* Soft-routing forward blend (gist.science summary section 2, "training
 * process": during training the continuous router weight r_soft combines the
 * two paths, o = r FA + (1 - r) SA).  Forward only: runs the FA pass into o,
 * then the SA pass (over the CSR list), whose epilogue reads that row of o and
 * writes r * o_FA + (1 - r) * o_SA with r = score[layer] read on the device
 * (the `score` output of flux_route).  Shapes, layouts and limits as
 * flux_attn_prefill; no lse.  r = 1 gives FA's output exactly, r = 0 SA's. */
int flux_attn_prefill_soft(flux_ctx* ctx, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                           uint16_t* o, int B, int T, int Hq, int Hkv, int d,
                           const float* score, int layer,
                           const int32_t* row_ptr, const int32_t* col, int nqb, int block,
                           float scale, flux_stream_t stream);

/* --------------------------------------------------------------------------
 * Decode attention for one layer and one new token per sequence (gist.science
 * summary section 2, "efficient deployment": the prefill routing bit is
 * reused; SA layers read only the sink blocks and the last W blocks).
 *   q [B, Hq, d] bf16: the query of the token at position seqlens[b] - 1.
 *   k_cache, v_cache [B, S_max, Hkv, d] bf16; the caller has already appended
 *   the new token's k/v, so positions 0 .. seqlens[b]-1 are valid.
 *   seqlens [B] int32 device array, 0 <= seqlens[b] <= S_max (checked on the
 *   device; a bad value zeroes that sequence's output and sets the error word).
 *   o [B, Hq, d] bf16 out; lse [B, Hq] fp32 out (optional).
 *   layer_mode[layer]: 1 -> FA over all u < s; 0 -> SA over the tokens in
 *   blocks j < sink_blocks or j >= ceil(s / block) - window_blocks.
 *   layer_mode == NULL means FA.
 * Split-KV: each CTA streams one chunk of one (sequence, kv head) and serves
 * all Hq/Hkv query heads of the group from that single read; the last CTA of
 * the group (atomic ticket, no spin) merges the partials.  Partials live in
 * the ctx workspace (flux_decode_workspace_bytes).  Supported: d 64/128,
 * Hq/Hkv a whole number from 1 to 8 (else UNSUPPORTED).  Calls sharing a ctx
 * must not overlap in time.  Consecutive decode calls on one stream (one per
 * layer) overlap each launch's dispatch with the previous one's tail. */
int flux_attn_decode(flux_ctx* ctx, const uint16_t* q, const uint16_t* k_cache,
                     const uint16_t* v_cache, int S_max, const int32_t* seqlens,
                     uint16_t* o, float* lse, int B, int Hq, int Hkv, int d,
                     const uint8_t* layer_mode, int layer,
                     int sink_blocks, int window_blocks, int block, float scale,
                     flux_stream_t stream);

/* --------------------------------------------------------------------------
 * KV-cache writes, and decode over the compact SA cache (gist.science summary
 * section 2, "efficient deployment": SA layers keep only the minimal KV cache
 * -- the sink blocks and the last W blocks -- and never read the history).
 *
 * flux_kv_write copies the tokens at positions [s - n_src, s) of each sequence
 * (s = seqlens[b], the length AFTER the write) from k_src/v_src
 * [B, n_src, Hkv, d] bf16 into a cache:
 *   window_blocks == 0: a full cache [B, cache_rows, Hkv, d]; row = position
 *     (an FA layer's per-step append, n_src = 1);
 *   window_blocks  > 0: the compact ring of an SA layer, [B, cache_rows, Hkv, d]
 *     with cache_rows = (sink_blocks + window_blocks) * block: rows
 *     [0, sink*block) hold the sink tokens, block j >= sink_blocks lives in
 *     slot j mod window_blocks at rows (sink_blocks + j mod W) * block + ...
 *     Only tokens still live at length s are written (so a whole prompt,
 *     n_src = T, fills the ring with its sink and last W blocks).
 * Hkv * d must be a multiple of 8.  A seqlens entry below n_src (or above
 * cache_rows for a full cache) skips that sequence and sets the error word.
 *
 * flux_attn_decode_sa_compact is flux_attn_decode for an SA layer whose cache
 * is that ring: the same tokens (blocks j < sink or j >= ceil(s/block) - W),
 * hence the same result as SA decode over the full cache, read from
 * (sink + W) * block rows per sequence.  block must be a multiple of 64;
 * seqlens[b] may exceed the ring size (it is the sequence length). */
int flux_kv_write(flux_ctx* ctx, const uint16_t* k_src, const uint16_t* v_src, int n_src,
                  const int32_t* seqlens, int B, int Hkv, int d,
                  uint16_t* k_cache, uint16_t* v_cache, int cache_rows,
                  int sink_blocks, int window_blocks, int block, flux_stream_t stream);

int flux_attn_decode_sa_compact(flux_ctx* ctx, const uint16_t* q, const uint16_t* k_ring,
                                const uint16_t* v_ring, const int32_t* seqlens,
                                uint16_t* o, float* lse, int B, int Hq, int Hkv, int d,
                                int sink_blocks, int window_blocks, int block, float scale,
                                flux_stream_t stream);

/* flux_attn_decode_append: one decode step of one layer with the step's KV
 * append fused in (same section of the gist.science summary: the new token's
 * K/V enters the layer's cache, then the query attends).  k_new/v_new
 * [B, Hkv, d] bf16 are the new token's rows; seqlens[b] = s counts it (the new
 * token is token s - 1).  The decode CTA whose split reads token s - 1 writes
 * the rows into the cache first, so the result equals flux_kv_write (n_src 1)
 * followed by the decode, in one launch:
 *   compact == 0: k_cache/v_cache is a full cache [B, cache_rows, Hkv, d]
 *     (cache_rows = S_max, s <= S_max), routed by layer_mode[layer] exactly as
 *     flux_attn_decode (layer_mode NULL = FA);
 *   compact == 1: it is an SA layer's ring, cache_rows = (sink_blocks +
 *     window_blocks) * block, block a multiple of 64, as
 *     flux_attn_decode_sa_compact; layer_mode is ignored.
 * A seqlens entry below 1 (no token to append) or above S_max for a full cache
 * is a device-checked error: nothing is written for that sequence and its
 * output is zero.  Other limits and the workspace as flux_attn_decode. */
int flux_attn_decode_append(flux_ctx* ctx, const uint16_t* q, const uint16_t* k_new,
                            const uint16_t* v_new, uint16_t* k_cache, uint16_t* v_cache,
                            int cache_rows, const int32_t* seqlens, uint16_t* o, float* lse,
                            int B, int Hq, int Hkv, int d, const uint8_t* layer_mode, int layer,
                            int sink_blocks, int window_blocks, int block, int compact,
                            float scale, flux_stream_t stream);

/* --------------------------------------------------------------------------
 * Per-head routing (the contrast case).  Flux Attention routes whole layers;
 * the head-level alternative it is compared with (Elastic Attention on the
 * same page list) routes each attention head, and the arXiv abstract states
 * that head-level dynamic sparsity causes load imbalance and synchronisation
 * long-tails in decoding.  These two calls make that measurable:
 *   head_mode [Hq] uint8 device array: 1 = FA, 0 = SA for query head h.
 * flux_attn_prefill_heads: as flux_attn_prefill, mode per query head.
 * flux_attn_decode_heads: as flux_attn_decode; the CTA serving a GQA group
 * streams the whole history if any head of the group is FA, and masks the
 * tokens outside the sink + window blocks for its SA heads -- so a mixed group
 * costs a full FA read.  Results equal per-head FA / SA attention. */
int flux_attn_prefill_heads(flux_ctx* ctx, const uint16_t* q, const uint16_t* k,
                            const uint16_t* v, uint16_t* o, float* lse, int B, int T,
                            int Hq, int Hkv, int d, const uint8_t* head_mode,
                            const int32_t* row_ptr, const int32_t* col, int nqb, int block,
                            float scale, flux_stream_t stream);

int flux_attn_decode_heads(flux_ctx* ctx, const uint16_t* q, const uint16_t* k_cache,
                           const uint16_t* v_cache, int S_max, const int32_t* seqlens,
                           uint16_t* o, float* lse, int B, int Hq, int Hkv, int d,
                           const uint8_t* head_mode, int sink_blocks, int window_blocks,
                           int block, float scale, flux_stream_t stream);

/* --------------------------------------------------------------------------
 * Decode attention that allocates nothing.  The pages have no counterpart of
 * this entry point; it exists for callers that cannot call cudaMalloc: an
 * inference engine that reserves all device memory up front and owns every
 * later allocation through its own pool, a plugin host that forbids libraries
 * from allocating, or a latency-critical loop that cannot afford cudaMalloc's
 * implicit device synchronisation.  Such callers cannot create a flux_ctx, so
 * this variant of flux_attn_decode keeps its split-KV scratch (partials,
 * merge tickets, error word) in one file-scope static device array of
 * 32 MiB inside libflux.so, which every GPU that loads the library holds until
 * the process exits.
 *   Arguments, layouts and results are those of flux_attn_decode, without the
 *   ctx.  status: optional device int32 that receives the device error word
 *   of this call (0 = OK, 2 = a seqlens entry out of range, 1 = a bounded
 *   wait ran out); NULL to skip.
 *   Limits: B * Hkv <= 4096 and B * Hq * nsplit * (d + 2) * 4 bytes of
 *   partials within the 32 MiB (nsplit as flux_decode_workspace_bytes plans
 *   it; e.g. B 16, Hq 32, d 128 at 131072 tokens takes 4 splits, 1.1 MiB).  Larger shapes
 *   return FLUX_ERR_SHAPE before any device work.
 *   Every call looks up the array's device address on the current device
 *   (cudaGetSymbolAddress, a host query that allocates nothing), so the entry
 *   point stays valid after cudaDeviceReset.  The first call on a device may
 *   load the library's device code there; make that first call before any
 *   stream capture.  Every call clears the error word and the tickets it uses
 *   on `stream`, then reuses the same array: calls that overlap on the GPU (on
 *   different streams or host threads) race and must be serialised by the
 *   caller. */
int flux_attn_decode_noalloc(const uint16_t* q, const uint16_t* k_cache, const uint16_t* v_cache,
                             int S_max, const int32_t* seqlens, uint16_t* o, float* lse,
                             int B, int Hq, int Hkv, int d,
                             const uint8_t* layer_mode, int layer,
                             int sink_blocks, int window_blocks, int block, float scale,
                             int32_t* status, flux_stream_t stream);

/* Workspace bytes flux_attn_decode needs on this ctx's device for this shape
 * and SA window (host-only query; no device work). */
int flux_decode_workspace_bytes(flux_ctx* ctx, int B, int Hq, int Hkv, int d, int S_max,
                                int sink_blocks, int window_blocks, int block, size_t* bytes);

#ifdef __cplusplus
}
#endif

#endif /* FLUX_H */
