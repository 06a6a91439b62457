// api.cu -- the C ABI of libflux (declared in include/flux.h): context and
// workspace management, host-side argument checks, TMA tensor-map encoding
// and the kernel launches.  No torch types cross this boundary.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>

#include "flux.h"
#include "kernels.h"

struct flux_ctx {
  int device;
  int num_sms;
  void* workspace;        // scratch shared by the calls (they must not overlap in time)
  size_t workspace_bytes;
  int* tickets;           // [kMaxTickets + 1] ints, zero between calls; last one: router
  int* err;               // device error word
  long long spin_ns;
};

namespace {

constexpr int kMaxTickets = 1 << 16;
thread_local std::string g_last_error;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(FLUX_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ---- TMA descriptor encoding through the driver entry point (no -lcuda)
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;
std::once_flag g_encode_once;

EncodeTiledFn encode_fn() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  });
  return g_encode;
}

// A bf16 tensor [d3][d2][d1][d0] (d0 innermost), boxes of box0 x 1 x box2 x 1
// with the 128-byte swizzle; out-of-range rows read as zero.  With step2 > 1 a
// box takes every step2-th d2 row of its box2-row span (box2 / step2 rows).
int make_map_4d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                uint64_t d3, uint32_t box0, uint32_t box2, uint32_t step2 = 1) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(FLUX_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  const cuuint64_t gdim[4] = {d0, d1, d2, d3};
  const cuuint64_t gstride[3] = {d0 * 2, d0 * d1 * 2, d0 * d1 * d2 * 2};
  const cuuint32_t box[4] = {box0, 1, box2, 1};
  const cuuint32_t estride[4] = {1, 1, step2, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), gdim,
                         gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(FLUX_ERR_SHAPE, "tensor map encoding failed (CUresult %d)", r);
  return FLUX_OK;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

flux::DevStatus status_of(const flux_ctx* c) { return flux::DevStatus{c->err, c->spin_ns}; }

// ---- prefill entry points: one argument set, one set of host checks, one launch path
struct PrefillCall {
  const char* name;
  const uint16_t* q;
  const uint16_t* k;
  const uint16_t* v;
  uint16_t* o;
  float* lse;
  int B, T, Hq, Hkv, d;
  const uint8_t* layer_mode;
  int layer;
  const int32_t* row_ptr;
  const int32_t* col;
  int nqb, block;
  float scale;
  int force_mode;                // -1: layer_mode / head_mode decide; 0: SA; 1: FA
  const uint8_t* head_mode;      // per-query-head routing, or null
  const float* blend_score;      // soft routing: blend into o with r = score[layer], or null
};

// The checks every prefill entry point shares; nothing is launched on failure.
// A call that may take the SA path needs the CSR block index.
int check_prefill(const PrefillCall& a) {
  if (!a.q || !a.k || !a.v || !a.o) return fail(FLUX_ERR_INVALID_ARG, "%s: null tensor", a.name);
  if (a.B < 1 || a.T < 1 || a.Hq < 1 || a.Hkv < 1)
    return fail(FLUX_ERR_SHAPE, "%s: sizes must be positive", a.name);
  if (a.d != 64 && a.d != 128)
    return fail(FLUX_ERR_UNSUPPORTED, "%s: head_dim %d (supported: 64, 128)", a.name, a.d);
  if (a.Hq % a.Hkv != 0)
    return fail(FLUX_ERR_UNSUPPORTED, "%s: Hq %% Hkv != 0 (%d, %d)", a.name, a.Hq, a.Hkv);
  if (a.block != 64 && (a.block < 128 || a.block % 128 != 0))
    return fail(FLUX_ERR_UNSUPPORTED, "%s: block %d (64 or a multiple of 128)", a.name, a.block);
  if (!(a.scale == a.scale) || a.scale <= 0.f || a.scale > 3.0e38f)
    return fail(FLUX_ERR_INVALID_ARG, "%s: scale must be finite and positive", a.name);
  if ((a.layer_mode || a.blend_score) && a.layer < 0)
    return fail(FLUX_ERR_INVALID_ARG, "%s: negative layer", a.name);
  const bool routed = a.layer_mode || a.head_mode || a.force_mode == 0;
  if (routed) {
    if (!a.row_ptr || !a.col)
      return fail(FLUX_ERR_INVALID_ARG, "%s: row_ptr/col are required for a routed call", a.name);
    if (a.nqb < (a.T + a.block - 1) / a.block)
      return fail(FLUX_ERR_SHAPE, "%s: nqb %d < ceil(T / block) = %d", a.name, a.nqb,
                  (a.T + a.block - 1) / a.block);
    if ((a.T + 127) / 128 > flux::kPrefillMaxKvTiles)
      return fail(FLUX_ERR_SHAPE, "%s: routed prefill supports T <= %d", a.name,
                  flux::kPrefillMaxKvTiles * 128);
  }
  if (!aligned16(a.q) || !aligned16(a.k) || !aligned16(a.v) || !aligned16(a.o))
    return fail(FLUX_ERR_INVALID_ARG, "%s: tensors must be 16-byte aligned", a.name);
  return FLUX_OK;
}

// Checks, tensor maps and the launch of one prefill pass on a context.
int run_prefill(flux_ctx* c, const PrefillCall& a, flux_stream_t stream) {
  if (!c) return fail(FLUX_ERR_INVALID_ARG, "%s: null context", a.name);
  int rc = check_prefill(a);
  if (rc != FLUX_OK) return rc;
  CUtensorMap tq, tk, tv, to;
  if ((rc = make_map_4d(&tq, a.q, a.d, a.Hq, a.T, a.B, 64, 128)) != FLUX_OK) return rc;
  if ((rc = make_map_4d(&tk, a.k, a.d, a.Hkv, a.T, a.B, 64, 128)) != FLUX_OK) return rc;
  if ((rc = make_map_4d(&tv, a.v, a.d, a.Hkv, a.T, a.B, 64, 128)) != FLUX_OK) return rc;
  if ((rc = make_map_4d(&to, a.o, a.d, a.Hq, a.T, a.B, 64, 128)) != FLUX_OK) return rc;
  const bool routed = a.layer_mode || a.head_mode || a.force_mode == 0;
  flux::PrefillLaunch p;
  p.B = a.B;
  p.T = a.T;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.d = a.d;
  p.block = a.block;
  p.nqb = routed ? a.nqb : 0;
  p.scale = a.scale;
  p.layer_mode = a.layer_mode;
  p.layer = a.layer;
  p.row_ptr = a.row_ptr;
  p.col = a.col;
  p.o = a.o;
  p.lse = a.lse;
  p.force_mode = a.force_mode;
  p.head_mode = a.head_mode;
  p.blend_score = a.blend_score;
  p.st = status_of(c);
  const cudaError_t e = flux::launch_prefill(tq, tk, tv, to, p, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FLUX_OK : cuda_fail(e, a.name);
}

// ---- decode entry points: one argument set, one set of host checks, one launch path
struct DecodeCall {
  const char* name;
  const uint16_t* q;
  const uint16_t* k_cache;
  const uint16_t* v_cache;
  int rows;                      // cache rows per sequence: S_max, or the ring's
  const int32_t* seqlens;
  uint16_t* o;
  float* lse;
  int B, Hq, Hkv, d;
  const uint8_t* layer_mode;
  int layer;
  const uint8_t* head_mode;      // per-query-head routing, or null
  int sink_blocks, window_blocks, block;
  float scale;
  int compact;                   // the cache is an SA ring of (sink + W) * block rows
  const uint16_t* k_new;         // fused append of token seqlens[b] - 1, or null
  const uint16_t* v_new;
};

// The checks every decode entry point shares; nothing is launched on failure.
int check_decode(const DecodeCall& a, long long max_groups) {
  if (!a.q || !a.k_cache || !a.v_cache || !a.seqlens || !a.o)
    return fail(FLUX_ERR_INVALID_ARG, "%s: null tensor", a.name);
  if (a.B < 1 || a.Hq < 1 || a.Hkv < 1 || a.rows < 1)
    return fail(FLUX_ERR_SHAPE, "%s: sizes must be positive", a.name);
  if (a.d != 64 && a.d != 128)
    return fail(FLUX_ERR_UNSUPPORTED, "%s: head_dim %d (supported: 64, 128)", a.name, a.d);
  if (a.Hq % a.Hkv != 0 || a.Hq / a.Hkv > flux::kDecodeMaxGroup)
    return fail(FLUX_ERR_UNSUPPORTED, "%s: Hq/Hkv must be a whole number from 1 to %d (%d, %d)",
                a.name, flux::kDecodeMaxGroup, a.Hq, a.Hkv);
  if (a.block < 1 || a.sink_blocks < 0 || a.window_blocks < 1)
    return fail(FLUX_ERR_INVALID_ARG, "%s: bad block / sink / window", a.name);
  if (a.compact && (a.block < 64 || a.block % 64 != 0))
    return fail(FLUX_ERR_UNSUPPORTED, "%s: a ring needs block a multiple of 64", a.name);
  if (a.compact && static_cast<long long>(a.sink_blocks + a.window_blocks) * a.block != a.rows)
    return fail(FLUX_ERR_SHAPE, "%s: ring rows must be (sink + window) * block", a.name);
  if (a.layer_mode && a.layer < 0) return fail(FLUX_ERR_INVALID_ARG, "%s: negative layer", a.name);
  if (!(a.scale == a.scale) || a.scale <= 0.f || a.scale > 3.0e38f)
    return fail(FLUX_ERR_INVALID_ARG, "%s: scale must be finite and positive", a.name);
  if (static_cast<long long>(a.B) * a.Hkv > max_groups)
    return fail(FLUX_ERR_SHAPE, "%s: B * Hkv = %lld exceeds %lld", a.name,
                static_cast<long long>(a.B) * a.Hkv, max_groups);
  if (!aligned16(a.q) || !aligned16(a.k_cache) || !aligned16(a.v_cache) ||
      (a.k_new && !aligned16(a.k_new)) || (a.v_new && !aligned16(a.v_new)))
    return fail(FLUX_ERR_INVALID_ARG, "%s: tensors must be 16-byte aligned", a.name);
  return FLUX_OK;
}

// The call's split plan (a ring needs only its SA splits) and the bytes of its
// split partials: o [B, Hq, nsplit, d] then (m, l), each 256-byte aligned.
size_t plan_decode(const DecodeCall& a, int num_sms, flux::DecodeLaunch* p, size_t* o_bytes) {
  flux::decode_plan(a.B, a.Hkv, a.rows, a.sink_blocks, a.window_blocks, a.block, num_sms,
                    &p->nsplit, &p->chunk_fa, &p->tiles_sa);
  if (a.compact)
    p->nsplit = flux::decode_sa_splits(a.sink_blocks, a.window_blocks, a.block, p->tiles_sa);
  const size_t rows = static_cast<size_t>(a.B) * a.Hq * p->nsplit;
  *o_bytes = align256(rows * a.d * sizeof(float));
  return *o_bytes + align256(rows * 2 * sizeof(float));
}

// Tensor maps and the launch, with the partials at `part`, the merge tickets
// and the error word / wait bound given.
int launch_decode_call(const DecodeCall& a, flux::DecodeLaunch& p, void* part, size_t o_bytes,
                       int* tickets, flux::DevStatus st, cudaStream_t stream) {
  CUtensorMap tk, tv;
  int rc;
  if ((rc = make_map_4d(&tk, a.k_cache, a.d, a.Hkv, a.rows, a.B, 64, 64)) != FLUX_OK) return rc;
  if ((rc = make_map_4d(&tv, a.v_cache, a.d, a.Hkv, a.rows, a.B, 64, 64)) != FLUX_OK) return rc;
  p.B = a.B;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.d = a.d;
  p.S_max = a.rows;
  p.q = a.q;
  p.seqlens = a.seqlens;
  p.o = a.o;
  p.lse = a.lse;
  p.layer_mode = a.layer_mode;
  p.layer = a.layer;
  p.sink_blocks = a.sink_blocks;
  p.window_blocks = a.window_blocks;
  p.block = a.block;
  p.scale = a.scale;
  p.compact = a.compact;
  p.head_mode = a.head_mode;
  p.part_o = static_cast<float*>(part);
  p.part_ml = reinterpret_cast<float*>(static_cast<char*>(part) + o_bytes);
  p.tickets = tickets;
  p.st = st;
  p.k_new = a.k_new;
  p.v_new = a.v_new;
  p.k_cache = const_cast<uint16_t*>(a.k_cache);
  p.v_cache = const_cast<uint16_t*>(a.v_cache);
  const cudaError_t e = flux::launch_decode(tk, tv, p, stream);
  return e == cudaSuccess ? FLUX_OK : cuda_fail(e, a.name);
}

// A decode call on a context: its workspace holds the partials.
int run_decode(flux_ctx* c, const DecodeCall& a, flux_stream_t stream) {
  if (!c) return fail(FLUX_ERR_INVALID_ARG, "%s: null context", a.name);
  int rc = check_decode(a, kMaxTickets);
  if (rc != FLUX_OK) return rc;
  flux::DecodeLaunch p;
  size_t o_bytes = 0;
  const size_t need = plan_decode(a, c->num_sms, &p, &o_bytes);
  if (need > c->workspace_bytes)
    return fail(FLUX_ERR_SHAPE, "%s: workspace %zu < %zu bytes", a.name, c->workspace_bytes, need);
  return launch_decode_call(a, p, c->workspace, o_bytes, c->tickets, status_of(c),
                            static_cast<cudaStream_t>(stream));
}

}  // namespace

extern "C" {

int flux_version(void) { return FLUX_ABI_VERSION; }

const char* flux_last_error(void) { return g_last_error.c_str(); }

int flux_ctx_create(flux_ctx** out, int device, size_t workspace_bytes) {
  if (!out) return fail(FLUX_ERR_INVALID_ARG, "flux_ctx_create: null output pointer");
  *out = nullptr;
  int ndev = 0;
  cudaError_t e = cudaGetDeviceCount(&ndev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDeviceCount");
  if (device < 0 || device >= ndev) return fail(FLUX_ERR_INVALID_ARG, "no CUDA device %d", device);
  if ((e = cudaSetDevice(device)) != cudaSuccess) return cuda_fail(e, "cudaSetDevice");
  cudaDeviceProp prop;
  if ((e = cudaGetDeviceProperties(&prop, device)) != cudaSuccess)
    return cuda_fail(e, "cudaGetDeviceProperties");
  if (prop.major != 10)
    return fail(FLUX_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a",
                device, prop.major, prop.minor);
  flux_ctx* c = static_cast<flux_ctx*>(calloc(1, sizeof(flux_ctx)));
  if (!c) return fail(FLUX_ERR_INVALID_ARG, "out of host memory");
  c->device = device;
  c->num_sms = prop.multiProcessorCount;
  c->workspace_bytes = workspace_bytes ? workspace_bytes : (size_t(64) << 20);
  c->spin_ns = 2000LL * 1000000LL;
  if (const char* s = getenv("FLUX_SPIN_LIMIT_MS")) {
    const long long ms = atoll(s);
    if (ms > 0) c->spin_ns = ms * 1000000LL;
  }
  if ((e = cudaMalloc(&c->workspace, c->workspace_bytes)) != cudaSuccess ||
      (e = cudaMalloc(reinterpret_cast<void**>(&c->tickets), (kMaxTickets + 1) * sizeof(int))) !=
          cudaSuccess ||
      (e = cudaMalloc(reinterpret_cast<void**>(&c->err), sizeof(int))) != cudaSuccess ||
      (e = cudaMemset(c->tickets, 0, (kMaxTickets + 1) * sizeof(int))) != cudaSuccess ||
      (e = cudaMemset(c->err, 0, sizeof(int))) != cudaSuccess ||
      (e = cudaDeviceSynchronize()) != cudaSuccess) {
    cudaFree(c->workspace);
    cudaFree(c->tickets);
    cudaFree(c->err);
    free(c);
    return cuda_fail(e, "flux_ctx_create: device allocation");
  }
  *out = c;
  return FLUX_OK;
}

int flux_ctx_destroy(flux_ctx* c) {
  if (!c) return fail(FLUX_ERR_INVALID_ARG, "flux_ctx_destroy: null ctx");
  cudaFree(c->workspace);
  cudaFree(c->tickets);
  cudaFree(c->err);
  free(c);
  return FLUX_OK;
}

int flux_ctx_set_spin_limit_ms(flux_ctx* c, int ms) {
  if (!c || ms <= 0) return fail(FLUX_ERR_INVALID_ARG, "flux_ctx_set_spin_limit_ms: bad argument");
  c->spin_ns = static_cast<long long>(ms) * 1000000LL;
  return FLUX_OK;
}

int flux_ctx_check(flux_ctx* c, flux_stream_t stream) {
  if (!c) return fail(FLUX_ERR_INVALID_ARG, "flux_ctx_check: null ctx");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "flux_ctx_check: stream synchronize");
  int word = 0;
  if ((e = cudaMemcpy(&word, c->err, sizeof(int), cudaMemcpyDeviceToHost)) != cudaSuccess)
    return cuda_fail(e, "flux_ctx_check: read error word");
  if (word == flux::DEV_OK) return FLUX_OK;
  // Clear the word and any ticket an aborted kernel left behind.
  cudaMemset(c->err, 0, sizeof(int));
  cudaMemset(c->tickets, 0, (kMaxTickets + 1) * sizeof(int));
  cudaDeviceSynchronize();
  switch (word) {
    case flux::DEV_ERR_TIMEOUT:
      return fail(FLUX_ERR_TIMEOUT, "a bounded device-side wait ran out");
    case flux::DEV_ERR_SEQLEN:
      return fail(FLUX_ERR_DEVICE_CHECK, "seqlens entry outside [0, S_max]");
    case flux::DEV_ERR_CSR:
      return fail(FLUX_ERR_DEVICE_CHECK,
                  "block-index list entry out of range or a row not strictly ascending");
    case flux::DEV_ERR_CAPACITY:
      return fail(FLUX_ERR_DEVICE_CHECK, "block-index nnz exceeds the col capacity");
    default:
      return fail(FLUX_ERR_DEVICE_CHECK, "device error word %d", word);
  }
}

int flux_route(flux_ctx* c, const uint16_t* hidden, int T, int Hd, int n_pool, const float* W1,
               const float* b1, int H1, const float* W2, const float* b2, int L, float thresh,
               uint8_t* layer_mode, float* score, flux_stream_t stream) {
  if (!c || !hidden || !W1 || !b1 || !W2 || !b2 || !layer_mode)
    return fail(FLUX_ERR_INVALID_ARG, "flux_route: null pointer argument");
  if (T < 1 || Hd < 1 || n_pool < 1 || H1 < 1 || L < 1)
    return fail(FLUX_ERR_INVALID_ARG, "flux_route: sizes must be positive");
  if (!(thresh == thresh) || thresh > 3.0e38f || thresh < -3.0e38f)
    return fail(FLUX_ERR_INVALID_ARG, "flux_route: thresh must be finite");
  if (!aligned16(hidden) || !aligned16(W1) || !aligned16(W2))
    return fail(FLUX_ERR_INVALID_ARG, "flux_route: hidden, W1 and W2 must be 16-byte aligned");
  const size_t need = flux::route_workspace_bytes(Hd, H1);
  if (need > c->workspace_bytes)
    return fail(FLUX_ERR_SHAPE, "flux_route: workspace %zu < %zu bytes", c->workspace_bytes, need);
  flux::RouteLaunch p;
  p.hidden = hidden;
  p.T = T;
  p.Hd = Hd;
  p.n_pool = n_pool;
  p.W1 = W1;
  p.b1 = b1;
  p.H1 = H1;
  p.W2 = W2;
  p.b2 = b2;
  p.L = L;
  p.thresh = thresh;
  p.layer_mode = layer_mode;
  p.score = score;
  p.pooled = static_cast<float*>(c->workspace);
  p.hidden1 = p.pooled + flux::route_hidden1_offset(Hd);
  p.ticket = c->tickets + kMaxTickets;
  const cudaError_t e = flux::launch_route(p, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FLUX_OK : cuda_fail(e, "flux_route: launch");
}

size_t flux_select_blocks_workspace_bytes(int B, int T, int Hq, int Hkv, int stride) {
  if (B < 1 || T < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || stride != 8 ||
      (T + 127) / 128 > flux::kSelectMaxBlocks)
    return 0;
  return flux::block_select_workspace_bytes(B, T, Hq, Hkv, stride);
}

int flux_select_blocks(flux_ctx* c, const uint16_t* q, const uint16_t* k, int B, int T, int Hq,
                       int Hkv, int d, int block, int stride, float scale, float tau,
                       int sink_blocks, uint8_t* block_mask, float* block_score,
                       flux_stream_t stream) {
  if (!c || !q || !k || !block_mask)
    return fail(FLUX_ERR_INVALID_ARG, "flux_select_blocks: null pointer argument");
  if (B < 1 || T < 1 || Hq < 1 || Hkv < 1)
    return fail(FLUX_ERR_SHAPE, "flux_select_blocks: sizes must be positive");
  if (d != 64 && d != 128)
    return fail(FLUX_ERR_UNSUPPORTED, "flux_select_blocks: head_dim %d (supported: 64, 128)", d);
  if (Hq % Hkv != 0)
    return fail(FLUX_ERR_UNSUPPORTED, "flux_select_blocks: Hq %% Hkv != 0 (%d, %d)", Hq, Hkv);
  if (block != 128 || stride != 8)
    return fail(FLUX_ERR_UNSUPPORTED, "flux_select_blocks: block %d stride %d (supported: "
                "block 128, stride 8)", block, stride);
  if ((T + block - 1) / block > flux::kSelectMaxBlocks)
    return fail(FLUX_ERR_UNSUPPORTED, "flux_select_blocks: T %d above %d", T,
                flux::kSelectMaxBlocks * block);
  if (!(scale == scale) || scale <= 0.f || scale > 3.0e38f)
    return fail(FLUX_ERR_INVALID_ARG, "flux_select_blocks: scale must be finite and positive");
  if (!(tau == tau) || tau < 0.f || tau > 3.0e38f || sink_blocks < 0)
    return fail(FLUX_ERR_INVALID_ARG, "flux_select_blocks: tau must be finite and >= 0, "
                "sink_blocks >= 0");
  if (!aligned16(q) || !aligned16(k))
    return fail(FLUX_ERR_INVALID_ARG, "flux_select_blocks: q and k must be 16-byte aligned");
  const size_t need = flux::block_select_workspace_bytes(B, T, Hq, Hkv, stride);
  if (need > c->workspace_bytes)
    return fail(FLUX_ERR_SHAPE, "flux_select_blocks: workspace %zu < %zu bytes",
                c->workspace_bytes, need);
  CUtensorMap tq, tk;
  int rc;
  // Strided boxes: each load brings the rows of one antidiagonal offset, so the
  // strided positions are consecutive rows in shared memory (Q: 16 rows of one
  // block; K: 32 rows spanning two blocks).
  if ((rc = make_map_4d(&tq, q, d, Hq, T, B, 64, 128, stride)) != FLUX_OK) return rc;
  if ((rc = make_map_4d(&tk, k, d, Hkv, T, B, 64, 256, stride)) != FLUX_OK) return rc;
  flux::BlockSelectLaunch p;
  p.B = B;
  p.T = T;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.d = d;
  p.stride = stride;
  p.scale = scale;
  p.tau = tau;
  p.sink_blocks = sink_blocks;
  p.block_mask = block_mask;
  p.block_score = block_score;
  p.workspace = static_cast<float*>(c->workspace);
  p.st = status_of(c);
  const cudaError_t e = flux::launch_block_select(tq, tk, p, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FLUX_OK : cuda_fail(e, "flux_select_blocks: launch");
}

int flux_build_streaming_mask(int nqb, int nkb, int sink_blocks, int window_blocks,
                              uint8_t* block_mask, flux_stream_t stream) {
  if (!block_mask) return fail(FLUX_ERR_INVALID_ARG, "flux_build_streaming_mask: null mask");
  if (nqb < 1 || nkb < 1 || sink_blocks < 0 || window_blocks < 1)
    return fail(FLUX_ERR_INVALID_ARG, "flux_build_streaming_mask: bad sizes");
  const cudaError_t e = flux::launch_streaming_mask(nqb, nkb, sink_blocks, window_blocks,
                                                    block_mask, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FLUX_OK : cuda_fail(e, "flux_build_streaming_mask: launch");
}

int flux_build_block_index(flux_ctx* c, const uint8_t* block_mask, int nqb, int nkb,
                           int32_t* row_ptr, int32_t* col, int cap, flux_stream_t stream) {
  if (!c || !block_mask || !row_ptr || !col)
    return fail(FLUX_ERR_INVALID_ARG, "flux_build_block_index: null pointer argument");
  if (nqb < 1 || nkb < 1 || cap < 0)
    return fail(FLUX_ERR_INVALID_ARG, "flux_build_block_index: bad sizes");
  if (static_cast<size_t>(nqb) * sizeof(int32_t) > c->workspace_bytes)
    return fail(FLUX_ERR_SHAPE, "flux_build_block_index: workspace too small");
  const cudaError_t e = flux::launch_block_index(block_mask, nqb, nkb, row_ptr, col, cap,
                                                 static_cast<int32_t*>(c->workspace), c->err,
                                                 static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FLUX_OK : cuda_fail(e, "flux_build_block_index: launch");
}

int flux_attn_prefill(flux_ctx* c, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                      uint16_t* o, float* lse, int B, int T, int Hq, int Hkv, int d,
                      const uint8_t* layer_mode, int layer, const int32_t* row_ptr,
                      const int32_t* col, int nqb, int block, float scale,
                      flux_stream_t stream) {
  const PrefillCall a{"flux_attn_prefill", q, k, v, o, lse, B, T, Hq, Hkv, d, layer_mode, layer,
                      row_ptr, col, nqb, block, scale, -1, nullptr, nullptr};
  return run_prefill(c, a, stream);
}

int flux_attn_prefill_soft(flux_ctx* c, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                           uint16_t* o, int B, int T, int Hq, int Hkv, int d, const float* score,
                           int layer, const int32_t* row_ptr, const int32_t* col, int nqb,
                           int block, float scale, flux_stream_t stream) {
  if (!score) return fail(FLUX_ERR_INVALID_ARG, "flux_attn_prefill_soft: score is required");
  // The SA pass is checked first, so that nothing is launched if either pass would fail.
  const PrefillCall sa{"flux_attn_prefill_soft", q, k, v, o, nullptr, B, T, Hq, Hkv, d, nullptr,
                       layer, row_ptr, col, nqb, block, scale, 0, nullptr, score};
  int rc = check_prefill(sa);
  if (rc != FLUX_OK) return rc;
  // FA pass into o, then the SA pass whose epilogue blends r * o_FA + (1 - r) * o_SA.
  const PrefillCall fa{"flux_attn_prefill_soft", q, k, v, o, nullptr, B, T, Hq, Hkv, d, nullptr,
                       layer, row_ptr, col, nqb, block, scale, 1, nullptr, nullptr};
  if ((rc = run_prefill(c, fa, stream)) != FLUX_OK) return rc;
  return run_prefill(c, sa, stream);
}

int flux_decode_workspace_bytes(flux_ctx* c, int B, int Hq, int Hkv, int d, int S_max,
                                int sink_blocks, int window_blocks, int block, size_t* bytes) {
  if (!c || !bytes || B < 1 || Hq < 1 || Hkv < 1 || d < 1 || S_max < 1 || block < 1 ||
      sink_blocks < 0 || window_blocks < 1)
    return fail(FLUX_ERR_INVALID_ARG, "flux_decode_workspace_bytes: bad arguments");
  int ns, cfa, csa;
  flux::decode_plan(B, Hkv, S_max, sink_blocks, window_blocks, block, c->num_sms, &ns, &cfa, &csa);
  *bytes = flux::decode_workspace_bytes(B, Hq, Hkv, d, ns);
  return FLUX_OK;
}

int flux_attn_decode(flux_ctx* c, const uint16_t* q, const uint16_t* k_cache,
                     const uint16_t* v_cache, int S_max, const int32_t* seqlens, uint16_t* o,
                     float* lse, int B, int Hq, int Hkv, int d, const uint8_t* layer_mode,
                     int layer, int sink_blocks, int window_blocks, int block, float scale,
                     flux_stream_t stream) {
  const DecodeCall a{"flux_attn_decode", q, k_cache, v_cache, S_max, seqlens, o, lse, B, Hq, Hkv,
                     d, layer_mode, layer, nullptr, sink_blocks, window_blocks, block, scale,
                     0, nullptr, nullptr};
  return run_decode(c, a, stream);
}

int flux_kv_write(flux_ctx* c, const uint16_t* k_src, const uint16_t* v_src, int n_src,
                  const int32_t* seqlens, int B, int Hkv, int d, uint16_t* k_cache,
                  uint16_t* v_cache, int cache_rows, int sink_blocks, int window_blocks,
                  int block, flux_stream_t stream) {
  if (!c || !k_src || !v_src || !seqlens || !k_cache || !v_cache)
    return fail(FLUX_ERR_INVALID_ARG, "flux_kv_write: null pointer argument");
  if (n_src < 1 || B < 1 || Hkv < 1 || d < 1 || cache_rows < 1 || sink_blocks < 0 ||
      window_blocks < 0 || block < 1)
    return fail(FLUX_ERR_INVALID_ARG, "flux_kv_write: bad sizes");
  if ((static_cast<long long>(Hkv) * d) % 8 != 0)
    return fail(FLUX_ERR_UNSUPPORTED, "flux_kv_write: Hkv * d must be a multiple of 8");
  if (window_blocks > 0 && static_cast<long long>(sink_blocks + window_blocks) * block != cache_rows)
    return fail(FLUX_ERR_SHAPE, "flux_kv_write: ring cache_rows must be (sink + window) * block");
  if (!aligned16(k_src) || !aligned16(v_src) || !aligned16(k_cache) || !aligned16(v_cache))
    return fail(FLUX_ERR_INVALID_ARG, "flux_kv_write: tensors must be 16-byte aligned");
  const cudaError_t e = flux::launch_ring_write(
      k_src, v_src, n_src, seqlens, B, Hkv, d, k_cache, v_cache, sink_blocks, window_blocks,
      window_blocks > 0 ? block : cache_rows, c->err, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FLUX_OK : cuda_fail(e, "flux_kv_write: launch");
}

int flux_attn_decode_sa_compact(flux_ctx* c, const uint16_t* q, const uint16_t* k_ring,
                                const uint16_t* v_ring, const int32_t* seqlens, uint16_t* o,
                                float* lse, int B, int Hq, int Hkv, int d, int sink_blocks,
                                int window_blocks, int block, float scale, flux_stream_t stream) {
  const long long rows = static_cast<long long>(sink_blocks + window_blocks) * block;
  if (rows < 1 || rows > (1LL << 30))
    return fail(FLUX_ERR_INVALID_ARG, "flux_attn_decode_sa_compact: bad sink / window / block");
  const DecodeCall a{"flux_attn_decode_sa_compact", q, k_ring, v_ring, static_cast<int>(rows),
                     seqlens, o, lse, B, Hq, Hkv, d, nullptr, 0, nullptr, sink_blocks,
                     window_blocks, block, scale, 1, nullptr, nullptr};
  return run_decode(c, a, stream);
}

int flux_attn_decode_append(flux_ctx* c, const uint16_t* q, const uint16_t* k_new,
                            const uint16_t* v_new, uint16_t* k_cache, uint16_t* v_cache,
                            int cache_rows, const int32_t* seqlens, uint16_t* o, float* lse,
                            int B, int Hq, int Hkv, int d, const uint8_t* layer_mode, int layer,
                            int sink_blocks, int window_blocks, int block, int compact,
                            float scale, flux_stream_t stream) {
  if (!k_new || !v_new)
    return fail(FLUX_ERR_INVALID_ARG, "flux_attn_decode_append: null k_new / v_new");
  if (compact != 0 && compact != 1)
    return fail(FLUX_ERR_INVALID_ARG, "flux_attn_decode_append: compact must be 0 or 1");
  const DecodeCall a{"flux_attn_decode_append", q, k_cache, v_cache, cache_rows, seqlens, o, lse,
                     B, Hq, Hkv, d, compact ? nullptr : layer_mode, compact ? 0 : layer, nullptr,
                     sink_blocks, window_blocks, block, scale, compact, k_new, v_new};
  return run_decode(c, a, stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// flux_attn_decode_noalloc: flux_attn_decode for callers that cannot call
// cudaMalloc (an engine that owns all device memory through its own pool, a
// plugin host that forbids library allocations, a loop that cannot take
// cudaMalloc's implicit synchronisation).  Its scratch is the static array
// below, which every device that loads libflux.so holds until the process
// exits.  Host code must not pass the array's name to a kernel -- on the host
// it is only a stand-in symbol -- so every call looks up the array's device
// address on the current device.  The lookup is a host query that allocates
// nothing; doing it per call (rather than caching the address) keeps the entry
// point valid after cudaDeviceReset, which unloads the module and gives the
// array a new address when the next call loads it again.  Only the SM count is
// cached per device.
namespace {

constexpr size_t kNoAllocBytes = size_t(32) << 20;        // 32 MiB
constexpr int kNoAllocMaxGroups = 4096;                    // B * Hkv
constexpr size_t kNoAllocErrOff = 0;                       // error word
constexpr size_t kNoAllocTicketOff = 256;                  // [kNoAllocMaxGroups] int
constexpr size_t kNoAllocPartOff = kNoAllocTicketOff + kNoAllocMaxGroups * sizeof(int);

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

constexpr int kNoAllocMaxDevices = 64;
int g_noalloc_sms[kNoAllocMaxDevices];   // 0 = not yet queried
std::mutex g_noalloc_mu;

// The scratch array's device address and the SM count of the current device.
int noalloc_setup(char** base, int* num_sms) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "flux_attn_decode_noalloc: cudaGetDevice");
  if (dev < 0 || dev >= kNoAllocMaxDevices)
    return fail(FLUX_ERR_UNSUPPORTED, "flux_attn_decode_noalloc: device %d out of range", dev);
  void* ptr = nullptr;
  if ((e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch)) != cudaSuccess)
    return cuda_fail(e, "flux_attn_decode_noalloc: cudaGetSymbolAddress");
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_sms[dev] == 0) {
    int sms = 0;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return cuda_fail(e, "flux_attn_decode_noalloc: SM count");
    g_noalloc_sms[dev] = sms;
  }
  *base = static_cast<char*>(ptr);
  *num_sms = g_noalloc_sms[dev];
  return FLUX_OK;
}

}  // namespace

extern "C" int flux_attn_decode_noalloc(const uint16_t* q, const uint16_t* k_cache,
                                        const uint16_t* v_cache, int S_max,
                                        const int32_t* seqlens, uint16_t* o, float* lse, int B,
                                        int Hq, int Hkv, int d, const uint8_t* layer_mode,
                                        int layer, int sink_blocks, int window_blocks, int block,
                                        float scale, int32_t* status, flux_stream_t stream) {
  const DecodeCall a{"flux_attn_decode_noalloc", q, k_cache, v_cache, S_max, seqlens, o, lse, B,
                     Hq, Hkv, d, layer_mode, layer, nullptr, sink_blocks, window_blocks, block,
                     scale, 0, nullptr, nullptr};
  int rc = check_decode(a, kNoAllocMaxGroups);
  if (rc != FLUX_OK) return rc;
  char* base = nullptr;
  int num_sms = 0;
  if ((rc = noalloc_setup(&base, &num_sms)) != FLUX_OK) return rc;
  flux::DecodeLaunch p;
  size_t o_bytes = 0;
  const size_t need = plan_decode(a, num_sms, &p, &o_bytes);
  if (kNoAllocPartOff + need > kNoAllocBytes)
    return fail(FLUX_ERR_SHAPE,
                "flux_attn_decode_noalloc: %zu bytes of split partials exceed the %zu-byte static "
                "scratch (use flux_attn_decode with a ctx for this shape)",
                need, kNoAllocBytes - kNoAllocPartOff);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* err = reinterpret_cast<int*>(base + kNoAllocErrOff);
  int* tickets = reinterpret_cast<int*>(base + kNoAllocTicketOff);
  // The array keeps the previous call's contents: the error word and this
  // call's tickets must start at zero.
  cudaError_t e = cudaMemsetAsync(err, 0, sizeof(int), s);
  if (e == cudaSuccess)
    e = cudaMemsetAsync(tickets, 0, static_cast<size_t>(B) * Hkv * sizeof(int), s);
  if (e != cudaSuccess) return cuda_fail(e, "flux_attn_decode_noalloc: clear scratch");
  rc = launch_decode_call(a, p, base + kNoAllocPartOff, o_bytes, tickets,
                          flux::DevStatus{err, 2000LL * 1000000LL}, s);
  if (rc != FLUX_OK) return rc;
  if (status && (e = cudaMemcpyAsync(status, err, sizeof(int), cudaMemcpyDeviceToDevice, s)) !=
                    cudaSuccess)
    return cuda_fail(e, "flux_attn_decode_noalloc: copy status");
  return FLUX_OK;
}

// ---------------------------------------------------------------------------
// Per-head routing: the contrast case for layer-level routing.

extern "C" int flux_attn_prefill_heads(flux_ctx* c, const uint16_t* q, const uint16_t* k,
                                       const uint16_t* v, uint16_t* o, float* lse, int B, int T,
                                       int Hq, int Hkv, int d, const uint8_t* head_mode,
                                       const int32_t* row_ptr, const int32_t* col, int nqb,
                                       int block, float scale, flux_stream_t stream) {
  if (!head_mode) return fail(FLUX_ERR_INVALID_ARG, "flux_attn_prefill_heads: head_mode is required");
  const PrefillCall a{"flux_attn_prefill_heads", q, k, v, o, lse, B, T, Hq, Hkv, d, nullptr, 0,
                      row_ptr, col, nqb, block, scale, -1, head_mode, nullptr};
  return run_prefill(c, a, stream);
}

extern "C" int flux_attn_decode_heads(flux_ctx* c, const uint16_t* q, const uint16_t* k_cache,
                                      const uint16_t* v_cache, int S_max, const int32_t* seqlens,
                                      uint16_t* o, float* lse, int B, int Hq, int Hkv, int d,
                                      const uint8_t* head_mode, int sink_blocks, int window_blocks,
                                      int block, float scale, flux_stream_t stream) {
  if (!head_mode) return fail(FLUX_ERR_INVALID_ARG, "flux_attn_decode_heads: head_mode is required");
  const DecodeCall a{"flux_attn_decode_heads", q, k_cache, v_cache, S_max, seqlens, o, lse, B, Hq,
                     Hkv, d, nullptr, 0, head_mode, sink_blocks, window_blocks, block, scale, 0,
                     nullptr, nullptr};
  return run_decode(c, a, stream);
}

// ---------------------------------------------------------------------------
extern "C" int flux_selftest_bounded_wait(flux_ctx* c, int spin_limit_ms, int* waited_us,
                                          flux_stream_t stream) {
  if (!c || spin_limit_ms < 1 || spin_limit_ms > 10000)
    return fail(FLUX_ERR_INVALID_ARG, "flux_selftest_bounded_wait: spin limit in [1, 10000] ms");
  flux::DevStatus st{c->err, static_cast<long long>(spin_limit_ms) * 1000000LL};
  const cudaError_t e = flux::launch_selftest_wait(st, waited_us, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FLUX_OK : cuda_fail(e, "flux_selftest_bounded_wait: launch");
}
