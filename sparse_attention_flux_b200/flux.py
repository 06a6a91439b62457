"""Thin Python binding of libflux (the C ABI in include/flux.h).

Argument marshalling only: every step of the routed-attention path runs in
the CUDA kernels of libflux.so.  Tensors are torch tensors on the CUDA device
(torch provides device memory and streams); their data pointers and the
current torch stream are passed straight through the C ABI.  There is no CPU
fallback: if libflux.so is missing or a call fails, an exception is raised.

Names follow the C ABI: ``route``, ``build_streaming_mask``,
``build_block_index``, ``attn_prefill``, ``attn_decode``.
"""
from __future__ import annotations

import ctypes
import os
import re
import threading

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libflux.so")
HEADER = os.path.join(os.path.dirname(PKG), "include", "flux.h")

FLUX_OK = 0
FLUX_ERR_INVALID_ARG = -1
FLUX_ERR_SHAPE = -2
FLUX_ERR_UNSUPPORTED = -3
FLUX_ERR_CUDA = -4
FLUX_ERR_TIMEOUT = -5
FLUX_ERR_DEVICE_CHECK = -6


class FluxError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"libflux error {code}: {msg}")
        self.code = code


_lock = threading.Lock()
_lib = None

_vp = ctypes.c_void_p
_i = ctypes.c_int
_f = ctypes.c_float

_SIGNATURES = {
    "flux_version": ([], _i),
    "flux_last_error": ([], ctypes.c_char_p),
    "flux_ctx_create": ([ctypes.POINTER(_vp), _i, ctypes.c_size_t], _i),
    "flux_ctx_destroy": ([_vp], _i),
    "flux_ctx_check": ([_vp, _vp], _i),
    "flux_ctx_set_spin_limit_ms": ([_vp, _i], _i),
    "flux_route": ([_vp, _vp, _i, _i, _i, _vp, _vp, _i, _vp, _vp, _i, _f, _vp, _vp, _vp], _i),
    "flux_build_streaming_mask": ([_i, _i, _i, _i, _vp, _vp], _i),
    "flux_build_block_index": ([_vp, _vp, _i, _i, _vp, _vp, _i, _vp], _i),
    "flux_select_blocks": ([_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _f, _f, _i, _vp, _vp, _vp],
                           _i),
    "flux_select_blocks_workspace_bytes": ([_i, _i, _i, _i, _i], ctypes.c_size_t),
    "flux_attn_prefill": ([_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _i, _vp, _vp,
                           _i, _i, _f, _vp], _i),
    "flux_attn_decode": ([_vp, _vp, _vp, _vp, _i, _vp, _vp, _vp, _i, _i, _i, _i, _vp, _i, _i, _i,
                          _i, _f, _vp], _i),
    "flux_decode_workspace_bytes": ([_vp, _i, _i, _i, _i, _i, _i, _i, _i,
                                     ctypes.POINTER(ctypes.c_size_t)], _i),
    "flux_attn_prefill_soft": ([_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _i, _vp, _vp, _i,
                                _i, _f, _vp], _i),
    "flux_attn_prefill_heads": ([_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _vp, _vp,
                                 _i, _i, _f, _vp], _i),
    "flux_attn_decode_heads": ([_vp, _vp, _vp, _vp, _i, _vp, _vp, _vp, _i, _i, _i, _i, _vp, _i, _i,
                                _i, _f, _vp], _i),
    "flux_selftest_bounded_wait": ([_vp, _i, _vp, _vp], _i),
    "flux_kv_write": ([_vp, _vp, _vp, _i, _vp, _i, _i, _i, _vp, _vp, _i, _i, _i, _i, _vp], _i),
    "flux_attn_decode_sa_compact": ([_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i,
                                     _f, _vp], _i),
    "flux_attn_decode_noalloc": ([_vp, _vp, _vp, _i, _vp, _vp, _vp, _i, _i, _i, _i, _vp, _i, _i,
                                  _i, _i, _f, _vp, _vp], _i),
    "flux_attn_decode_append": ([_vp, _vp, _vp, _vp, _vp, _vp, _i, _vp, _vp, _vp, _i, _i, _i, _i,
                                 _vp, _i, _i, _i, _i, _i, _f, _vp], _i),
}


def header_symbols(path: str = HEADER):
    """Function names declared in include/flux.h."""
    with open(path) as f:
        text = re.sub(r"/\*.*?\*/", "", f.read(), flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(flux_\w+)\s*\(", text, flags=re.M)))


def lib() -> ctypes.CDLL:
    """Load libflux.so (built in-tree by sparse_attention_flux_b200.build)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"{LIB_PATH} is missing: build it with `python -m sparse_attention_flux_b200.build`"
                    " (there is no CPU fallback)")
            L = ctypes.CDLL(LIB_PATH)
            for name, (args, res) in _SIGNATURES.items():
                fn = getattr(L, name)
                fn.argtypes = args
                fn.restype = res
            _lib = L
    return _lib


def _check(rc: int):
    if rc != FLUX_OK:
        raise FluxError(rc, lib().flux_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _need(t, dtype, name, device=None):
    import torch
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")


class Context:
    """Owns a flux_ctx: the device workspace and the device error word."""

    def __init__(self, device: int = 0, workspace_bytes: int = 0):
        import torch
        self.device = torch.device("cuda", device)
        h = ctypes.c_void_p()
        _check(lib().flux_ctx_create(ctypes.byref(h), device, workspace_bytes))
        self._h = h

    def close(self):
        if getattr(self, "_h", None):
            lib().flux_ctx_destroy(self._h)
            self._h = None

    def __del__(self):  # pragma: no cover - interpreter shutdown order
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    @property
    def handle(self):
        return self._h

    def check(self, stream=None) -> None:
        """Synchronize the stream and raise if a device-side check failed."""
        _check(lib().flux_ctx_check(self._h, _stream(stream)))

    def set_spin_limit_ms(self, ms: int) -> None:
        _check(lib().flux_ctx_set_spin_limit_ms(self._h, int(ms)))

    def selftest_bounded_wait(self, spin_limit_ms: int, waited_us=None, stream=None) -> None:
        """Launch a wait that can never complete; the bounded wait must give up."""
        _check(lib().flux_selftest_bounded_wait(self._h, int(spin_limit_ms), _ptr(waited_us),
                                                _stream(stream)))

    def decode_workspace_bytes(self, B, Hq, Hkv, d, S_max, sink_blocks, window_blocks, block) -> int:
        n = ctypes.c_size_t()
        _check(lib().flux_decode_workspace_bytes(self._h, B, Hq, Hkv, d, S_max, sink_blocks,
                                                 window_blocks, block, ctypes.byref(n)))
        return n.value

    # ------------------------------------------------------------------ router
    def route(self, hidden, W1, b1, W2, b2, thresh: float, layer_mode, score=None,
              n_pool: int = 100, stream=None):
        import torch
        _need(hidden, torch.bfloat16, "hidden", self.device)
        for n_, t in (("W1", W1), ("b1", b1), ("W2", W2), ("b2", b2), ("score", score)):
            _need(t, torch.float32, n_, self.device)
        _need(layer_mode, torch.uint8, "layer_mode", self.device)
        T, Hd = hidden.shape
        H1, L = W1.shape[0], W2.shape[0]
        if W1.shape != (H1, 2 * Hd) or W2.shape != (L, H1) or b1.numel() != H1 or b2.numel() != L:
            raise ValueError("router weight shapes do not match hidden")
        if layer_mode.numel() < L or (score is not None and score.numel() < L):
            raise ValueError("layer_mode/score too small")
        _check(lib().flux_route(self._h, _ptr(hidden), T, Hd, n_pool, _ptr(W1), _ptr(b1), H1,
                                _ptr(W2), _ptr(b2), L, float(thresh), _ptr(layer_mode),
                                _ptr(score), _stream(stream)))

    # ------------------------------------------------------------------ masks
    def build_streaming_mask(self, nqb: int, nkb: int, sink_blocks: int, window_blocks: int,
                             block_mask, stream=None):
        import torch
        _need(block_mask, torch.uint8, "block_mask", self.device)
        if block_mask.numel() < nqb * nkb:
            raise ValueError("block_mask too small")
        _check(lib().flux_build_streaming_mask(nqb, nkb, sink_blocks, window_blocks,
                                               _ptr(block_mask), _stream(stream)))

    def build_block_index(self, block_mask, row_ptr, col, stream=None):
        import torch
        _need(block_mask, torch.uint8, "block_mask", self.device)
        _need(row_ptr, torch.int32, "row_ptr", self.device)
        _need(col, torch.int32, "col", self.device)
        nqb, nkb = block_mask.shape
        if row_ptr.numel() < nqb + 1:
            raise ValueError("row_ptr needs nqb + 1 entries")
        _check(lib().flux_build_block_index(self._h, _ptr(block_mask), nqb, nkb, _ptr(row_ptr),
                                            _ptr(col), col.numel(), _stream(stream)))

    def select_blocks_workspace_bytes(self, B: int, T: int, Hq: int, Hkv: int,
                                      stride: int = 8) -> int:
        """Bytes of ctx workspace flux_select_blocks needs (0 for unsupported sizes)."""
        return int(lib().flux_select_blocks_workspace_bytes(B, T, Hq, Hkv, stride))

    def select_blocks(self, q, k, block_mask, scale: float, tau: float, sink_blocks: int = 0,
                      stride: int = 8, block: int = 128, block_score=None, stream=None):
        """flux_select_blocks: a dynamic SA block mask [nb, nb] from this layer's q, k."""
        import torch
        _need(q, torch.bfloat16, "q", self.device)
        _need(k, torch.bfloat16, "k", self.device)
        _need(block_mask, torch.uint8, "block_mask", self.device)
        B, T, Hq, d = q.shape
        Hkv = k.shape[2]
        if k.shape != (B, T, Hkv, d):
            raise ValueError("q/k shapes are inconsistent")
        nb = (T + block - 1) // block
        if block_mask.numel() < nb * nb:
            raise ValueError("block_mask needs nb * nb entries")
        if block_score is not None:
            _need(block_score, torch.float32, "block_score", self.device)
            if block_score.numel() < nb * nb:
                raise ValueError("block_score needs nb * nb entries")
        _check(lib().flux_select_blocks(self._h, _ptr(q), _ptr(k), B, T, Hq, Hkv, d, block,
                                        stride, float(scale), float(tau), sink_blocks,
                                        _ptr(block_mask), _ptr(block_score), _stream(stream)))

    # ------------------------------------------------------------------ attention
    def attn_prefill(self, q, k, v, o, scale: float, layer_mode=None, layer: int = 0,
                     row_ptr=None, col=None, block: int = 128, lse=None, stream=None):
        import torch
        for n_, t in (("q", q), ("k", k), ("v", v), ("o", o)):
            _need(t, torch.bfloat16, n_, self.device)
        _need(lse, torch.float32, "lse", self.device)
        _need(layer_mode, torch.uint8, "layer_mode", self.device)
        _need(row_ptr, torch.int32, "row_ptr", self.device)
        _need(col, torch.int32, "col", self.device)
        B, T, Hq, d = q.shape
        Hkv = k.shape[2]
        if k.shape != (B, T, Hkv, d) or v.shape != k.shape or o.shape != q.shape:
            raise ValueError("q/k/v/o shapes are inconsistent")
        if lse is not None and lse.numel() < B * Hq * T:
            raise ValueError("lse too small")
        nqb = 0 if row_ptr is None else row_ptr.numel() - 1
        _check(lib().flux_attn_prefill(self._h, _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B,
                                       T, Hq, Hkv, d, _ptr(layer_mode), layer, _ptr(row_ptr),
                                       _ptr(col), nqb, block, float(scale), _stream(stream)))

    def attn_prefill_soft(self, q, k, v, o, scale: float, score, layer: int, row_ptr, col,
                          block: int = 128, stream=None):
        """o = r * FA + (1 - r) * SA with r = score[layer] (device), forward only."""
        import torch
        for n_, t in (("q", q), ("k", k), ("v", v), ("o", o)):
            _need(t, torch.bfloat16, n_, self.device)
        _need(score, torch.float32, "score", self.device)
        _need(row_ptr, torch.int32, "row_ptr", self.device)
        _need(col, torch.int32, "col", self.device)
        B, T, Hq, d = q.shape
        Hkv = k.shape[2]
        if k.shape != (B, T, Hkv, d) or v.shape != k.shape or o.shape != q.shape:
            raise ValueError("q/k/v/o shapes are inconsistent")
        _check(lib().flux_attn_prefill_soft(self._h, _ptr(q), _ptr(k), _ptr(v), _ptr(o), B, T, Hq,
                                            Hkv, d, _ptr(score), layer, _ptr(row_ptr), _ptr(col),
                                            row_ptr.numel() - 1, block, float(scale),
                                            _stream(stream)))

    def attn_decode(self, q, k_cache, v_cache, seqlens, o, scale: float, layer_mode=None,
                    layer: int = 0, sink_blocks: int = 1, window_blocks: int = 16,
                    block: int = 128, lse=None, stream=None):
        import torch
        for n_, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache), ("o", o)):
            _need(t, torch.bfloat16, n_, self.device)
        _need(seqlens, torch.int32, "seqlens", self.device)
        _need(lse, torch.float32, "lse", self.device)
        _need(layer_mode, torch.uint8, "layer_mode", self.device)
        B, Hq, d = q.shape
        _, S_max, Hkv, _ = k_cache.shape
        if k_cache.shape != (B, S_max, Hkv, d) or v_cache.shape != k_cache.shape:
            raise ValueError("cache shapes are inconsistent")
        if o.shape != q.shape or seqlens.numel() < B:
            raise ValueError("o/seqlens shapes are inconsistent")
        if lse is not None and lse.numel() < B * Hq:
            raise ValueError("lse too small")
        _check(lib().flux_attn_decode(self._h, _ptr(q), _ptr(k_cache), _ptr(v_cache), S_max,
                                      _ptr(seqlens), _ptr(o), _ptr(lse), B, Hq, Hkv, d,
                                      _ptr(layer_mode), layer, sink_blocks, window_blocks, block,
                                      float(scale), _stream(stream)))

    # ------------------------------------------------------------------ per-head routing
    def attn_prefill_heads(self, q, k, v, o, scale: float, head_mode, row_ptr, col,
                           block: int = 128, lse=None, stream=None):
        import torch
        for n_, t in (("q", q), ("k", k), ("v", v), ("o", o)):
            _need(t, torch.bfloat16, n_, self.device)
        _need(head_mode, torch.uint8, "head_mode", self.device)
        _need(lse, torch.float32, "lse", self.device)
        _need(row_ptr, torch.int32, "row_ptr", self.device)
        _need(col, torch.int32, "col", self.device)
        if row_ptr is None or col is None:
            raise ValueError("row_ptr and col are required")
        B, T, Hq, d = q.shape
        Hkv = k.shape[2]
        if head_mode.numel() < Hq or k.shape != (B, T, Hkv, d) or v.shape != k.shape \
                or o.shape != q.shape:
            raise ValueError("shapes are inconsistent")
        if lse is not None and lse.numel() < B * Hq * T:
            raise ValueError("lse too small")
        _check(lib().flux_attn_prefill_heads(self._h, _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                             B, T, Hq, Hkv, d, _ptr(head_mode), _ptr(row_ptr),
                                             _ptr(col), row_ptr.numel() - 1, block, float(scale),
                                             _stream(stream)))

    def attn_decode_heads(self, q, k_cache, v_cache, seqlens, o, scale: float, head_mode,
                          sink_blocks: int = 1, window_blocks: int = 16, block: int = 128,
                          lse=None, stream=None):
        import torch
        for n_, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache), ("o", o)):
            _need(t, torch.bfloat16, n_, self.device)
        _need(head_mode, torch.uint8, "head_mode", self.device)
        _need(seqlens, torch.int32, "seqlens", self.device)
        _need(lse, torch.float32, "lse", self.device)
        B, Hq, d = q.shape
        _, S_max, Hkv, _ = k_cache.shape
        if head_mode.numel() < Hq or k_cache.shape != (B, S_max, Hkv, d) \
                or v_cache.shape != k_cache.shape or o.shape != q.shape or seqlens.numel() < B:
            raise ValueError("shapes are inconsistent")
        if lse is not None and lse.numel() < B * Hq:
            raise ValueError("lse too small")
        _check(lib().flux_attn_decode_heads(self._h, _ptr(q), _ptr(k_cache), _ptr(v_cache), S_max,
                                            _ptr(seqlens), _ptr(o), _ptr(lse), B, Hq, Hkv, d,
                                            _ptr(head_mode), sink_blocks, window_blocks, block,
                                            float(scale), _stream(stream)))

    # ------------------------------------------------------------------ KV caches
    def kv_write(self, k_src, v_src, seqlens, k_cache, v_cache, sink_blocks: int = 0,
                 window_blocks: int = 0, block: int = 128, stream=None):
        """Write the last n_src tokens of each sequence into a full cache (window_blocks=0)
        or an SA layer's compact ring cache."""
        import torch
        for n_, t in (("k_src", k_src), ("v_src", v_src), ("k_cache", k_cache),
                      ("v_cache", v_cache)):
            _need(t, torch.bfloat16, n_, self.device)
        _need(seqlens, torch.int32, "seqlens", self.device)
        B, n_src, Hkv, d = k_src.shape
        if v_src.shape != k_src.shape or k_cache.shape[0] != B or k_cache.shape[2:] != (Hkv, d) \
                or v_cache.shape != k_cache.shape or seqlens.numel() < B:
            raise ValueError("source / cache shapes are inconsistent")
        _check(lib().flux_kv_write(self._h, _ptr(k_src), _ptr(v_src), n_src, _ptr(seqlens), B, Hkv,
                                   d, _ptr(k_cache), _ptr(v_cache), k_cache.shape[1], sink_blocks,
                                   window_blocks, block, _stream(stream)))

    def attn_decode_sa_compact(self, q, k_ring, v_ring, seqlens, o, scale: float,
                               sink_blocks: int = 1, window_blocks: int = 16, block: int = 128,
                               lse=None, stream=None):
        import torch
        for n_, t in (("q", q), ("k_ring", k_ring), ("v_ring", v_ring), ("o", o)):
            _need(t, torch.bfloat16, n_, self.device)
        _need(seqlens, torch.int32, "seqlens", self.device)
        _need(lse, torch.float32, "lse", self.device)
        B, Hq, d = q.shape
        rows = (sink_blocks + window_blocks) * block
        if k_ring.shape[0] != B or k_ring.shape[1] != rows or k_ring.shape[3] != d \
                or v_ring.shape != k_ring.shape or o.shape != q.shape:
            raise ValueError("ring / q / o shapes are inconsistent")
        _check(lib().flux_attn_decode_sa_compact(self._h, _ptr(q), _ptr(k_ring), _ptr(v_ring),
                                                 _ptr(seqlens), _ptr(o), _ptr(lse), B, Hq,
                                                 k_ring.shape[2], d, sink_blocks, window_blocks,
                                                 block, float(scale), _stream(stream)))

    def attn_decode_append(self, q, k_new, v_new, k_cache, v_cache, seqlens, o, scale: float,
                           layer_mode=None, layer: int = 0, sink_blocks: int = 1,
                           window_blocks: int = 16, block: int = 128, compact: bool = False,
                           lse=None, stream=None):
        """One decode step with the step's KV append fused: k_new/v_new [B, Hkv, d] (or
        [B, 1, Hkv, d]) become token seqlens[b] - 1 of the cache -- a full cache routed by
        layer_mode, or (compact=True) an SA layer's ring -- and q attends."""
        import torch
        for n_, t in (("q", q), ("k_new", k_new), ("v_new", v_new), ("k_cache", k_cache),
                      ("v_cache", v_cache), ("o", o)):
            _need(t, torch.bfloat16, n_, self.device)
        _need(seqlens, torch.int32, "seqlens", self.device)
        _need(lse, torch.float32, "lse", self.device)
        _need(layer_mode, torch.uint8, "layer_mode", self.device)
        B, Hq, d = q.shape
        _, rows, Hkv, _ = k_cache.shape
        if k_cache.shape[0] != B or k_cache.shape[3] != d or v_cache.shape != k_cache.shape \
                or o.shape != q.shape or k_new.numel() != B * Hkv * d or v_new.shape != k_new.shape \
                or seqlens.numel() < B:
            raise ValueError("q / k_new / cache / o shapes are inconsistent")
        if lse is not None and lse.numel() < B * Hq:
            raise ValueError("lse too small")
        _check(lib().flux_attn_decode_append(self._h, _ptr(q), _ptr(k_new), _ptr(v_new),
                                             _ptr(k_cache), _ptr(v_cache), rows, _ptr(seqlens),
                                             _ptr(o), _ptr(lse), B, Hq, Hkv, d, _ptr(layer_mode),
                                             layer, sink_blocks, window_blocks, block,
                                             1 if compact else 0, float(scale), _stream(stream)))


def attn_decode_noalloc(q, k_cache, v_cache, seqlens, o, scale: float, layer_mode=None,
                        layer: int = 0, sink_blocks: int = 1, window_blocks: int = 16,
                        block: int = 128, lse=None, status=None, stream=None):
    """flux_attn_decode_noalloc: decode without a Context; scratch lives in a static
    32 MiB device array inside libflux.so (see include/flux.h for the limits)."""
    import torch
    for n_, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache), ("o", o)):
        _need(t, torch.bfloat16, n_)
    _need(seqlens, torch.int32, "seqlens")
    _need(lse, torch.float32, "lse")
    _need(layer_mode, torch.uint8, "layer_mode")
    _need(status, torch.int32, "status")
    B, Hq, d = q.shape
    _, S_max, Hkv, _ = k_cache.shape
    if k_cache.shape != (B, S_max, Hkv, d) or v_cache.shape != k_cache.shape or o.shape != q.shape \
            or seqlens.numel() < B:
        raise ValueError("q/cache/o shapes are inconsistent")
    if lse is not None and lse.numel() < B * Hq:
        raise ValueError("lse too small")
    _check(lib().flux_attn_decode_noalloc(_ptr(q), _ptr(k_cache), _ptr(v_cache), S_max,
                                          _ptr(seqlens), _ptr(o), _ptr(lse), B, Hq, Hkv, d,
                                          _ptr(layer_mode), layer, sink_blocks, window_blocks,
                                          block, float(scale), _ptr(status), _stream(stream)))
