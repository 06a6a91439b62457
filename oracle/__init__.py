"""The oracle: a plain fp64 CPU implementation of the routed-attention hot path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg (``bench.py``) may import this package.  The
product path in ``sparse_attention_flux_b200`` never imports it and shares no
code with it.

The arithmetic lives in ``flux_oracle.c`` (plain C, fp64, OpenMP over
independent rows); this module only compiles it with gcc and marshals numpy
arrays through ctypes.  bf16 tensors are passed as their raw 16-bit patterns
(``numpy.uint16``), which the C code widens exactly to double.

Each function cites the passage it follows in its C definition.  Pins:
``tests/test_oracle.py`` and ``tests/test_block_select_oracle.py``.  One part is
"parity unpinned" against the pages: the dynamic SA block selector
(``block_scores``, ``select_blocks``), whose algorithm the pages do not give;
it is pinned to brute force, closed forms and invariants of the reading stated
in its C definition.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "flux_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

_u16p = np.ctypeslib.ndpointer(dtype=np.uint16, flags="C_CONTIGUOUS")
_f32p = np.ctypeslib.ndpointer(dtype=np.float32, flags="C_CONTIGUOUS")
_f64p = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")
_u8p = np.ctypeslib.ndpointer(dtype=np.uint8, flags="C_CONTIGUOUS")
_i32p = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")
_vp = ctypes.c_void_p


def build(force: bool = False) -> str:
    """Compile flux_oracle.c into liboracle.so (gcc, -O2, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-Wall", "-Wextra",
               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", _LIB, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


def lib() -> ctypes.CDLL:
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_LIB)
            i, d, f = ctypes.c_int, ctypes.c_double, ctypes.c_float
            L.oracle_num_threads.restype = i
            L.oracle_set_num_threads.argtypes = [i]
            L.oracle_pool.argtypes = [_u16p, i, i, i, _f64p]
            L.oracle_mlp.argtypes = [_f64p, i, _f32p, _f32p, i, _f32p, _f32p, i, _f64p]
            L.oracle_threshold.argtypes = [_f64p, i, f, _u8p, _vp]
            L.oracle_route.argtypes = [_u16p, i, i, i, _f32p, _f32p, i, _f32p, _f32p, i, f,
                                       _u8p, _vp, _vp]
            L.oracle_streaming_mask.argtypes = [i, i, i, i, _u8p]
            L.oracle_block_index.argtypes = [_u8p, i, i, _i32p, _i32p]
            L.oracle_attn_prefill.argtypes = [_u16p, _u16p, _u16p, i, i, i, i, i, _vp, i, i, d,
                                              _vp, ctypes.c_longlong, _f64p, _vp]
            L.oracle_attn_prefill_soft.argtypes = [_u16p, _u16p, _u16p, i, i, i, i, i, _u8p, i, i, d,
                                                   d, _vp, ctypes.c_longlong, _f64p]
            L.oracle_attn_probs.argtypes = [_u16p, _u16p, i, i, i, i, i, _vp, i, i, d, i, i, _f64p]
            L.oracle_attn_decode.argtypes = [_u16p, _u16p, _u16p, i, _i32p, i, i, i, i, i, i, i,
                                             i, d, _f64p, _vp]
            L.oracle_block_scores.argtypes = [_u16p, _u16p, i, i, i, i, i, i, i, d, _f64p]
            L.oracle_block_scores_rows.argtypes = [_u16p, _u16p, i, i, i, i, i, i, i, d,
                                                   _i32p, i, _f64p]
            L.oracle_select_blocks.argtypes = [_f32p, i, f, i, _u8p]
            _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _check(rc, what):
    if rc < 0:
        raise ValueError(f"oracle {what}: invalid arguments")
    return rc


def num_threads() -> int:
    return lib().oracle_num_threads()


def set_num_threads(n: int) -> None:
    lib().oracle_set_num_threads(int(n))


def pool(hidden_bits: np.ndarray, n_pool: int = 100) -> np.ndarray:
    """Concatenated means of the first and last min(n_pool, T) rows, fp64 [2*Hd]."""
    h = np.ascontiguousarray(hidden_bits, dtype=np.uint16)
    T, Hd = h.shape
    p = np.empty(2 * Hd, np.float64)
    _check(lib().oracle_pool(h, T, Hd, n_pool, p), "pool")
    return p


def mlp(p, W1, b1, W2, b2) -> np.ndarray:
    """z = W2 relu(W1 p + b1) + b2 in fp64; weights fp32."""
    p = np.ascontiguousarray(p, np.float64)
    W1 = np.ascontiguousarray(W1, np.float32)
    W2 = np.ascontiguousarray(W2, np.float32)
    b1 = np.ascontiguousarray(b1, np.float32)
    b2 = np.ascontiguousarray(b2, np.float32)
    H1, L = W1.shape[0], W2.shape[0]
    assert W1.shape[1] == p.size and W2.shape[1] == H1
    z = np.empty(L, np.float64)
    _check(lib().oracle_mlp(p, p.size, W1, b1, H1, W2, b2, L, z), "mlp")
    return z


def threshold(z, thresh: float):
    """(mode uint8 [L], r = sigmoid(z) fp64 [L]); mode 1 = FA iff fp32(r) > thresh."""
    z = np.ascontiguousarray(z, np.float64)
    mode = np.empty(z.size, np.uint8)
    r = np.empty(z.size, np.float64)
    _check(lib().oracle_threshold(z, z.size, thresh, mode, _ptr(r)), "threshold")
    return mode, r


def route(hidden_bits, W1, b1, W2, b2, thresh: float, n_pool: int = 100):
    """Router end to end: (mode uint8 [L], z fp64 [L], r fp64 [L])."""
    h = np.ascontiguousarray(hidden_bits, np.uint16)
    T, Hd = h.shape
    W1 = np.ascontiguousarray(W1, np.float32)
    W2 = np.ascontiguousarray(W2, np.float32)
    b1 = np.ascontiguousarray(b1, np.float32)
    b2 = np.ascontiguousarray(b2, np.float32)
    H1, L = W1.shape[0], W2.shape[0]
    assert W1.shape[1] == 2 * Hd and W2.shape[1] == H1
    mode = np.empty(L, np.uint8)
    z = np.empty(L, np.float64)
    r = np.empty(L, np.float64)
    _check(lib().oracle_route(h, T, Hd, n_pool, W1, b1, H1, W2, b2, L, thresh, mode, _ptr(z),
                              _ptr(r)), "route")
    return mode, z, r


def streaming_mask(nqb: int, nkb: int, sink_blocks: int, window_blocks: int) -> np.ndarray:
    m = np.empty((nqb, nkb), np.uint8)
    _check(lib().oracle_streaming_mask(nqb, nkb, sink_blocks, window_blocks, m), "mask")
    return m


def block_index(mask: np.ndarray):
    """(row_ptr int32 [nqb+1], col int32 [nnz]) of the ascending kept kv blocks."""
    m = np.ascontiguousarray(mask, np.uint8)
    nqb, nkb = m.shape
    row_ptr = np.empty(nqb + 1, np.int32)
    col = np.empty(nqb * nkb, np.int32)
    nnz = _check(lib().oracle_block_index(m, nqb, nkb, row_ptr, col), "block_index")
    return row_ptr, col[:nnz].copy()


def attn_prefill(q, k, v, scale: float, block_mask=None, block: int = 0, rows=None):
    """Prefill attention in fp64.

    q: uint16 [B, T, Hq, d]; k, v: uint16 [B, T, Hkv, d] (bf16 bit patterns).
    block_mask: uint8 [nqb, nkb] (SA) or None (FA).  rows: int32 [n, 3] of
    (b, h, t) or None for all rows.  Returns (o, lse): with rows, o is
    [n, d] and lse [n]; without, o is [B, T, Hq, d] and lse [B, T, Hq].
    """
    q = np.ascontiguousarray(q, np.uint16)
    k = np.ascontiguousarray(k, np.uint16)
    v = np.ascontiguousarray(v, np.uint16)
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    assert k.shape == (B, T, Hkv, d) and v.shape == k.shape
    mask = None if block_mask is None else np.ascontiguousarray(block_mask, np.uint8)
    nkb = 0 if mask is None else mask.shape[1]
    if rows is not None:
        rows = np.ascontiguousarray(rows, np.int32).reshape(-1, 3)
        n = rows.shape[0]
    else:
        n = B * T * Hq
    o = np.empty((n, d), np.float64)
    lse = np.empty(n, np.float64)
    _check(lib().oracle_attn_prefill(q, k, v, B, T, Hq, Hkv, d, _ptr(mask), nkb, block, scale,
                                     _ptr(rows), n, o, _ptr(lse)), "attn_prefill")
    if rows is None:
        return o.reshape(B, T, Hq, d), lse.reshape(B, T, Hq)
    return o, lse


def attn_prefill_soft(q, k, v, scale: float, r: float, block_mask, block: int, rows=None):
    """Soft-routing blend r * FA + (1 - r) * SA in fp64; shapes as attn_prefill."""
    q = np.ascontiguousarray(q, np.uint16)
    k = np.ascontiguousarray(k, np.uint16)
    v = np.ascontiguousarray(v, np.uint16)
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    mask = np.ascontiguousarray(block_mask, np.uint8)
    if rows is not None:
        rows = np.ascontiguousarray(rows, np.int32).reshape(-1, 3)
        n = rows.shape[0]
    else:
        n = B * T * Hq
    o = np.empty((n, d), np.float64)
    _check(lib().oracle_attn_prefill_soft(q, k, v, B, T, Hq, Hkv, d, mask, mask.shape[1], block,
                                          scale, r, _ptr(rows), n, o), "attn_prefill_soft")
    return o if rows is not None else o.reshape(B, T, Hq, d)


def attn_probs(q, k, scale: float, b: int, h: int, block_mask=None, block: int = 0):
    """The full T x T probability matrix of head (b, h), fp64."""
    q = np.ascontiguousarray(q, np.uint16)
    k = np.ascontiguousarray(k, np.uint16)
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    mask = None if block_mask is None else np.ascontiguousarray(block_mask, np.uint8)
    nkb = 0 if mask is None else mask.shape[1]
    P = np.empty((T, T), np.float64)
    _check(lib().oracle_attn_probs(q, k, B, T, Hq, Hkv, d, _ptr(mask), nkb, block, scale, b, h, P),
           "attn_probs")
    return P


def attn_decode(q, k_cache, v_cache, seqlens, scale: float, mode: int, sink_blocks: int = 0,
                window_blocks: int = 1, block: int = 128):
    """Decode attention in fp64: q uint16 [B, Hq, d]; caches uint16 [B, S_max, Hkv, d].

    mode 1 = FA over u < s; mode 0 = SA over the sink and last-W blocks.
    Returns (o [B, Hq, d], lse [B, Hq]).
    """
    q = np.ascontiguousarray(q, np.uint16)
    kc = np.ascontiguousarray(k_cache, np.uint16)
    vc = np.ascontiguousarray(v_cache, np.uint16)
    sl = np.ascontiguousarray(seqlens, np.int32)
    B, Hq, d = q.shape
    _, S_max, Hkv, _ = kc.shape
    o = np.empty((B, Hq, d), np.float64)
    lse = np.empty((B, Hq), np.float64)
    _check(lib().oracle_attn_decode(q, kc, vc, S_max, sl, B, Hq, Hkv, d, int(mode), sink_blocks,
                                    window_blocks, block, scale, o, _ptr(lse)), "attn_decode")
    return o, lse


def block_scores(q, k, block: int, stride: int, scale: float) -> np.ndarray:
    """Dynamic SA block selection, step 1 (reading stated in flux_oracle.c):
    fp64 layer scores P [nb, nb] from strided antidiagonal logits; q uint16
    [B, T, Hq, d], k uint16 [B, T, Hkv, d].  Row i sums to 1 over j <= i.
    Parity unpinned against the pages."""
    q = np.ascontiguousarray(q, np.uint16)
    k = np.ascontiguousarray(k, np.uint16)
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    nr = (T + stride - 1) // stride
    R = block // stride
    nb = (nr + R - 1) // R
    P = np.zeros((nb, nb), np.float64)
    _check(lib().oracle_block_scores(q, k, B, T, Hq, Hkv, d, block, stride, scale, P),
           "block_scores")
    return P


def block_scores_rows(q, k, block: int, stride: int, scale: float, rows) -> np.ndarray:
    """The rows of block_scores for the query blocks listed in ``rows`` only:
    fp64 [len(rows), nb], row n = query block rows[n] (a query block's row
    depends on its own queries alone).  Parity unpinned against the pages."""
    q = np.ascontiguousarray(q, np.uint16)
    k = np.ascontiguousarray(k, np.uint16)
    rows = np.ascontiguousarray(rows, np.int32)
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    nr = (T + stride - 1) // stride
    R = block // stride
    nb = (nr + R - 1) // R
    P = np.zeros((len(rows), nb), np.float64)
    _check(lib().oracle_block_scores_rows(q, k, B, T, Hq, Hkv, d, block, stride, scale, rows,
                                          len(rows), P), "block_scores_rows")
    return P


def select_blocks(P, tau: float, sink_blocks: int) -> np.ndarray:
    """Dynamic SA block selection, step 2: the block mask uint8 [nb, nb] kept
    from fp32 scores P (an fp64 P is rounded to fp32 first).  Parity unpinned
    against the pages."""
    P32 = np.ascontiguousarray(P, np.float32)
    nb = P32.shape[0]
    mask = np.zeros((nb, nb), np.uint8)
    _check(lib().oracle_select_blocks(P32, nb, float(tau), int(sink_blocks), mask),
           "select_blocks")
    return mask
