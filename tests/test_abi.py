"""The C-ABI library: it loads, exports every symbol include/flux.h declares,
and rejects bad arguments on the host before any launch (no GPU needed)."""
import ctypes
import os

import pytest

from sparse_attention_flux_b200 import build, flux


@pytest.fixture(scope="module")
def lib():
    build.build(quiet=True)
    return flux.lib()


def test_header_declares_the_hot_path_entry_points():
    names = flux.header_symbols()
    for must in ("flux_route", "flux_build_streaming_mask", "flux_build_block_index",
                 "flux_attn_prefill", "flux_attn_decode", "flux_ctx_create", "flux_ctx_destroy",
                 "flux_ctx_check", "flux_last_error"):
        assert must in names


def test_library_exports_every_declared_symbol(lib):
    for name in flux.header_symbols():
        assert hasattr(lib, name), f"libflux.so does not export {name}"


def test_binding_covers_every_declared_symbol():
    assert set(flux.header_symbols()) <= set(flux._SIGNATURES)


def test_library_is_built_for_sm100a_and_in_tree(lib):
    assert os.path.dirname(flux.LIB_PATH) == os.path.dirname(os.path.abspath(flux.__file__))
    assert lib.flux_version() == 1


def test_host_side_argument_checks_need_no_gpu(lib):
    # Null pointers and bad sizes are rejected before any CUDA call.
    assert lib.flux_build_streaming_mask(4, 4, 1, 2, None, None) == flux.FLUX_ERR_INVALID_ARG
    assert b"null" in lib.flux_last_error()
    assert lib.flux_build_streaming_mask(4, 4, 1, 0, ctypes.c_void_p(16), None) == \
        flux.FLUX_ERR_INVALID_ARG
    assert lib.flux_route(None, None, 1, 1, 1, None, None, 1, None, None, 1, 0.5, None, None,
                          None) == flux.FLUX_ERR_INVALID_ARG
    assert lib.flux_attn_prefill(None, None, None, None, None, None, 1, 1, 1, 1, 128, None, 0,
                                 None, None, 0, 128, 0.1, None) == flux.FLUX_ERR_INVALID_ARG
    assert lib.flux_attn_decode(None, None, None, None, 1, None, None, None, 1, 1, 1, 128, None,
                                0, 1, 1, 128, 0.1, None) == flux.FLUX_ERR_INVALID_ARG
    assert lib.flux_ctx_destroy(None) == flux.FLUX_ERR_INVALID_ARG
    assert lib.flux_ctx_check(None, None) == flux.FLUX_ERR_INVALID_ARG


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(flux, "LIB_PATH", str(tmp_path / "libflux.so"))
    monkeypatch.setattr(flux, "_lib", None)
    with pytest.raises(RuntimeError, match="no CPU fallback"):
        flux.lib()


def test_decode_family_host_checks_need_no_gpu(lib):
    """The decode entry points share one set of host checks: each rejects a null context or
    tensor, an unsupported group size, a ring of the wrong size, a bad scale or too many
    (sequence, kv head) groups before any CUDA call."""
    P = ctypes.c_void_p(256)                      # aligned, never dereferenced
    ctx = ctypes.c_void_p(4096)                   # never dereferenced: checks fail first
    # flux_attn_decode: null context
    assert lib.flux_attn_decode(None, P, P, P, 64, P, P, None, 1, 2, 1, 64, None, 0, 1, 1, 64,
                                0.1, None) == flux.FLUX_ERR_INVALID_ARG
    assert b"null" in lib.flux_last_error()
    # group sizes above 8 (and Hq not a multiple of Hkv) are not supported
    assert lib.flux_attn_decode(ctx, P, P, P, 64, P, P, None, 1, 9, 1, 64, None, 0, 1, 1, 64,
                                0.1, None) == flux.FLUX_ERR_UNSUPPORTED
    assert b"1 to 8" in lib.flux_last_error()
    assert lib.flux_attn_decode(ctx, P, P, P, 64, P, P, None, 1, 6, 4, 64, None, 0, 1, 1, 64,
                                0.1, None) == flux.FLUX_ERR_UNSUPPORTED
    # non-finite scale
    assert lib.flux_attn_decode_heads(ctx, P, P, P, 64, P, P, None, 1, 2, 1, 64, P, 1, 1, 64,
                                      float("nan"), None) == flux.FLUX_ERR_INVALID_ARG
    # fused append: ring rows must be (sink + window) * block
    assert lib.flux_attn_decode_append(ctx, P, P, P, P, P, 100, P, P, None, 1, 2, 1, 64, None, 0,
                                       1, 1, 64, 1, 0.1, None) == flux.FLUX_ERR_SHAPE
    assert lib.flux_attn_decode_append(ctx, P, None, P, P, P, 128, P, P, None, 1, 2, 1, 64, None,
                                       0, 1, 1, 64, 1, 0.1, None) == flux.FLUX_ERR_INVALID_ARG
    # compact ring decode: block must be a multiple of 64
    assert lib.flux_attn_decode_sa_compact(ctx, P, P, P, P, P, None, 1, 2, 1, 64, 1, 1, 96, 0.1,
                                           None) == flux.FLUX_ERR_UNSUPPORTED
    # no-allocation decode: at most 4096 (sequence, kv head) groups
    assert lib.flux_attn_decode_noalloc(P, P, P, 64, P, P, None, 8192, 2, 1, 64, None, 0, 1, 1,
                                        64, 0.1, None, None) == flux.FLUX_ERR_SHAPE
    assert b"4096" in lib.flux_last_error()
    # misaligned cache pointer
    assert lib.flux_attn_decode(ctx, P, ctypes.c_void_p(258), P, 64, P, P, None, 1, 2, 1, 64,
                                None, 0, 1, 1, 64, 0.1, None) == flux.FLUX_ERR_INVALID_ARG


def test_select_blocks_host_checks_need_no_gpu(lib):
    """flux_select_blocks rejects bad arguments before any CUDA call."""
    P = ctypes.c_void_p(256)
    ctx = ctypes.c_void_p(4096)   # never dereferenced: the checks fail first
    M = ctypes.c_void_p(512)
    f = lib.flux_select_blocks
    assert f(None, P, P, 1, 256, 2, 1, 64, 128, 8, 0.125, 0.9, 0, M, None, None) == \
        flux.FLUX_ERR_INVALID_ARG
    assert f(ctx, P, P, 1, 256, 2, 1, 96, 128, 8, 0.125, 0.9, 0, M, None, None) == \
        flux.FLUX_ERR_UNSUPPORTED
    assert f(ctx, P, P, 1, 256, 2, 1, 64, 64, 8, 0.125, 0.9, 0, M, None, None) == \
        flux.FLUX_ERR_UNSUPPORTED
    assert f(ctx, P, P, 1, 256, 2, 1, 64, 128, 16, 0.125, 0.9, 0, M, None, None) == \
        flux.FLUX_ERR_UNSUPPORTED
    assert f(ctx, P, P, 1, 200000, 2, 1, 64, 128, 8, 0.125, 0.9, 0, M, None, None) == \
        flux.FLUX_ERR_UNSUPPORTED
    assert f(ctx, P, P, 1, 131073, 2, 1, 64, 128, 8, 0.125, 0.9, 0, M, None, None) == \
        flux.FLUX_ERR_UNSUPPORTED   # 1025 blocks: one past the largest layer
    assert f(ctx, P, P, 1, 256, 3, 2, 64, 128, 8, 0.125, 0.9, 0, M, None, None) == \
        flux.FLUX_ERR_UNSUPPORTED
    assert f(ctx, P, P, 1, 256, 2, 1, 64, 128, 8, float("nan"), 0.9, 0, M, None, None) == \
        flux.FLUX_ERR_INVALID_ARG
    assert f(ctx, P, P, 1, 256, 2, 1, 64, 128, 8, 0.125, -0.5, 0, M, None, None) == \
        flux.FLUX_ERR_INVALID_ARG
    assert f(ctx, ctypes.c_void_p(258), P, 1, 256, 2, 1, 64, 128, 8, 0.125, 0.9, 0, M, None,
             None) == flux.FLUX_ERR_INVALID_ARG
    # workspace: B * Hkv * nb * nb floats (4 query heads per CTA here)
    nb = 32768 // 128
    assert lib.flux_select_blocks_workspace_bytes(1, 32768, 32, 8, 8) == 8 * nb * nb * 4
    assert lib.flux_select_blocks_workspace_bytes(1, 256, 3, 2, 8) == 0
    assert lib.flux_select_blocks_workspace_bytes(1, 131073, 4, 1, 8) == 0   # above the largest
    assert lib.flux_select_blocks_workspace_bytes(1, 131072, 4, 1, 8) == 1024 * 1024 * 4
