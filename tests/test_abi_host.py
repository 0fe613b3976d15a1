"""Host-only checks of the C ABI (no GPU): the library loads, exports every function that
include/e2d2_attn.h declares, and rejects bad arguments with the documented status before
touching the GPU."""
import ctypes
import re
from pathlib import Path

import pytest

from block_discrete_diffusion_tcgen05_b200 import _lib, build

ROOT = Path(__file__).resolve().parents[1]
HEADER = ROOT / "include" / "e2d2_attn.h"


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def header_functions():
    text = HEADER.read_text()
    return re.findall(r"E2D2_API\s+[\w\s\*]+?\b(e2d2_\w+)\s*\(", text)


def test_header_declares_the_boundary():
    names = set(header_functions())
    assert {"e2d2_attn_encoder_blockcausal", "e2d2_attn_decoder_train", "e2d2_attn_decoder_sample",
            "e2d2_kv_cache_append", "e2d2_attn_decoder_sample_workspace", "e2d2_attn_encoder_block_step",
            "e2d2_attn_train_backward_workspace", "e2d2_attn_encoder_backward",
            "e2d2_attn_decoder_train_backward"} <= names


def test_library_exports_every_declared_symbol(lib):
    for name in header_functions():
        assert hasattr(lib, name), name
    assert set(_lib.EXPORTS) <= set(header_functions())


def test_status_strings(lib):
    for code, name in _lib.STATUS.items():
        assert lib.e2d2_status_string(code).decode() == name
    assert lib.e2d2_version() == 100


DIMS = _lib.Dims(2, 4, 2, 64, 0.0)
P16 = 0x10000  # fake 16-byte aligned addresses; validation must fail before any use


def test_encoder_argument_errors(lib):
    f = lib.e2d2_attn_encoder_blockcausal
    assert f(None, P16, P16, P16, None, DIMS, 64, 8, None) == 1          # null q
    assert f(P16, P16, P16, P16, None, _lib.Dims(2, 4, 2, 96, 0.0), 64, 8, None) == 2  # head_dim
    assert f(P16, P16, P16, P16, None, _lib.Dims(2, 4, 3, 64, 0.0), 64, 8, None) == 1  # GQA ratio
    assert f(P16, P16, P16, P16, None, _lib.Dims(0, 4, 2, 64, 0.0), 64, 8, None) == 1  # batch
    # S need not divide L (short last block) and may exceed L (one block): such calls get past
    # the shape checks to the alignment check (a misaligned lse keeps them from launching)
    for L, S in ((60, 8), (8, 16)):
        assert f(P16, P16, P16, P16, P16 + 2, DIMS, L, S, None) == 4
    assert f(P16, P16, P16, P16, None, DIMS, 64, 0, None) == 1           # S = 0
    assert f(P16, P16, P16, P16, None, DIMS, 0, 8, None) == 1            # L = 0
    assert f(P16 + 8, P16, P16, P16, None, DIMS, 64, 8, None) == 4       # misaligned q
    assert f(P16, P16, P16, P16, P16 + 2, DIMS, 64, 8, None) == 4        # misaligned lse
    assert f(P16, P16, P16, P16, None, _lib.Dims(2, 4, 2, 64, float("nan")), 64, 8, None) == 1


def test_decoder_train_argument_errors(lib):
    f = lib.e2d2_attn_decoder_train
    assert f(P16, P16, P16, None, P16, P16, None, DIMS, 64, 8, None) == 1
    assert f(P16, P16, P16, P16, P16 + 4, P16, None, DIMS, 64, 8, None) == 4
    assert f(P16, P16, P16, P16, P16, P16, None, DIMS, 64, -1, None) == 1


def test_encoder_block_step_argument_errors(lib):
    f = lib.e2d2_attn_encoder_block_step
    ws = 1 << 20
    # (q, k_cache, v_cache, capacity, P, k_blk, v_blk, out, lse, dims, S, workspace, ws_bytes, stream)
    assert f(P16, P16, P16, 20, 10, P16, P16, P16, None, DIMS, 16, P16, ws, None) == 5  # P + S > capacity
    assert f(P16, P16, P16, 20, 21, P16, P16, P16, None, DIMS, 16, P16, ws, None) == 5  # P > capacity
    assert f(P16, None, P16, 64, 0, P16, P16, P16, None, DIMS, 16, P16, ws, None) == 1  # null cache


def test_train_backward_workspace_query_needs_no_gpu(lib):
    # two floats (D_i and the scaled lse) per query row, rows padded to a multiple of 128
    assert lib.e2d2_attn_train_backward_workspace(DIMS, 64) == 2 * 2 * 4 * 128 * 4
    assert lib.e2d2_attn_train_backward_workspace(DIMS, 129) == 2 * 2 * 4 * 256 * 4
    assert lib.e2d2_attn_train_backward_workspace(_lib.Dims(2, 4, 2, 96, 0.0), 64) == 0
    assert lib.e2d2_attn_train_backward_workspace(DIMS, 0) == 0


def test_encoder_backward_argument_errors(lib):
    f = lib.e2d2_attn_encoder_backward
    ws = lib.e2d2_attn_train_backward_workspace(DIMS, 64)
    # (q, k, v, out, lse, dout, dq, dk, dv, dims, L, S, workspace, ws_bytes, stream)
    a = [P16] * 9
    assert f(*a[:4], None, *a[5:], DIMS, 64, 8, P16, ws, None) == 1                 # lse is required
    assert f(*a[:3], None, *a[4:], DIMS, 64, 8, P16, ws, None) == 1                 # out is required
    assert f(*a[:8], None, DIMS, 64, 8, P16, ws, None) == 1                         # null dv
    assert f(*a, DIMS, 64, 8, P16, ws - 1, None) == 6                               # small workspace
    assert f(*a, DIMS, 64, 8, None, ws, None) == 6                                  # no workspace
    assert f(P16 + 8, *a[1:], DIMS, 64, 8, P16, ws, None) == 4                      # misaligned q
    assert f(*a[:3], P16 + 8, *a[4:], DIMS, 64, 8, P16, ws, None) == 4              # misaligned out
    assert f(*a[:4], P16 + 2, *a[5:], DIMS, 64, 8, P16, ws, None) == 4              # misaligned lse
    assert f(*a, DIMS, 64, 8, P16 + 4, ws, None) == 4                               # misaligned workspace
    assert f(*a, DIMS, 64, 0, P16, ws, None) == 1                                   # S = 0
    assert f(*a, _lib.Dims(2, 4, 2, 96, 0.0), 64, 8, P16, ws, None) == 2            # head_dim
    assert f(*a, _lib.Dims(2, 4, 3, 64, 0.0), 64, 8, P16, ws, None) == 1            # GQA ratio
    # a short last block passes the shape checks (stopped here by the misaligned lse)
    assert f(*a[:4], P16 + 2, *a[5:], DIMS, 60, 8, P16, ws, None) == 4


def test_decoder_train_backward_argument_errors(lib):
    f = lib.e2d2_attn_decoder_train_backward
    ws = lib.e2d2_attn_train_backward_workspace(DIMS, 64)
    # (q, k_enc, v_enc, k_dec, v_dec, out, lse, dout, dq, dk_enc, dv_enc, dk_dec, dv_dec, dims, L, S,
    #  workspace, ws_bytes, stream)
    a = [P16] * 13
    assert f(*a[:12], None, DIMS, 64, 8, P16, ws, None) == 1                        # null dv_dec
    assert f(*a[:6], None, *a[7:], DIMS, 64, 8, P16, ws, None) == 1                 # lse is required
    assert f(*a[:5], None, *a[6:], DIMS, 64, 8, P16, ws, None) == 1                 # out is required
    assert f(*a[:11], P16 + 8, a[12], DIMS, 64, 8, P16, ws, None) == 4              # misaligned dk_dec
    assert f(*a, DIMS, 64, 8, P16, ws - 4, None) == 6
    assert f(*a, DIMS, -1, 8, P16, ws, None) == 1


def test_sample_workspace_query_needs_no_gpu(lib):
    n = lib.e2d2_attn_decoder_sample_workspace(_lib.Dims(32, 16, 8, 128, 0.0), 16, 2064)
    assert n > 0
    assert lib.e2d2_attn_decoder_sample_workspace(_lib.Dims(32, 16, 8, 96, 0.0), 16, 2064) == 0


def test_sample_argument_errors(lib):
    f = lib.e2d2_attn_decoder_sample
    dm = _lib.Dims(2, 4, 2, 128, 0.0)
    ws = lib.e2d2_attn_decoder_sample_workspace(dm, 16, 64)
    assert f(P16, P16, P16, 64, 65, P16, P16, P16, None, dm, 16, P16, ws, None) == 5   # P > capacity
    assert f(P16, P16, P16, 64, 32, P16, P16, P16, None, dm, 16, None, ws, None) == 6  # no workspace
    assert f(P16, P16, P16, 64, 32, P16, P16, P16, None, dm, 16, P16, ws - 1, None) == 6
    assert f(P16, P16, P16, 64, -1, P16, P16, P16, None, dm, 16, P16, ws, None) == 1
    assert f(P16, P16, P16 + 8, 64, 32, P16, P16, P16, None, dm, 16, P16, ws, None) == 4
    assert f(P16, P16, P16, 64, 32, P16, P16, None, None, dm, 16, P16, ws, None) == 1


def test_append_argument_errors(lib):
    f = lib.e2d2_kv_cache_append
    dm = _lib.Dims(2, 2, 2, 64, 0.0)
    assert f(P16, P16, 32, 30, P16, P16, 4, dm, None) == 5
    assert f(P16, None, 32, 0, P16, P16, 4, dm, None) == 1
    assert f(P16, P16, 32, 0, P16 + 2, P16, 4, dm, None) == 4
    assert f(P16, P16, 32, 0, P16, P16, 0, dm, None) == 0  # nothing to copy: no launch


def test_product_package_never_imports_the_oracle():
    pkg = ROOT / "block_discrete_diffusion_tcgen05_b200"
    for p in pkg.rglob("*.py"):
        src = p.read_text()
        assert "import oracle" not in src and "from oracle" not in src, p
    for p in (ROOT / "oracle").rglob("*.py"):
        src = p.read_text()
        assert "import block_discrete_diffusion_tcgen05_b200" not in src, p
        assert "from block_discrete_diffusion_tcgen05_b200" not in src, p


def test_ragged_sample_argument_errors(lib):
    f = lib.e2d2_attn_decoder_sample_ragged
    dims = _lib.Dims(2, 4, 2, 128, 0.0)
    ws = lib.e2d2_attn_decoder_sample_workspace(dims, 16, 64)
    # (q_blk, k_cache, v_cache, capacity, P_dev, k_blk, v_blk, out, lse, dims, S, workspace, ws_bytes, stream)
    assert f(P16, P16, P16, 64, None, P16, P16, P16, None, dims, 16, P16, ws, None) == 1       # P is required
    assert f(P16, P16, P16, 64, P16 + 2, P16, P16, P16, None, dims, 16, P16, ws, None) == 4   # misaligned P
    assert f(P16, P16, P16, 64, P16, P16, P16, P16, None, _lib.Dims(257, 4, 2, 128, 0.0), 16, P16, ws, None) == 3
    assert f(P16, None, P16, 64, P16, P16, P16, P16, None, dims, 16, P16, ws, None) == 1      # null cache
    assert f(P16, P16, P16, 64, P16, P16, P16, P16, None, dims, 16, P16, ws - 1, None) == 6   # small workspace
    assert f(P16, P16, P16, -1, P16, P16, P16, P16, None, dims, 16, P16, ws, None) == 1       # capacity < 0


def test_debug_library_exports_every_declared_symbol():
    """The E2D2_DEBUG build (device-side bounds checks) has the same C ABI."""
    dbg = _lib.load(build.build(debug=True))
    for name in header_functions():
        assert hasattr(dbg, name), name
    dbg.e2d2_status_string.restype = ctypes.c_char_p
    assert dbg.e2d2_status_string(9) == b"E2D2_ERR_DEVICE_CHECK"


def test_status_strings_cover_every_status(lib):
    for code, name in _lib.STATUS.items():
        assert lib.e2d2_status_string(code).decode() == name


def test_ragged_append_argument_errors(lib):
    f = lib.e2d2_kv_cache_append_ragged
    dims = _lib.Dims(2, 2, 2, 128, 0.0)
    # (k_cache, v_cache, capacity, P_dev, k_new, v_new, S_new, dims, stream)
    assert f(P16, P16, 64, None, P16, P16, 16, dims, None) == 1        # P is required
    assert f(P16, P16, 64, P16 + 2, P16, P16, 16, dims, None) == 4     # misaligned P
    assert f(P16, P16, 64, P16, P16 + 8, P16, 16, dims, None) == 4     # misaligned rows
    assert f(P16, P16, 8, P16, P16, P16, 16, dims, None) == 5          # S_new > capacity
    assert f(P16, P16, 64, P16, P16, P16, -1, dims, None) == 1
    assert f(P16, P16, 64, P16, P16, P16, 0, dims, None) == 0          # nothing to append

