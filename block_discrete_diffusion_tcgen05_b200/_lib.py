"""ctypes loader for the in-tree CUDA library ``libe2d2_attn.so`` (the C ABI of
include/e2d2_attn.h).  Argument marshalling only; there is no fallback of any kind: if the
library is missing, importing the attention calls fails loudly."""
from __future__ import annotations

import ctypes
import os
from pathlib import Path

PKG = Path(__file__).resolve().parent
LIBRARY = PKG / "libe2d2_attn.so"
# E2D2_DEBUG=1 selects the build with device-side bounds checks (E2D2_ERR_DEVICE_CHECK)
DEBUG_LIBRARY = PKG / "libe2d2_attn_debug.so"

# Names and values of include/e2d2_attn.h's e2d2_status.
STATUS = {0: "E2D2_OK", 1: "E2D2_ERR_INVALID_ARG", 2: "E2D2_ERR_UNSUPPORTED", 3: "E2D2_ERR_SHAPE",
          4: "E2D2_ERR_ALIGNMENT", 5: "E2D2_ERR_CAPACITY", 6: "E2D2_ERR_WORKSPACE",
          7: "E2D2_ERR_CUDA", 8: "E2D2_ERR_TIMEOUT", 9: "E2D2_ERR_DEVICE_CHECK"}

EXPORTS = ("e2d2_attn_encoder_blockcausal", "e2d2_attn_decoder_train",
           "e2d2_attn_decoder_sample_workspace", "e2d2_attn_decoder_sample",
           "e2d2_kv_cache_append", "e2d2_status_string", "e2d2_last_device_error", "e2d2_version",
           "e2d2_attn_decoder_sample_noalloc", "e2d2_attn_encoder_block_step",
           "e2d2_attn_train_backward_workspace", "e2d2_attn_encoder_backward",
           "e2d2_attn_decoder_train_backward", "e2d2_attn_decoder_sample_plan", "e2d2_attn_train_order",
           "e2d2_attn_decoder_sample_ragged", "e2d2_attn_decoder_sample_ragged_plan",
           "e2d2_debug_set_wait_test", "e2d2_kv_cache_append_ragged")

# E2D2_SAMPLE_NOALLOC_MAX_BYTES of include/e2d2_attn.h
SAMPLE_NOALLOC_MAX_BYTES = 32 << 20


class Dims(ctypes.Structure):
    """e2d2_dims."""

    _fields_ = [("batch", ctypes.c_int), ("q_heads", ctypes.c_int), ("kv_heads", ctypes.c_int),
                ("head_dim", ctypes.c_int), ("scale", ctypes.c_float)]


class SamplePlan(ctypes.Structure):
    """e2d2_sample_plan."""

    _fields_ = [("kernel", ctypes.c_int), ("units", ctypes.c_int), ("tiles_per_unit", ctypes.c_int),
                ("split_units", ctypes.c_int), ("split_ctas", ctypes.c_int), ("whole_units", ctypes.c_int),
                ("grid", ctypes.c_int)]


class RaggedPlan(ctypes.Structure):
    """e2d2_ragged_plan."""

    _fields_ = [("kernel", ctypes.c_int), ("units", ctypes.c_int), ("units_per_entry", ctypes.c_int),
                ("total_tiles", ctypes.c_longlong), ("grid", ctypes.c_int), ("stream_ctas", ctypes.c_int)]


class E2D2Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


_lib = None


def load(path: Path | str | None = None):
    """Load the library (once).  Raises if it has not been built."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    if path is not None:
        p = Path(path)
    else:
        p = DEBUG_LIBRARY if os.environ.get("E2D2_DEBUG", "0") not in ("", "0") else LIBRARY
    if not p.exists():
        raise ImportError(f"{p} is missing: build it with `python -m block_discrete_diffusion_tcgen05_b200.build`"
                          " (or __graft_entry__.build()); there is no CPU fallback")
    lib = ctypes.CDLL(str(p))
    vp, ci, st = ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p
    fp = ctypes.c_void_p
    lib.e2d2_attn_encoder_blockcausal.argtypes = [vp, vp, vp, vp, fp, Dims, ci, ci, st]
    lib.e2d2_attn_decoder_train.argtypes = [vp, vp, vp, vp, vp, vp, fp, Dims, ci, ci, st]
    lib.e2d2_attn_decoder_sample_workspace.argtypes = [Dims, ci, ci]
    lib.e2d2_attn_decoder_sample_workspace.restype = ctypes.c_size_t
    lib.e2d2_attn_decoder_sample.argtypes = [vp, vp, vp, ci, ci, vp, vp, vp, fp, Dims, ci, vp,
                                             ctypes.c_size_t, st]
    lib.e2d2_kv_cache_append.argtypes = [vp, vp, ci, ci, vp, vp, ci, Dims, st]
    lib.e2d2_kv_cache_append_ragged.argtypes = [vp, vp, ci, vp, vp, vp, ci, Dims, st]
    lib.e2d2_kv_cache_append_ragged.restype = ctypes.c_int
    lib.e2d2_attn_encoder_block_step.argtypes = [vp, vp, vp, ci, ci, vp, vp, vp, fp, Dims, ci, vp,
                                                 ctypes.c_size_t, st]
    lib.e2d2_attn_decoder_sample_noalloc.argtypes = [vp, vp, vp, ci, ci, vp, vp, vp, fp, Dims, ci, st]
    lib.e2d2_attn_decoder_sample_noalloc.restype = ctypes.c_int
    lib.e2d2_attn_train_backward_workspace.argtypes = [Dims, ci]
    lib.e2d2_attn_train_backward_workspace.restype = ctypes.c_size_t
    lib.e2d2_attn_encoder_backward.argtypes = [vp, vp, vp, vp, fp, vp, vp, vp, vp, Dims, ci, ci, vp,
                                               ctypes.c_size_t, st]
    lib.e2d2_attn_decoder_train_backward.argtypes = [vp, vp, vp, vp, vp, vp, fp, vp, vp, vp, vp, vp, vp,
                                                     Dims, ci, ci, vp, ctypes.c_size_t, st]
    lib.e2d2_attn_decoder_sample_plan.argtypes = [Dims, ci, ci, ci, ctypes.POINTER(SamplePlan)]
    lib.e2d2_attn_decoder_sample_plan.restype = ctypes.c_int
    pi = ctypes.POINTER(ctypes.c_int)
    lib.e2d2_attn_train_order.argtypes = [ci, Dims, ci, ci, ci, pi, pi, pi, pi]
    lib.e2d2_attn_train_order.restype = ctypes.c_int
    lib.e2d2_attn_decoder_sample_ragged.argtypes = [vp, vp, vp, ci, vp, vp, vp, vp, fp, Dims, ci, vp,
                                                    ctypes.c_size_t, st]
    lib.e2d2_attn_decoder_sample_ragged.restype = ctypes.c_int
    lib.e2d2_attn_decoder_sample_ragged_plan.argtypes = [Dims, ci, ctypes.POINTER(ctypes.c_int), ci, ci,
                                                         ctypes.POINTER(RaggedPlan)]
    lib.e2d2_attn_decoder_sample_ragged_plan.restype = ctypes.c_int
    lib.e2d2_status_string.argtypes = [ci]
    lib.e2d2_status_string.restype = ctypes.c_char_p
    lib.e2d2_last_device_error.argtypes = [st]
    lib.e2d2_debug_set_wait_test.argtypes = [ctypes.c_ulonglong, ctypes.c_ulonglong]
    lib.e2d2_debug_set_wait_test.restype = ctypes.c_int
    for name in ("e2d2_attn_encoder_blockcausal", "e2d2_attn_decoder_train",
                 "e2d2_attn_decoder_sample", "e2d2_kv_cache_append", "e2d2_last_device_error",
                 "e2d2_version", "e2d2_attn_encoder_backward", "e2d2_attn_decoder_train_backward"):
        getattr(lib, name).restype = ctypes.c_int
    if path is None:
        _lib = lib
    return lib


def check(status: int, where: str) -> None:
    if status != 0:
        raise E2D2Error(status, where)
