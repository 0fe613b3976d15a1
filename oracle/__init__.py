"""Plain CPU oracle for the E2D2 fused block-diffusion attention.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline / reference legs of ``bench.py`` may import this package.  The product
path (``block_discrete_diffusion_tcgen05_b200``) never imports it, and this package never
imports the product package: the two share no code.

The arithmetic lives in ``e2d2_oracle.c`` (fp64, explicit boolean masks, one query at a
time).  This module only compiles it with gcc, loads it with ctypes and marshals numpy
arrays.  What each function computes, and which passage of the pages it follows, is
written beside the C function.

Parity pins (tests/test_oracle_pins.py) tie every function here to facts that do not come
from this code: the pair count of the FLOPs table of "Encoder-Decoder Diffusion Language
Models for Efficient Training and Inference" (paper notes, sec. 4), the block-size limits
of "Block Diffusion: Interpolating Between Autoregressive and Diffusion Language Models"
(sec. 2: block size 1 is autoregressive, block size L is full diffusion) checked against
torch's own attention routine, closed forms, and a separately written brute force.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
SOURCE = _HERE / "e2d2_oracle.c"
LIBRARY = _HERE / "liboracle_e2d2.so"

_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)
_u8p = ctypes.POINTER(ctypes.c_uint8)
_u16p = ctypes.POINTER(ctypes.c_uint16)


def build(source: Path = SOURCE, output: Path = LIBRARY, extra_flags=()) -> Path:
    """Compile the oracle with gcc (-O2, OpenMP, strict IEEE: no -ffast-math)."""
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", *extra_flags,
           str(source), "-o", str(output), "-lm"]
    subprocess.run(cmd, check=True)
    return output


def _needs_build(lib: Path, src: Path) -> bool:
    return (not lib.exists()) or lib.stat().st_mtime < src.stat().st_mtime


class Oracle:
    """ctypes front-end of one compiled oracle library."""

    def __init__(self, path: Path | str | None = None):
        if path is None:
            if _needs_build(LIBRARY, SOURCE):
                build()
            path = LIBRARY
        self.path = Path(path)
        lib = ctypes.CDLL(str(self.path))
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_set_num_threads.argtypes = [ctypes.c_int]
        lib.oracle_set_num_threads.restype = None
        for name in ("oracle_mask_encoder", "oracle_mask_decoder", "oracle_mask_bd3lm"):
            getattr(lib, name).argtypes = [ctypes.c_int, ctypes.c_int, _u8p]
        lib.oracle_mask_sample.argtypes = [ctypes.c_int, ctypes.c_int, _u8p]
        ii = ctypes.c_int
        lib.oracle_encoder.argtypes = [_f32p, _f32p, _f32p, ii, ii, ii, ii, ii, ii,
                                       ctypes.c_double, _f64p, _f64p]
        lib.oracle_decoder_train.argtypes = [_f32p] * 5 + [ii] * 6 + [ctypes.c_double, _f64p, _f64p]
        lib.oracle_bd3lm_train.argtypes = [_f32p] * 3 + [ii] * 6 + [ctypes.c_double, _f64p, _f64p]
        lib.oracle_decoder_sample.argtypes = [_f32p, _f32p, _f32p, ii, ii, _f32p, _f32p,
                                              ii, ii, ii, ii, ii, ctypes.c_double, _f64p, _f64p]
        lib.oracle_decoder_sample_ragged.argtypes = [_f32p, _f32p, _f32p, ii, ctypes.POINTER(ctypes.c_int),
                                                     _f32p, _f32p, ii, ii, ii, ii, ii, ctypes.c_double,
                                                     _f64p, _f64p]
        lib.oracle_kv_append.argtypes = [_u16p, _u16p, ii, ii, _u16p, _u16p, ii, ii, ii, ii]
        lib.oracle_encoder_backward.argtypes = [_f32p] * 4 + [ii] * 6 + [ctypes.c_double] + [_f64p] * 3
        lib.oracle_decoder_train_backward.argtypes = [_f32p] * 6 + [ii] * 6 + [ctypes.c_double] + [_f64p] * 5
        for name in ("oracle_encoder", "oracle_decoder_train", "oracle_bd3lm_train", "oracle_decoder_sample",
                     "oracle_kv_append", "oracle_encoder_backward", "oracle_decoder_train_backward",
                     "oracle_decoder_sample_ragged"):
            getattr(lib, name).restype = ctypes.c_int
        self.lib = lib

    # ---- helpers -----------------------------------------------------------------
    @staticmethod
    def _f32(a):
        a = np.ascontiguousarray(a, dtype=np.float32)
        return a, a.ctypes.data_as(_f32p)

    def num_threads(self) -> int:
        return int(self.lib.oracle_num_threads())

    def set_num_threads(self, n: int) -> None:
        self.lib.oracle_set_num_threads(int(n))

    # ---- masks -------------------------------------------------------------------
    def mask_encoder(self, L: int, S: int) -> np.ndarray:
        m = np.zeros((L, L), dtype=np.uint8)
        self.lib.oracle_mask_encoder(L, S, m.ctypes.data_as(_u8p))
        return m.astype(bool)

    def mask_decoder(self, L: int, S: int) -> np.ndarray:
        m = np.zeros((L, 2 * L), dtype=np.uint8)
        self.lib.oracle_mask_decoder(L, S, m.ctypes.data_as(_u8p))
        return m.astype(bool)

    def mask_bd3lm(self, L: int, S: int) -> np.ndarray:
        """BD3LM's [2L, 2L] training mask (noised positions first, then clean)."""
        m = np.zeros((2 * L, 2 * L), dtype=np.uint8)
        self.lib.oracle_mask_bd3lm(L, S, m.ctypes.data_as(_u8p))
        return m.astype(bool)

    def mask_sample(self, S: int, P: int) -> np.ndarray:
        m = np.zeros((S, P + S), dtype=np.uint8)
        self.lib.oracle_mask_sample(S, P, m.ctypes.data_as(_u8p))
        return m.astype(bool)

    # ---- attention ---------------------------------------------------------------
    def encoder(self, q, k, v, S: int, scale: float = 0.0):
        """q [B,Hq,L,d], k/v [B,Hkv,L,d] -> (out [B,Hq,L,d] f64, lse [B,Hq,L] f64)."""
        B, Hq, L, d = q.shape
        Hkv = k.shape[1]
        assert k.shape == (B, Hkv, L, d) and v.shape == k.shape
        q, qp = self._f32(q)
        k, kp = self._f32(k)
        v, vp = self._f32(v)
        out = np.zeros((B, Hq, L, d), dtype=np.float64)
        lse = np.zeros((B, Hq, L), dtype=np.float64)
        rc = self.lib.oracle_encoder(qp, kp, vp, B, Hq, Hkv, L, S, d, float(scale),
                                     out.ctypes.data_as(_f64p), lse.ctypes.data_as(_f64p))
        if rc:
            raise RuntimeError(f"oracle_encoder failed ({rc})")
        return out, lse

    def decoder_train(self, q, k_enc, v_enc, k_dec, v_dec, S: int, scale: float = 0.0):
        """q [B,Hq,L,d]; k_enc/v_enc/k_dec/v_dec [B,Hkv,L,d] -> (out, lse)."""
        B, Hq, L, d = q.shape
        Hkv = k_enc.shape[1]
        for t in (k_enc, v_enc, k_dec, v_dec):
            assert t.shape == (B, Hkv, L, d)
        arrs = [self._f32(t) for t in (q, k_enc, v_enc, k_dec, v_dec)]
        out = np.zeros((B, Hq, L, d), dtype=np.float64)
        lse = np.zeros((B, Hq, L), dtype=np.float64)
        rc = self.lib.oracle_decoder_train(*[p for _, p in arrs], B, Hq, Hkv, L, S, d,
                                           float(scale), out.ctypes.data_as(_f64p),
                                           lse.ctypes.data_as(_f64p))
        if rc:
            raise RuntimeError(f"oracle_decoder_train failed ({rc})")
        return out, lse

    # ---- backward of the train calls ----------------------------------------------
    def bd3lm_train(self, q, k, v, S: int, scale: float = 0.0):
        """BD3LM's attention over 2L tokens (noised copy first, then clean): q [B,Hq,2L,d],
        k/v [B,Hkv,2L,d] -> (out [B,Hq,2L,d] f64, lse [B,Hq,2L] f64)."""
        B, Hq, W, d = q.shape
        Hkv = k.shape[1]
        assert W % 2 == 0 and k.shape == (B, Hkv, W, d) and v.shape == k.shape
        q, qp = self._f32(q)
        k, kp = self._f32(k)
        v, vp = self._f32(v)
        out = np.zeros((B, Hq, W, d), dtype=np.float64)
        lse = np.zeros((B, Hq, W), dtype=np.float64)
        rc = self.lib.oracle_bd3lm_train(qp, kp, vp, B, Hq, Hkv, W // 2, S, d, float(scale),
                                         out.ctypes.data_as(_f64p), lse.ctypes.data_as(_f64p))
        if rc:
            raise RuntimeError(f"oracle_bd3lm_train failed ({rc})")
        return out, lse

    def encoder_backward(self, q, k, v, dout, S: int, scale: float = 0.0):
        """Gradients of sum(dout * encoder(q, k, v)) -> (dq [B,Hq,L,d], dk, dv [B,Hkv,L,d]), fp64."""
        B, Hq, L, d = q.shape
        Hkv = k.shape[1]
        assert k.shape == (B, Hkv, L, d) and v.shape == k.shape and dout.shape == q.shape
        arrs = [self._f32(t) for t in (q, k, v, dout)]
        dq = np.zeros((B, Hq, L, d), dtype=np.float64)
        dk = np.zeros((B, Hkv, L, d), dtype=np.float64)
        dv = np.zeros((B, Hkv, L, d), dtype=np.float64)
        rc = self.lib.oracle_encoder_backward(*[p for _, p in arrs], B, Hq, Hkv, L, S, d, float(scale),
                                              *[t.ctypes.data_as(_f64p) for t in (dq, dk, dv)])
        if rc:
            raise RuntimeError(f"oracle_encoder_backward failed ({rc})")
        return dq, dk, dv

    def decoder_train_backward(self, q, k_enc, v_enc, k_dec, v_dec, dout, S: int, scale: float = 0.0):
        """Gradients of sum(dout * decoder_train(...)) -> (dq, dk_enc, dv_enc, dk_dec, dv_dec), fp64."""
        B, Hq, L, d = q.shape
        Hkv = k_enc.shape[1]
        for t in (k_enc, v_enc, k_dec, v_dec):
            assert t.shape == (B, Hkv, L, d)
        assert dout.shape == q.shape
        arrs = [self._f32(t) for t in (q, k_enc, v_enc, k_dec, v_dec, dout)]
        dq = np.zeros((B, Hq, L, d), dtype=np.float64)
        grads = [np.zeros((B, Hkv, L, d), dtype=np.float64) for _ in range(4)]
        rc = self.lib.oracle_decoder_train_backward(*[p for _, p in arrs], B, Hq, Hkv, L, S, d, float(scale),
                                                    dq.ctypes.data_as(_f64p),
                                                    *[t.ctypes.data_as(_f64p) for t in grads])
        if rc:
            raise RuntimeError(f"oracle_decoder_train_backward failed ({rc})")
        return (dq, *grads)

    def decoder_sample(self, q, k_cache, v_cache, P: int, k_blk, v_blk, scale: float = 0.0):
        """q [B,Hq,S,d]; caches [B,Hkv,cap,d] (first P rows valid); k_blk/v_blk [B,Hkv,S,d]."""
        B, Hq, S, d = q.shape
        Hkv, cap = k_cache.shape[1], k_cache.shape[2]
        assert k_cache.shape == (B, Hkv, cap, d) and v_cache.shape == k_cache.shape
        assert k_blk.shape == (B, Hkv, S, d) and v_blk.shape == k_blk.shape
        arrs = [self._f32(t) for t in (q, k_cache, v_cache, k_blk, v_blk)]
        out = np.zeros((B, Hq, S, d), dtype=np.float64)
        lse = np.zeros((B, Hq, S), dtype=np.float64)
        rc = self.lib.oracle_decoder_sample(arrs[0][1], arrs[1][1], arrs[2][1], cap, P,
                                            arrs[3][1], arrs[4][1], B, Hq, Hkv, S, d,
                                            float(scale), out.ctypes.data_as(_f64p),
                                            lse.ctypes.data_as(_f64p))
        if rc:
            raise RuntimeError(f"oracle_decoder_sample failed ({rc})")
        return out, lse

    def decoder_sample_ragged(self, q, k_cache, v_cache, P, k_blk, v_blk, scale: float = 0.0):
        """Sampling step with a prefix length per batch entry: P is a sequence of B ints."""
        B, Hq, S, d = q.shape
        Hkv, cap = k_cache.shape[1], k_cache.shape[2]
        assert k_cache.shape == (B, Hkv, cap, d) and v_cache.shape == k_cache.shape
        assert k_blk.shape == (B, Hkv, S, d) and v_blk.shape == k_blk.shape
        Pa = np.ascontiguousarray(np.asarray(P, dtype=np.int32))
        assert Pa.shape == (B,)
        arrs = [self._f32(t) for t in (q, k_cache, v_cache, k_blk, v_blk)]
        out = np.zeros((B, Hq, S, d), dtype=np.float64)
        lse = np.zeros((B, Hq, S), dtype=np.float64)
        rc = self.lib.oracle_decoder_sample_ragged(arrs[0][1], arrs[1][1], arrs[2][1], cap,
                                                   Pa.ctypes.data_as(ctypes.POINTER(ctypes.c_int)),
                                                   arrs[3][1], arrs[4][1], B, Hq, Hkv, S, d, float(scale),
                                                   out.ctypes.data_as(_f64p), lse.ctypes.data_as(_f64p))
        if rc:
            raise RuntimeError(f"oracle_decoder_sample_ragged failed ({rc})")
        return out, lse

    def kv_append(self, k_cache_bits, v_cache_bits, P: int, k_new_bits, v_new_bits):
        """In-place append on uint16 (bf16 bit pattern) caches [B,Hkv,cap,d]."""
        B, Hkv, cap, d = k_cache_bits.shape
        S_new = k_new_bits.shape[2]
        for a in (k_cache_bits, v_cache_bits, k_new_bits, v_new_bits):
            assert a.dtype == np.uint16 and a.flags.c_contiguous
        rc = self.lib.oracle_kv_append(k_cache_bits.ctypes.data_as(_u16p),
                                       v_cache_bits.ctypes.data_as(_u16p), cap, P,
                                       k_new_bits.ctypes.data_as(_u16p),
                                       v_new_bits.ctypes.data_as(_u16p), S_new, B, Hkv, d)
        if rc:
            raise RuntimeError(f"oracle_kv_append failed ({rc})")


_default: Oracle | None = None


def default() -> Oracle:
    """The oracle built from ``e2d2_oracle.c`` (compiled on first use)."""
    global _default
    if _default is None:
        _default = Oracle()
    return _default

