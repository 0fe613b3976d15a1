"""Python front-end of the E2D2 attention C ABI, taking torch tensors.

Argument marshalling only: every step of the attention runs in the CUDA kernels of
``libe2d2_attn.so``.  PyTorch provides device memory and the stream (the current stream of
the tensors' device).  Names follow the C ABI (include/e2d2_attn.h)."""
from __future__ import annotations

import ctypes
import functools
import math

import torch

from . import _lib

_BF16 = torch.bfloat16


def _dims(batch, q_heads, kv_heads, head_dim, scale):
    return _lib.Dims(batch, q_heads, kv_heads, head_dim, 0.0 if scale is None else float(scale))


def _need(t: torch.Tensor, name: str, dtype=_BF16, ndim=4):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _device_guard(fn):
    """Runs a call with the GPU of its first tensor current (the C calls read the current device:
    SM count, error word) and rejects tensors spread over several devices."""

    @functools.wraps(fn)
    def wrapper(*args, **kwargs):
        first = args[0] if args else None
        if isinstance(first, torch.Tensor) and first.is_cuda:
            idx = first.get_device()
            for a in (*args, *kwargs.values()):
                if isinstance(a, torch.Tensor) and a.get_device() != idx:
                    raise ValueError(f"{fn.__name__}: every tensor must be on cuda:{idx}")
            if idx != torch.cuda.current_device():
                with torch.cuda.device(idx):
                    return fn(*args, **kwargs)
        return fn(*args, **kwargs)

    return wrapper


def _out_tensor(out, like: torch.Tensor) -> torch.Tensor:
    """The output buffer: a new one like `like`, or the caller's, checked (the kernels write
    every element of it through a plain pointer)."""
    if out is None:
        return torch.empty_like(like)
    _need(out, "out")
    if out.shape != like.shape:
        raise ValueError(f"out must have shape {tuple(like.shape)}, got {tuple(out.shape)}")
    return out


def _lse_tensor(lse, shape, device):
    """lse=True: a new fp32 tensor; None/False: not computed; a tensor: the caller's, checked."""
    if lse is True:
        return torch.empty(shape, dtype=torch.float32, device=device)
    if lse is None or lse is False:
        return None
    _need(lse, "lse", dtype=torch.float32, ndim=3)
    if tuple(lse.shape) != tuple(shape):
        raise ValueError(f"lse must have shape {tuple(shape)}, got {tuple(lse.shape)}")
    return lse


def _need_workspace(ws: torch.Tensor) -> torch.Tensor:
    if not isinstance(ws, torch.Tensor) or not ws.is_cuda or not ws.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    return ws


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(t: torch.Tensor):
    return ctypes_stream(torch.cuda.current_stream(t.device))


def ctypes_stream(s: torch.cuda.Stream):
    return s.cuda_stream


@_device_guard
def encoder_blockcausal(q, k, v, S: int, scale=None, out=None, lse=True):
    """Block-causal encoder self-attention.  q [B,Hq,L,d], k/v [B,Hkv,L,d] (bf16, CUDA).
    Returns (out [B,Hq,L,d] bf16, lse [B,Hq,L] fp32 or None)."""
    lib = _lib.load()
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n)
    B, Hq, L, d = q.shape
    Hkv = k.shape[1]
    if k.shape != (B, Hkv, L, d) or v.shape != k.shape:
        raise ValueError("k/v must be [B, Hkv, L, d] matching q")
    out = _out_tensor(out, q)
    lse_t = _lse_tensor(lse, (B, Hq, L), q.device)
    st = lib.e2d2_attn_encoder_blockcausal(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), _ptr(lse_t),
                                           _dims(B, Hq, Hkv, d, scale), L, S, _stream(q))
    _lib.check(st, "e2d2_attn_encoder_blockcausal")
    return out, lse_t


@_device_guard
def decoder_train(q, k_enc, v_enc, k_dec, v_dec, S: int, scale=None, out=None, lse=True):
    """Decoder fused self+cross attention (training mode) over 2L keys."""
    lib = _lib.load()
    for t, n in ((q, "q"), (k_enc, "k_enc"), (v_enc, "v_enc"), (k_dec, "k_dec"), (v_dec, "v_dec")):
        _need(t, n)
    B, Hq, L, d = q.shape
    Hkv = k_enc.shape[1]
    for t in (k_enc, v_enc, k_dec, v_dec):
        if t.shape != (B, Hkv, L, d):
            raise ValueError("k_enc/v_enc/k_dec/v_dec must be [B, Hkv, L, d] matching q")
    out = _out_tensor(out, q)
    lse_t = _lse_tensor(lse, (B, Hq, L), q.device)
    st = lib.e2d2_attn_decoder_train(q.data_ptr(), k_enc.data_ptr(), v_enc.data_ptr(), k_dec.data_ptr(),
                                     v_dec.data_ptr(), out.data_ptr(), _ptr(lse_t),
                                     _dims(B, Hq, Hkv, d, scale), L, S, _stream(q))
    _lib.check(st, "e2d2_attn_decoder_train")
    return out, lse_t


def train_backward_workspace_bytes(batch, q_heads, kv_heads, head_dim, L) -> int:
    """Bytes of workspace the backward calls need (no GPU needed)."""
    lib = _lib.load()
    return int(lib.e2d2_attn_train_backward_workspace(_dims(batch, q_heads, kv_heads, head_dim, None), L))


def _train_backward_ws(lib, B, Hq, Hkv, d, L, scale, device, workspace):
    need = lib.e2d2_attn_train_backward_workspace(_dims(B, Hq, Hkv, d, scale), L)
    if workspace is None:
        return torch.empty(max(need, 16), dtype=torch.uint8, device=device)
    return _need_workspace(workspace)


@_device_guard
def encoder_backward(q, k, v, out, lse, dout, S: int, scale=None, workspace=None):
    """Gradients of the encoder call: (dq [B,Hq,L,d], dk, dv [B,Hkv,L,d]) bf16, from the forward's
    output out (bf16) and lse (fp32) and the output gradient dout."""
    lib = _lib.load()
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out"), (dout, "dout")):
        _need(t, n)
    _need(lse, "lse", dtype=torch.float32, ndim=3)
    B, Hq, L, d = q.shape
    Hkv = k.shape[1]
    if k.shape != (B, Hkv, L, d) or v.shape != k.shape or dout.shape != q.shape or out.shape != q.shape:
        raise ValueError("k/v must be [B, Hkv, L, d]; out and dout must match q")
    if lse.shape != (B, Hq, L):
        raise ValueError("lse must be [B, Hq, L]")
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = _train_backward_ws(lib, B, Hq, Hkv, d, L, scale, q.device, workspace)
    st = lib.e2d2_attn_encoder_backward(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                        dout.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                                        _dims(B, Hq, Hkv, d, scale), L, S, ws.data_ptr(),
                                        ws.numel() * ws.element_size(), _stream(q))
    _lib.check(st, "e2d2_attn_encoder_backward")
    return dq, dk, dv


@_device_guard
def decoder_train_backward(q, k_enc, v_enc, k_dec, v_dec, out, lse, dout, S: int, scale=None, workspace=None):
    """Gradients of the decoder train call: (dq, dk_enc, dv_enc, dk_dec, dv_dec) bf16, from the
    forward's output out and lse and the output gradient dout."""
    lib = _lib.load()
    for t, n in ((q, "q"), (k_enc, "k_enc"), (v_enc, "v_enc"), (k_dec, "k_dec"), (v_dec, "v_dec"),
                 (out, "out"), (dout, "dout")):
        _need(t, n)
    _need(lse, "lse", dtype=torch.float32, ndim=3)
    B, Hq, L, d = q.shape
    Hkv = k_enc.shape[1]
    for t in (k_enc, v_enc, k_dec, v_dec):
        if t.shape != (B, Hkv, L, d):
            raise ValueError("k_enc/v_enc/k_dec/v_dec must be [B, Hkv, L, d] matching q")
    if dout.shape != q.shape or out.shape != q.shape or lse.shape != (B, Hq, L):
        raise ValueError("out and dout must match q and lse must be [B, Hq, L]")
    dq = torch.empty_like(q)
    grads = [torch.empty_like(k_enc) for _ in range(4)]
    ws = _train_backward_ws(lib, B, Hq, Hkv, d, L, scale, q.device, workspace)
    st = lib.e2d2_attn_decoder_train_backward(q.data_ptr(), k_enc.data_ptr(), v_enc.data_ptr(), k_dec.data_ptr(),
                                              v_dec.data_ptr(), out.data_ptr(), lse.data_ptr(), dout.data_ptr(),
                                              dq.data_ptr(), *[g.data_ptr() for g in grads],
                                              _dims(B, Hq, Hkv, d, scale), L, S, ws.data_ptr(),
                                              ws.numel() * ws.element_size(), _stream(q))
    _lib.check(st, "e2d2_attn_decoder_train_backward")
    return (dq, *grads)


def sample_workspace_bytes(batch, q_heads, kv_heads, head_dim, S, capacity) -> int:
    lib = _lib.load()
    return int(lib.e2d2_attn_decoder_sample_workspace(_dims(batch, q_heads, kv_heads, head_dim, None),
                                                      S, capacity))


def sample_plan(batch, q_heads, kv_heads, head_dim, S, P, num_sms) -> dict:
    """Work plan of a sampling call on a GPU with num_sms SMs (no GPU needed)."""
    lib = _lib.load()
    plan = _lib.SamplePlan()
    st = lib.e2d2_attn_decoder_sample_plan(_dims(batch, q_heads, kv_heads, head_dim, None), S, P, num_sms,
                                           ctypes.byref(plan))
    _lib.check(st, "e2d2_attn_decoder_sample_plan")
    return {name: getattr(plan, name) for name, _ in _lib.SamplePlan._fields_}


def train_order(decoder: bool, batch, q_heads, kv_heads, head_dim, L, S, num_sms) -> dict:
    """Work order of a train call on a GPU with num_sms SMs (no GPU needed): the CTA of each work
    item (pairs of 128-row query tiles), the grid, and whether the balanced order is used."""
    lib = _lib.load()
    items, grid, bal = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    st = lib.e2d2_attn_train_order(int(bool(decoder)), _dims(batch, q_heads, kv_heads, head_dim, None), L, S,
                                   num_sms, None, ctypes.byref(items), ctypes.byref(grid), ctypes.byref(bal))
    _lib.check(st, "e2d2_attn_train_order")
    cta = (ctypes.c_int * items.value)()
    st = lib.e2d2_attn_train_order(int(bool(decoder)), _dims(batch, q_heads, kv_heads, head_dim, None), L, S,
                                   num_sms, cta, None, None, None)
    _lib.check(st, "e2d2_attn_train_order")
    return {"items": items.value, "grid": grid.value, "balanced": bool(bal.value), "cta_of_item": list(cta)}


@_device_guard
def sample_workspace(q_blk: torch.Tensor, k_cache: torch.Tensor) -> torch.Tensor:
    """A zero-filled workspace for decoder_sample with these shapes."""
    B, Hq, S, d = q_blk.shape
    Hkv, cap = k_cache.shape[1], k_cache.shape[2]
    n = sample_workspace_bytes(B, Hq, Hkv, d, S, cap)
    return torch.zeros(n, dtype=torch.uint8, device=q_blk.device)


@_device_guard
def decoder_sample(q_blk, k_cache, v_cache, P: int, k_blk, v_blk, workspace=None, scale=None,
                   out=None, lse=True):
    """Decoder sampling step over the cached prefix k_cache[:, :, :P] plus the own block."""
    lib = _lib.load()
    for t, n in ((q_blk, "q_blk"), (k_cache, "k_cache"), (v_cache, "v_cache"), (k_blk, "k_blk"),
                 (v_blk, "v_blk")):
        _need(t, n)
    B, Hq, S, d = q_blk.shape
    Hkv, cap = k_cache.shape[1], k_cache.shape[2]
    if k_cache.shape != (B, Hkv, cap, d) or v_cache.shape != k_cache.shape:
        raise ValueError("caches must be [B, Hkv, capacity, d]")
    if k_blk.shape != (B, Hkv, S, d) or v_blk.shape != k_blk.shape:
        raise ValueError("k_blk/v_blk must be [B, Hkv, S, d]")
    ws = sample_workspace(q_blk, k_cache) if workspace is None else _need_workspace(workspace)
    out = _out_tensor(out, q_blk)
    lse_t = _lse_tensor(lse, (B, Hq, S), q_blk.device)
    st = lib.e2d2_attn_decoder_sample(q_blk.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), cap, int(P),
                                      k_blk.data_ptr(), v_blk.data_ptr(), out.data_ptr(),
                                      _ptr(lse_t),
                                      _dims(B, Hq, Hkv, d, scale), S, ws.data_ptr(),
                                      ws.numel() * ws.element_size(), _stream(q_blk))
    _lib.check(st, "e2d2_attn_decoder_sample")
    return out, lse_t


def sample_ragged_plan(batch, q_heads, kv_heads, head_dim, S, P, capacity, num_sms) -> dict:
    """Work plan of a ragged sampling call for host prefix lengths P (a sequence of batch ints)."""
    lib = _lib.load()
    P = [int(x) for x in P]
    if len(P) != batch:
        raise ValueError("P must hold one prefix length per batch entry")
    arr = (ctypes.c_int * max(batch, 1))(*P)
    plan = _lib.RaggedPlan()
    st = lib.e2d2_attn_decoder_sample_ragged_plan(_dims(batch, q_heads, kv_heads, head_dim, None), S, arr, capacity,
                                                  num_sms, ctypes.byref(plan))
    _lib.check(st, "e2d2_attn_decoder_sample_ragged_plan")
    return {name: getattr(plan, name) for name, _ in _lib.RaggedPlan._fields_}


@_device_guard
def decoder_sample_ragged(q_blk, k_cache, v_cache, P, k_blk, v_blk, workspace=None, scale=None, out=None, lse=True):
    """Sampling step with one prefix length per batch entry: P is a CUDA int32 tensor [B]; entry b
    attends to k_cache[b, :, :P[b]] and its own block."""
    lib = _lib.load()
    for t, n in ((q_blk, "q_blk"), (k_cache, "k_cache"), (v_cache, "v_cache"), (k_blk, "k_blk"),
                 (v_blk, "v_blk")):
        _need(t, n)
    _need(P, "P", dtype=torch.int32, ndim=1)
    B, Hq, S, d = q_blk.shape
    Hkv, cap = k_cache.shape[1], k_cache.shape[2]
    if k_cache.shape != (B, Hkv, cap, d) or v_cache.shape != k_cache.shape:
        raise ValueError("caches must be [B, Hkv, capacity, d]")
    if k_blk.shape != (B, Hkv, S, d) or v_blk.shape != k_blk.shape:
        raise ValueError("k_blk/v_blk must be [B, Hkv, S, d]")
    if P.shape != (B,):
        raise ValueError("P must be [B]")
    ws = sample_workspace(q_blk, k_cache) if workspace is None else _need_workspace(workspace)
    out = _out_tensor(out, q_blk)
    lse_t = _lse_tensor(lse, (B, Hq, S), q_blk.device)
    st = lib.e2d2_attn_decoder_sample_ragged(q_blk.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), cap,
                                             P.data_ptr(), k_blk.data_ptr(), v_blk.data_ptr(), out.data_ptr(),
                                             _ptr(lse_t), _dims(B, Hq, Hkv, d, scale), S, ws.data_ptr(),
                                             ws.numel() * ws.element_size(), _stream(q_blk))
    _lib.check(st, "e2d2_attn_decoder_sample_ragged")
    return out, lse_t


@_device_guard
def encoder_block_step(q_blk, k_cache, v_cache, P: int, k_blk, v_blk, workspace=None, scale=None,
                       out=None, lse=True):
    """Encoder incremental block step: the block's S clean queries attend to k_cache[:, :, :P] and
    to their own block (block-causal rows of the encoder), and k_blk/v_blk are written to cache
    rows P..P+S-1 in the same launch.  Returns (out, lse); the new prefix length is P + S."""
    lib = _lib.load()
    for t, n in ((q_blk, "q_blk"), (k_cache, "k_cache"), (v_cache, "v_cache"), (k_blk, "k_blk"),
                 (v_blk, "v_blk")):
        _need(t, n)
    B, Hq, S, d = q_blk.shape
    Hkv, cap = k_cache.shape[1], k_cache.shape[2]
    if k_cache.shape != (B, Hkv, cap, d) or v_cache.shape != k_cache.shape:
        raise ValueError("caches must be [B, Hkv, capacity, d]")
    if k_blk.shape != (B, Hkv, S, d) or v_blk.shape != k_blk.shape:
        raise ValueError("k_blk/v_blk must be [B, Hkv, S, d]")
    ws = sample_workspace(q_blk, k_cache) if workspace is None else _need_workspace(workspace)
    out = _out_tensor(out, q_blk)
    lse_t = _lse_tensor(lse, (B, Hq, S), q_blk.device)
    st = lib.e2d2_attn_encoder_block_step(q_blk.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), cap, int(P),
                                          k_blk.data_ptr(), v_blk.data_ptr(), out.data_ptr(),
                                          _ptr(lse_t),
                                          _dims(B, Hq, Hkv, d, scale), S, ws.data_ptr(),
                                          ws.numel() * ws.element_size(), _stream(q_blk))
    _lib.check(st, "e2d2_attn_encoder_block_step")
    return out, lse_t


@_device_guard
def kv_cache_append(k_cache, v_cache, P: int, k_new, v_new):
    """Writes k_new/v_new [B,Hkv,S_new,d] into rows P..P+S_new-1 of the caches; returns P+S_new."""
    lib = _lib.load()
    for t, n in ((k_cache, "k_cache"), (v_cache, "v_cache"), (k_new, "k_new"), (v_new, "v_new")):
        _need(t, n)
    B, Hkv, cap, d = k_cache.shape
    S_new = k_new.shape[2]
    if k_new.shape != (B, Hkv, S_new, d) or v_new.shape != k_new.shape or v_cache.shape != k_cache.shape:
        raise ValueError("shape mismatch")
    st = lib.e2d2_kv_cache_append(k_cache.data_ptr(), v_cache.data_ptr(), cap, int(P), k_new.data_ptr(),
                                  v_new.data_ptr(), S_new, _dims(B, Hkv, Hkv, d, None), _stream(k_cache))
    _lib.check(st, "e2d2_kv_cache_append")
    return P + S_new


@_device_guard
def kv_cache_append_ragged(k_cache, v_cache, P, k_new, v_new):
    """Writes k_new/v_new [B,Hkv,S_new,d] into rows P[b]..P[b]+S_new-1 of entry b's caches, P a
    CUDA int32 tensor [B] (not advanced: the caller adds S_new when the block is final)."""
    lib = _lib.load()
    for t, n in ((k_cache, "k_cache"), (v_cache, "v_cache"), (k_new, "k_new"), (v_new, "v_new")):
        _need(t, n)
    _need(P, "P", dtype=torch.int32, ndim=1)
    B, Hkv, cap, d = k_cache.shape
    S_new = k_new.shape[2]
    if k_new.shape != (B, Hkv, S_new, d) or v_new.shape != k_new.shape or v_cache.shape != k_cache.shape:
        raise ValueError("shape mismatch")
    if P.shape != (B,):
        raise ValueError("P must be [B]")
    st = lib.e2d2_kv_cache_append_ragged(k_cache.data_ptr(), v_cache.data_ptr(), cap, P.data_ptr(), k_new.data_ptr(),
                                         v_new.data_ptr(), S_new, _dims(B, Hkv, Hkv, d, None), _stream(k_cache))
    _lib.check(st, "e2d2_kv_cache_append_ragged")


def last_device_error(device=None) -> int:
    lib = _lib.load()
    return int(lib.e2d2_last_device_error(torch.cuda.current_stream(device).cuda_stream))


def default_scale(head_dim: int) -> float:
    return 1.0 / math.sqrt(head_dim)
