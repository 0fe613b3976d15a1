"""Argument marshalling of the Python binding, checked on the CPU against the header itself: every
wrapper runs end to end with CPU tensors and a recording stand-in for the C library (only the
CUDA-residency check and the stream lookup are stubbed), and each recorded C call is matched,
parameter by parameter, to the names include/e2d2_attn.h declares -- q to q's pointer, lse to
the returned lse's pointer, dims to the right fields, and so on.  A swapped or missing argument
in a wrapper fails here without a GPU."""
import re
from pathlib import Path

import pytest
import torch

from block_discrete_diffusion_tcgen05_b200 import _lib, attn

HEADER = Path(__file__).resolve().parents[1] / "include" / "e2d2_attn.h"
STREAM = 0x5EED
WS_BYTES = 4096


def header_params():
    text = HEADER.read_text()
    out = {}
    for m in re.finditer(r"E2D2_API\s+[\w\s\*]+?\b(e2d2_\w+)\s*\(([^)]*)\)\s*;", text):
        params = [re.split(r"[\s\*]+", p.strip())[-1] for p in m.group(2).split(",")]
        out[m.group(1)] = [p for p in params if p and p != "void"]
    return out


PARAMS = header_params()


class Recorder:
    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def fn(*args):
            self.calls.append((name, args))
            return WS_BYTES if name.endswith("_workspace") else 0
        return fn

    def call(self, name):
        found = [dict(zip(PARAMS[name], args)) for n, args in self.calls if n == name]
        assert len(found) == 1, f"{name} called {len(found)} times"
        assert len(found[0]) == len(PARAMS[name])
        return found[0]


@pytest.fixture
def rec(monkeypatch):
    r = Recorder()
    monkeypatch.setattr(_lib, "load", lambda path=None: r)

    def need(t, name, dtype=torch.bfloat16, ndim=4):
        assert isinstance(t, torch.Tensor) and t.dtype == dtype and t.dim() == ndim and t.is_contiguous(), name

    monkeypatch.setattr(attn, "_need", need)
    monkeypatch.setattr(attn, "_need_workspace", lambda ws: ws)
    monkeypatch.setattr(attn, "_stream", lambda t: STREAM)
    return r


def bf16(*shape):
    return torch.randn(*shape).to(torch.bfloat16)


def check_dims(dims, B, Hq, Hkv, d, scale):
    assert (dims.batch, dims.q_heads, dims.kv_heads, dims.head_dim) == (B, Hq, Hkv, d)
    assert dims.scale == pytest.approx(0.0 if scale is None else scale)


B, Hq, Hkv, L, S, d = 2, 4, 2, 48, 8, 64


def test_every_wrapped_call_is_declared():
    for name in ("e2d2_attn_encoder_blockcausal", "e2d2_attn_decoder_train", "e2d2_attn_encoder_backward",
                 "e2d2_attn_decoder_train_backward", "e2d2_attn_decoder_sample", "e2d2_attn_encoder_block_step",
                 "e2d2_kv_cache_append", "e2d2_attn_train_backward_workspace",
                 "e2d2_attn_decoder_sample_workspace", "e2d2_attn_decoder_sample_ragged"):
        assert name in PARAMS, name


def test_encoder_blockcausal(rec):
    q, k, v = bf16(B, Hq, L, d), bf16(B, Hkv, L, d), bf16(B, Hkv, L, d)
    out, lse = attn.encoder_blockcausal(q, k, v, S, scale=0.3)
    a = rec.call("e2d2_attn_encoder_blockcausal")
    assert (a["q"], a["k"], a["v"]) == (q.data_ptr(), k.data_ptr(), v.data_ptr())
    assert a["out"] == out.data_ptr() and a["lse"] == lse.data_ptr() and lse.shape == (B, Hq, L)
    check_dims(a["dims"], B, Hq, Hkv, d, 0.3)
    assert (a["L"], a["S"], a["stream"]) == (L, S, STREAM)


def test_encoder_without_lse_passes_null(rec):
    q, k, v = bf16(B, Hq, L, d), bf16(B, Hkv, L, d), bf16(B, Hkv, L, d)
    given = bf16(B, Hq, L, d)
    out, lse = attn.encoder_blockcausal(q, k, v, S, out=given, lse=False)
    a = rec.call("e2d2_attn_encoder_blockcausal")
    assert out is given and a["out"] == given.data_ptr() and a["lse"] is None and lse is None


def test_decoder_train(rec):
    q = bf16(B, Hq, L, d)
    ke, ve, kd, vd = (bf16(B, Hkv, L, d) for _ in range(4))
    lse_given = torch.zeros(B, Hq, L)
    out, lse = attn.decoder_train(q, ke, ve, kd, vd, S, lse=lse_given)
    a = rec.call("e2d2_attn_decoder_train")
    assert (a["q_dec"], a["k_enc"], a["v_enc"], a["k_dec"], a["v_dec"]) == tuple(
        t.data_ptr() for t in (q, ke, ve, kd, vd))
    assert a["out"] == out.data_ptr() and lse is lse_given and a["lse"] == lse_given.data_ptr()
    check_dims(a["dims"], B, Hq, Hkv, d, None)
    assert (a["L"], a["S"], a["stream"]) == (L, S, STREAM)


def test_encoder_backward(rec):
    q, k, v, g = bf16(B, Hq, L, d), bf16(B, Hkv, L, d), bf16(B, Hkv, L, d), bf16(B, Hq, L, d)
    o = bf16(B, Hq, L, d)
    lse = torch.zeros(B, Hq, L)
    dq, dk, dv = attn.encoder_backward(q, k, v, o, lse, g, S, scale=0.25)
    a = rec.call("e2d2_attn_encoder_backward")
    assert (a["q"], a["k"], a["v"], a["out"], a["lse"], a["dout"]) == tuple(
        t.data_ptr() for t in (q, k, v, o, lse, g))
    assert (a["dq"], a["dk"], a["dv"]) == (dq.data_ptr(), dk.data_ptr(), dv.data_ptr())
    assert dq.shape == q.shape and dk.shape == k.shape and dv.shape == v.shape
    check_dims(a["dims"], B, Hq, Hkv, d, 0.25)
    assert (a["L"], a["S"], a["stream"]) == (L, S, STREAM)
    assert a["ws_bytes"] >= WS_BYTES and a["workspace"] is not None
    w = rec.call("e2d2_attn_train_backward_workspace")
    check_dims(w["dims"], B, Hq, Hkv, d, 0.25)
    assert w["L"] == L


def test_decoder_train_backward(rec):
    q, g, o = bf16(B, Hq, L, d), bf16(B, Hq, L, d), bf16(B, Hq, L, d)
    ke, ve, kd, vd = (bf16(B, Hkv, L, d) for _ in range(4))
    lse = torch.zeros(B, Hq, L)
    ws = torch.zeros(B * Hq * L)
    dq, dke, dve, dkd, dvd = attn.decoder_train_backward(q, ke, ve, kd, vd, o, lse, g, S, workspace=ws)
    a = rec.call("e2d2_attn_decoder_train_backward")
    assert (a["q_dec"], a["k_enc"], a["v_enc"], a["k_dec"], a["v_dec"], a["out"], a["lse"], a["dout"]) == tuple(
        t.data_ptr() for t in (q, ke, ve, kd, vd, o, lse, g))
    assert (a["dq"], a["dk_enc"], a["dv_enc"], a["dk_dec"], a["dv_dec"]) == tuple(
        t.data_ptr() for t in (dq, dke, dve, dkd, dvd))
    assert a["workspace"] == ws.data_ptr() and a["ws_bytes"] == ws.numel() * 4
    assert (a["L"], a["S"], a["stream"]) == (L, S, STREAM)


@pytest.mark.parametrize("name", ["decoder_sample", "encoder_block_step"])
def test_sampling_calls(rec, name):
    Ss, cap, P = 16, 80, 32
    qb, kc, vc = bf16(B, Hq, Ss, d), bf16(B, Hkv, cap, d), bf16(B, Hkv, cap, d)
    kb, vb = bf16(B, Hkv, Ss, d), bf16(B, Hkv, Ss, d)
    out, lse = getattr(attn, name)(qb, kc, vc, P, kb, vb, scale=0.5)
    cname = "e2d2_attn_decoder_sample" if name == "decoder_sample" else "e2d2_attn_encoder_block_step"
    a = rec.call(cname)
    assert (a["q_blk"], a["k_cache"], a["v_cache"], a["k_blk"], a["v_blk"]) == tuple(
        t.data_ptr() for t in (qb, kc, vc, kb, vb))
    assert (a["capacity"], a["P"], a["S"], a["stream"]) == (cap, P, Ss, STREAM)
    assert a["out"] == out.data_ptr() and a["lse"] == lse.data_ptr() and lse.shape == (B, Hq, Ss)
    check_dims(a["dims"], B, Hq, Hkv, d, 0.5)
    assert a["ws_bytes"] == WS_BYTES
    w = rec.call("e2d2_attn_decoder_sample_workspace")
    assert (w["S"], w["capacity"]) == (Ss, cap)


def test_kv_cache_append(rec):
    cap, P, Sn = 64, 16, 8
    kc, vc, kn, vn = bf16(B, Hkv, cap, d), bf16(B, Hkv, cap, d), bf16(B, Hkv, Sn, d), bf16(B, Hkv, Sn, d)
    assert attn.kv_cache_append(kc, vc, P, kn, vn) == P + Sn
    a = rec.call("e2d2_kv_cache_append")
    assert (a["k_cache"], a["v_cache"], a["k_new"], a["v_new"]) == tuple(t.data_ptr() for t in (kc, vc, kn, vn))
    assert (a["capacity"], a["P"], a["S_new"], a["stream"]) == (cap, P, Sn, STREAM)
    check_dims(a["dims"], B, Hkv, Hkv, d, None)


def test_decoder_sample_ragged(rec):
    Ss, cap = 16, 80
    qb, kc, vc = bf16(B, Hq, Ss, d), bf16(B, Hkv, cap, d), bf16(B, Hkv, cap, d)
    kb, vb = bf16(B, Hkv, Ss, d), bf16(B, Hkv, Ss, d)
    P = torch.tensor([3, 80][:B], dtype=torch.int32)
    ws = torch.zeros(1024)
    out, lse = attn.decoder_sample_ragged(qb, kc, vc, P, kb, vb, workspace=ws, scale=0.5)
    a = rec.call("e2d2_attn_decoder_sample_ragged")
    assert (a["q_blk"], a["k_cache"], a["v_cache"], a["P_dev"], a["k_blk"], a["v_blk"]) == tuple(
        t.data_ptr() for t in (qb, kc, vc, P, kb, vb))
    assert a["capacity"] == cap and a["S"] == Ss and a["stream"] == STREAM
    assert a["out"] == out.data_ptr() and a["lse"] == lse.data_ptr()
    assert a["workspace"] == ws.data_ptr() and a["ws_bytes"] == ws.numel() * 4
    check_dims(a["dims"], B, Hq, Hkv, d, 0.5)
