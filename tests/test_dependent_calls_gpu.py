"""Chains of calls where each reads what the previous one wrote, queued back to back on one
stream with no host synchronisation in between, eagerly and inside a CUDA graph.  Every kernel
is launched with programmatic stream serialization and may start while its predecessor is still
running; its griddepcontrol.wait must hold it until the predecessor's writes are visible.  The
chain's results are compared with the oracle run step by step on the exact bf16 values the GPU
produced at each step (so only the dependency, not accumulated rounding, is under test)."""
import numpy as np
import pytest
import torch

from block_discrete_diffusion_tcgen05_b200 import attn
import gpu_helpers as H

pytestmark = pytest.mark.gpu


def _f32(t):
    return t.float().cpu().numpy()


def _encoder_chain(q, k, v, S, steps):
    """out_{i+1} = encoder(out_i, k, v), out_0 = q: each call's Q is the previous call's output."""
    outs, lses = [], []
    x = q
    for _ in range(steps):
        o, l = attn.encoder_blockcausal(x, k, v, S)
        outs.append(o)
        lses.append(l)
        x = o
    return outs, lses


def _check_chain(oracle, q, k, v, S, outs, lses):
    x = _f32(q)
    kf, vf = _f32(k), _f32(v)
    for i, (o, l) in enumerate(zip(outs, lses)):
        ref_o, ref_l = oracle.encoder(x, kf, vf, S)
        H.compare(o, l, ref_o, ref_l, f"chain step {i}")
        x = _f32(o)   # the next step's input is exactly what the GPU wrote


def test_encoder_chain_eager(oracle):
    B, Hq, Hkv, L, S, d = 2, 4, 2, 384, 16, 64
    q = H.gen((B, Hq, L, d), 2600, 1.0)[1]
    k = H.gen((B, Hkv, L, d), 2601, 1.0)[1]
    v = H.gen((B, Hkv, L, d), 2602, 1.0)[1]
    outs, lses = _encoder_chain(q, k, v, S, 6)
    torch.cuda.synchronize()
    _check_chain(oracle, q, k, v, S, outs, lses)


def test_encoder_chain_in_a_graph(oracle):
    B, Hq, Hkv, L, S, d = 1, 4, 4, 256, 16, 64
    q = H.gen((B, Hq, L, d), 2700, 1.0)[1]
    k = H.gen((B, Hkv, L, d), 2701, 1.0)[1]
    v = H.gen((B, Hkv, L, d), 2702, 1.0)[1]
    bufs = [torch.empty_like(q) for _ in range(5)]
    lses = [torch.empty(B, Hq, L, device="cuda") for _ in range(5)]
    attn.encoder_blockcausal(q, k, v, S, out=bufs[0], lse=lses[0])   # warm-up outside the capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            x = q
            for i in range(5):
                attn.encoder_blockcausal(x, k, v, S, out=bufs[i], lse=lses[i])
                x = bufs[i]
    torch.cuda.synchronize()
    for b in bufs:
        b.zero_()
    g.replay()
    torch.cuda.synchronize()
    _check_chain(oracle, q, k, v, S, bufs, lses)
    assert attn.last_device_error() == 0


def test_backward_feeds_the_next_backward(oracle):
    """dq of one backward call is the dout of the next (rows-Q, then rows-KV, then the next
    call's rows-Q reading what the previous rows-KV launch left in the shared workspace)."""
    B, Hq, Hkv, L, S, d = 1, 2, 2, 200, 16, 64
    qq, ks = H.train_inputs(B, Hq, Hkv, L, d, 1.0, 2800)
    (k, kt), (v, vt) = ks[0], ks[1]
    g0 = H.gen((B, Hq, L, d), 2809, 1.0)[1]
    o, l = attn.encoder_blockcausal(qq[1], kt, vt, S)
    g = g0
    grads = []
    for _ in range(3):
        dq, dk, dv = attn.encoder_backward(qq[1], kt, vt, o, l, g, S)
        grads.append((dq, dk, dv))
        g = dq
    torch.cuda.synchronize()
    gin = _f32(g0)
    for i, (dq, dk, dv) in enumerate(grads):
        ref = oracle.encoder_backward(qq[0].f32, k.f32, v.f32, gin, S)
        for a, r, nm in zip((dq, dk, dv), ref, ("dq", "dk", "dv")):
            err = np.abs(_f32(a) - r)
            assert (err <= 2e-2 + 2.0 ** -7 * np.abs(r)).all(), f"step {i} {nm}: max err {err.max():.3e}"
        gin = _f32(dq)
    assert attn.last_device_error() == 0
