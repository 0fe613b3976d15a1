"""GPU parity of the backward of the train calls: the CUDA path (forward, then backward, both
through the C ABI) against the oracle's fp64 gradients of the same bf16 inputs, element by
element.

Tolerance: every gradient is written in bf16 (relative rounding 2^-9) after fp32 accumulation
over at most a few thousand terms; the probabilities come from the forward's fp32 lse (within
its 1e-3 bar of the exact one, which scales every p_ij of a row by at most e^1e-3).  The bar is
|d grad| <= 2e-2 + 2^-7 |grad| per element (the forward's absolute output bar plus two bf16
rounding steps of the value), and the relative Frobenius error of each gradient tensor <= 1e-2."""
import numpy as np
import pytest
import torch

from block_discrete_diffusion_tcgen05_b200 import attn, synth, workloads
import gpu_helpers as H

pytestmark = pytest.mark.gpu

ATOL = 2e-2
RTOL = 2.0 ** -7
FRO_TOL = 1e-2

BWD_CASES = [
    # B, Hq, Hkv, L, S, d
    (1, 2, 2, 64, 8, 32),        # tiny check workload
    (2, 4, 2, 200, 16, 64),      # ragged L (200 = 12 blocks + 8), GQA 2
    (1, 8, 2, 256, 32, 64),      # GQA 4
    (1, 2, 1, 130, 1, 128),      # S = 1 (causal), d 128
    (1, 2, 2, 96, 96, 64),       # S = L: one bidirectional block
    (1, 4, 2, 300, 7, 32),       # short last block (6 rows)
    (1, 2, 1, 100, 160, 64),     # S > L
    (2, 2, 2, 256, 4, 64),       # translation-shaped block size
]


def grad_compare(got, ref, what):
    g = got.float().cpu().numpy().astype(np.float64)
    assert np.isfinite(g).all(), f"{what}: non-finite gradient"
    err = np.abs(g - ref)
    bound = ATOL + RTOL * np.abs(ref)
    worst = np.unravel_index(np.argmax(err - bound), err.shape)
    assert (err <= bound).all(), f"{what}: |d| = {err[worst]:.3e} at {worst} (ref {ref[worst]:.3e})"
    fro = np.linalg.norm(g - ref) / max(np.linalg.norm(ref), 1e-30)
    assert fro <= FRO_TOL, f"{what}: relative Frobenius error {fro:.3e}"
    return float(err.max())


def run_encoder_backward(orc, B, Hq, Hkv, L, S, d, seed0=700):
    q, ks = H.train_inputs(B, Hq, Hkv, L, d, 1.0, seed0)
    (k, kt), (v, vt) = ks[0], ks[1]
    g = H.gen((B, Hq, L, d), seed0 + 9)
    o, lse = attn.encoder_blockcausal(q[1], kt, vt, S)
    dq, dk, dv = attn.encoder_backward(q[1], kt, vt, o, lse, g[1], S)
    torch.cuda.synchronize()
    ref = orc.encoder_backward(q[0].f32, k.f32, v.f32, g[0].f32, S)
    tag = f"encoder bwd B{B} Hq{Hq} Hkv{Hkv} L{L} S{S} d{d}"
    for name, a, r in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
        grad_compare(a, r, f"{tag} {name}")
    return dq, dk, dv


def run_decoder_backward(orc, B, Hq, Hkv, L, S, d, seed0=800):
    q, ks = H.train_inputs(B, Hq, Hkv, L, d, 1.0, seed0)
    (ke, ket), (ve, vet), (kd, kdt), (vd, vdt) = ks
    g = H.gen((B, Hq, L, d), seed0 + 9)
    o, lse = attn.decoder_train(q[1], ket, vet, kdt, vdt, S)
    grads = attn.decoder_train_backward(q[1], ket, vet, kdt, vdt, o, lse, g[1], S)
    torch.cuda.synchronize()
    ref = orc.decoder_train_backward(q[0].f32, ke.f32, ve.f32, kd.f32, vd.f32, g[0].f32, S)
    tag = f"decoder bwd B{B} Hq{Hq} Hkv{Hkv} L{L} S{S} d{d}"
    for name, a, r in zip(("dq", "dk_enc", "dv_enc", "dk_dec", "dv_dec"), grads, ref):
        grad_compare(a, r, f"{tag} {name}")
    return grads


@pytest.mark.parametrize("B,Hq,Hkv,L,S,d", BWD_CASES)
def test_encoder_backward_parity(oracle, B, Hq, Hkv, L, S, d):
    run_encoder_backward(oracle, B, Hq, Hkv, L, S, d)


@pytest.mark.parametrize("B,Hq,Hkv,L,S,d", BWD_CASES)
def test_decoder_train_backward_parity(oracle, B, Hq, Hkv, L, S, d):
    run_decoder_backward(oracle, B, Hq, Hkv, L, S, d)


def test_backward_deterministic_and_fully_written(oracle):
    """No atomics: two calls give the same bits; every output element is written (outputs that
    start as NaN end finite); encoder-side keys of the last block get exactly zero gradient (no
    decoder query attends them)."""
    B, Hq, Hkv, L, S, d = 1, 4, 2, 96, 16, 64
    q, ks = H.train_inputs(B, Hq, Hkv, L, d, 1.0, 900)
    g = H.gen((B, Hq, L, d), 909)
    ket, vet, kdt, vdt = (t[1] for t in ks)
    o, lse = attn.decoder_train(q[1], ket, vet, kdt, vdt, S)
    first = attn.decoder_train_backward(q[1], ket, vet, kdt, vdt, o, lse, g[1], S)
    n_ws = attn.train_backward_workspace_bytes(B, Hq, Hkv, d, L) // 4
    ws = torch.full((n_ws,), float("nan"), dtype=torch.float32, device="cuda")
    second = attn.decoder_train_backward(q[1], ket, vet, kdt, vdt, o, lse, g[1], S, workspace=ws)
    torch.cuda.synchronize()
    for a, b in zip(first, second):
        assert torch.isfinite(a.float()).all()
        assert torch.equal(a, b)
    dk_enc, dv_enc = first[1], first[2]
    assert torch.count_nonzero(dk_enc[:, :, L - S:]) == 0 and torch.count_nonzero(dv_enc[:, :, L - S:]) == 0
    assert attn.last_device_error() == 0


def test_train_pass_backward_full_size_sampled_heads(oracle):
    """Backward of the E2D2 train pass at full size (B8 L1024 S16 H16 d64); the oracle recomputes
    two (batch, head) pairs (heads are independent: Hq = Hkv)."""
    w = workloads.TRAIN
    B, Hq, L, d, S = w.batch, w.q_heads, w.L, w.head_dim, w.S
    q = H.gen((B, Hq, L, d), synth.seed_for(2, 0, "q"), w.sigma)
    k = H.gen((B, Hq, L, d), synth.seed_for(2, 0, "k"), w.sigma)
    v = H.gen((B, Hq, L, d), synth.seed_for(2, 0, "v"), w.sigma)
    ke = H.gen((B, Hq, L, d), synth.seed_for(2, 0, "k_enc"), w.sigma)
    ve = H.gen((B, Hq, L, d), synth.seed_for(2, 0, "v_enc"), w.sigma)
    g = H.gen((B, Hq, L, d), synth.seed_for(2, 0, "dout"))
    o_e, lse_e = attn.encoder_blockcausal(q[1], k[1], v[1], S)
    enc = attn.encoder_backward(q[1], k[1], v[1], o_e, lse_e, g[1], S)
    o_d, lse_d = attn.decoder_train(q[1], ke[1], ve[1], k[1], v[1], S)
    dec = attn.decoder_train_backward(q[1], ke[1], ve[1], k[1], v[1], o_d, lse_d, g[1], S)
    torch.cuda.synchronize()
    for b, h in ((0, 0), (5, 11)):
        sl = (slice(b, b + 1), slice(h, h + 1))
        ref = oracle.encoder_backward(q[0].f32[sl], k[0].f32[sl], v[0].f32[sl], g[0].f32[sl], S)
        for name, a, r in zip(("dq", "dk", "dv"), enc, ref):
            grad_compare(a[sl], r, f"train-pass encoder bwd b{b} h{h} {name}")
        ref = oracle.decoder_train_backward(q[0].f32[sl], ke[0].f32[sl], ve[0].f32[sl], k[0].f32[sl],
                                            v[0].f32[sl], g[0].f32[sl], S)
        for name, a, r in zip(("dq", "dk_enc", "dv_enc", "dk_dec", "dv_dec"), dec, ref):
            grad_compare(a[sl], r, f"train-pass decoder bwd b{b} h{h} {name}")
