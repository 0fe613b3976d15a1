"""Shared helpers of the GPU parity tests: seeded inputs (synth), the CUDA path through the
C ABI (block_discrete_diffusion_tcgen05_b200.attn) and the CPU oracle, compared element by
element.  Tolerances are the ones the attention is specified to: max |d out| <= 2e-2 and per-row
|d lse| <= 1e-3 between the bf16-in / fp32-accumulate GPU result and the fp64 oracle."""
from __future__ import annotations

import numpy as np
import torch

from block_discrete_diffusion_tcgen05_b200 import attn, synth

OUT_TOL = 2e-2
LSE_TOL = 1e-3


def gen(shape, seed, sigma=1.0):
    a = synth.normal_bf16(shape, seed, sigma)
    return a, synth.to_torch(a, "cuda")


def compare(out_gpu, lse_gpu, out_ref, lse_ref, what=""):
    o = out_gpu.float().cpu().numpy().astype(np.float64)
    l = lse_gpu.cpu().numpy().astype(np.float64)
    assert np.isfinite(o).all(), f"{what}: non-finite output"
    assert np.isfinite(l).all(), f"{what}: non-finite lse"
    dout = np.abs(o - out_ref).max()
    dlse = np.abs(l - lse_ref).max()
    assert dout <= OUT_TOL, f"{what}: max|d out| = {dout:.3e} > {OUT_TOL}"
    assert dlse <= LSE_TOL, f"{what}: max|d lse| = {dlse:.3e} > {LSE_TOL}"
    return dout, dlse


def train_inputs(B, Hq, Hkv, L, d, sigma, seed0):
    """Q and the keys scaled by sigma (sigma > 1 sharpens the softmax); values stay N(0, 1) so
    outputs stay O(1), the range the absolute output tolerance is stated for."""
    q = gen((B, Hq, L, d), seed0 + 0, sigma)
    ks = [gen((B, Hkv, L, d), seed0 + t, sigma if t % 2 == 1 else 1.0) for t in range(1, 5)]
    return q, ks


def run_encoder_case(orc, B, Hq, Hkv, L, S, d, sigma=1.0, seed0=100):
    q, ks = train_inputs(B, Hq, Hkv, L, d, sigma, seed0)
    (k, kt), (v, vt) = ks[0], ks[1]
    out, lse = attn.encoder_blockcausal(q[1], kt, vt, S)
    torch.cuda.synchronize()
    ref_o, ref_l = orc.encoder(q[0].f32, k.f32, v.f32, S)
    return compare(out, lse, ref_o, ref_l, f"encoder B{B} Hq{Hq} Hkv{Hkv} L{L} S{S} d{d}")


def run_decoder_case(orc, B, Hq, Hkv, L, S, d, sigma=1.0, seed0=200):
    q, ks = train_inputs(B, Hq, Hkv, L, d, sigma, seed0)
    (ke, ket), (ve, vet), (kd, kdt), (vd, vdt) = ks
    out, lse = attn.decoder_train(q[1], ket, vet, kdt, vdt, S)
    torch.cuda.synchronize()
    ref_o, ref_l = orc.decoder_train(q[0].f32, ke.f32, ve.f32, kd.f32, vd.f32, S)
    return compare(out, lse, ref_o, ref_l, f"decoder B{B} Hq{Hq} Hkv{Hkv} L{L} S{S} d{d}")


def sample_inputs(B, Hq, Hkv, S, cap, d, sigma, seed0):
    # sigma sharpens the scores (Q, K); V stays N(0, 1) so the output tolerance keeps its meaning
    q = gen((B, Hq, S, d), seed0, sigma)
    kc = gen((B, Hkv, cap, d), seed0 + 1, sigma)
    vc = gen((B, Hkv, cap, d), seed0 + 2, 1.0)
    kb = gen((B, Hkv, S, d), seed0 + 3, sigma)
    vb = gen((B, Hkv, S, d), seed0 + 4, 1.0)
    return q, kc, vc, kb, vb


def run_sample_case(orc, B, Hq, Hkv, S, P, cap, d, sigma=1.0, seed0=300, poison_tail=True):
    q, kc, vc, kb, vb = sample_inputs(B, Hq, Hkv, S, cap, d, sigma, seed0)
    if poison_tail and cap > P:
        # Rows beyond P must never be read: make them NaN on the device copy.
        for t in (kc[1], vc[1]):
            t[:, :, P:, :] = float("nan")
    out, lse = attn.decoder_sample(q[1], kc[1], vc[1], P, kb[1], vb[1])
    torch.cuda.synchronize()
    ref_o, ref_l = orc.decoder_sample(q[0].f32, kc[0].f32, vc[0].f32, P, kb[0].f32, vb[0].f32)
    return compare(out, lse, ref_o, ref_l, f"sample B{B} Hq{Hq} Hkv{Hkv} S{S} P{P} d{d}")
