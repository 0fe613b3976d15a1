"""BD3LM's training attention over its 2L tokens (noised copy first, then clean copy), the
comparison point of "Encoder-Decoder Diffusion Language Models for Efficient Training and
Inference" (paper notes, sec. 1 and the FLOPs table of sec. 4: BD3LM 4ND(L^2 + LS) against E2D2's
half of it at equal layer count), computed on the GPU as one decoder-train call (noised rows: their
own noised block and the clean blocks before it) plus one encoder call (clean rows, block-causal),
and compared element by element with the oracle's own 2L-token function, which builds the
2L x 2L mask explicitly (pinned on the CPU by pin_bd3lm_train).  Bars as for every forward call:
max |d out| <= 2e-2, per-row |d lse| <= 1e-3."""
import numpy as np
import pytest
import torch

from block_discrete_diffusion_tcgen05_b200 import attn, synth, workloads
import gpu_helpers as H

pytestmark = pytest.mark.gpu

CASES = [
    # B, Hq, Hkv, L, S, d
    (1, 2, 2, 64, 8, 32),       # tiny check shape
    (2, 4, 2, 200, 16, 64),     # ragged L, GQA 2
    (1, 2, 1, 130, 1, 128),     # S = 1
    (1, 4, 4, 256, 4, 64),      # translation-shaped block size
    (1, 2, 2, 100, 7, 64),      # short last block
]


def bd3lm_on_gpu(qn, kn, vn, qc, kc, vc, S):
    out_n, lse_n = attn.decoder_train(qn, kc, vc, kn, vn, S)
    out_c, lse_c = attn.encoder_blockcausal(qc, kc, vc, S)
    return torch.cat([out_n, out_c], dim=2), torch.cat([lse_n, lse_c], dim=2)


@pytest.mark.parametrize("B,Hq,Hkv,L,S,d", CASES)
def test_bd3lm_layer_matches_oracle(oracle, B, Hq, Hkv, L, S, d):
    qn, qc = (H.gen((B, Hq, L, d), 1300 + t) for t in range(2))
    kn, vn, kc, vc = (H.gen((B, Hkv, L, d), 1302 + t) for t in range(4))
    out, lse = bd3lm_on_gpu(qn[1], kn[1], vn[1], qc[1], kc[1], vc[1], S)
    torch.cuda.synchronize()
    cat = lambda a, b: np.concatenate([a[0].f32, b[0].f32], axis=2)
    ref_o, ref_l = oracle.bd3lm_train(cat(qn, qc), cat(kn, kc), cat(vn, vc), S)
    H.compare(out, lse, ref_o, ref_l, f"bd3lm B{B} Hq{Hq} Hkv{Hkv} L{L} S{S} d{d}")


def test_bd3lm_layer_full_size_sampled_heads(oracle):
    """The train-pass size (B8 L1024 S16 H16 d64); the oracle recomputes two (batch, head) pairs."""
    w = workloads.TRAIN
    B, Hq, L, d, S = w.batch, w.q_heads, w.L, w.head_dim, w.S
    names = ("q", "k", "v", "k_enc", "v_enc")
    qn, kn, vn, kc, vc = (H.gen((B, Hq, L, d), synth.seed_for(2, 1, n), w.sigma) for n in names)
    qc = H.gen((B, Hq, L, d), synth.seed_for(2, 2, "q"), w.sigma)
    out, lse = bd3lm_on_gpu(qn[1], kn[1], vn[1], qc[1], kc[1], vc[1], S)
    torch.cuda.synchronize()
    for b, h in ((1, 3), (7, 15)):
        sl = (slice(b, b + 1), slice(h, h + 1))
        cat = lambda a, c: np.concatenate([a[0].f32[sl], c[0].f32[sl]], axis=2)
        ref_o, ref_l = oracle.bd3lm_train(cat(qn, qc), cat(kn, kc), cat(vn, vc), S)
        H.compare(out[sl], lse[sl], ref_o, ref_l, f"bd3lm train-pass size b{b} h{h}")
