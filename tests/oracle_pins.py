"""Pins that tie the CPU oracle to facts that do not come from the oracle itself.

Each ``pin_*`` function takes an ``oracle.Oracle`` and raises AssertionError when the oracle
disagrees with the fact it pins.  ``tests/test_oracle_pins.py`` runs them on the real
oracle; ``tests/test_oracle_mutants.py`` plants plausible mistakes in copies of the oracle's
C source and checks that every mistake trips at least one pin.

Sources (page title, section):
  [E2D2 notes]  "Encoder-Decoder Diffusion Language Models for Efficient Training and
                Inference" (paper notes): sec. 3 sampling algorithm, sec. 4 training
                algorithm with its FLOPs table.
  [BD3LM blog]  "Block Diffusion: Interpolating Between Autoregressive and Diffusion
                Language Models": sec. 2 core insight (block size 1 = autoregressive,
                block size = sequence length = full diffusion).
"""
from __future__ import annotations

import math

import numpy as np
import torch

from block_discrete_diffusion_tcgen05_b200 import synth

GOLDEN_PAIRS = __import__("pathlib").Path(__file__).resolve().parent / "golden" / "pair_counts.txt"


def _rand(shape, seed, sigma=1.0):
    return synth.normal_bf16(shape, seed, sigma).f32


def _sdpa(q, k, v, scale, mask=None, causal=False):
    """torch's own attention routine in float64 on the CPU (a library routine)."""
    tq, tk, tv = (torch.from_numpy(np.asarray(x, dtype=np.float64)) for x in (q, k, v))
    m = None if mask is None else torch.from_numpy(mask)
    out = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=m,
                                                           is_causal=causal, scale=scale)
    return out.numpy()


def _torch_lse(q, k, scale, mask):
    """torch.logsumexp of the masked scaled scores (library routine)."""
    tq, tk = (torch.from_numpy(np.asarray(x, dtype=np.float64)) for x in (q, k))
    s = scale * torch.matmul(tq, tk.transpose(-1, -2))
    s = s.masked_fill(~torch.from_numpy(mask), float("-inf"))
    return torch.logsumexp(s, dim=-1).numpy()


# ---------------------------------------------------------------------------------------
# 1. Pair count: the FLOPs table of [E2D2 notes, sec. 4] charges an E2D2 encoder or decoder
#    pass with (L^2 + L S) / 2 attended pairs (attention FLOPs 4 (N_E+N_D) D (L^2+LS)/2).
# ---------------------------------------------------------------------------------------
def pin_pair_count(orc, cases=((8, 1), (8, 2), (8, 8), (12, 3), (16, 4), (64, 8), (48, 16), (32, 32))):
    for L, S in cases:
        closed = (L * L + L * S) // 2
        assert int(orc.mask_encoder(L, S).sum()) == closed, ("encoder", L, S)
        assert int(orc.mask_decoder(L, S).sum()) == closed, ("decoder", L, S)


def read_golden_pairs():
    rows = []
    for line in GOLDEN_PAIRS.read_text().splitlines():
        line = line.split("#", 1)[0].strip()
        if line:
            L, S, pairs = (int(x) for x in line.split())
            rows.append((L, S, pairs))
    return rows


def pin_golden_pairs(orc):
    for L, S, pairs in read_golden_pairs():
        assert int(orc.mask_encoder(L, S).sum()) == pairs, ("encoder", L, S)
        assert int(orc.mask_decoder(L, S).sum()) == pairs, ("decoder", L, S)


# ---------------------------------------------------------------------------------------
# 2. Block size 1 is autoregressive ([BD3LM blog, sec. 2]): the encoder mask is the causal
#    mask and the encoder output is torch's causal attention.
# ---------------------------------------------------------------------------------------
def pin_block_size_one_is_causal(orc):
    L, d, B, H = 24, 16, 2, 2
    assert np.array_equal(orc.mask_encoder(L, 1), np.tril(np.ones((L, L), dtype=bool)))
    q, k, v = (_rand((B, H, L, d), 900 + t) for t in range(3))
    scale = 0.31
    out, lse = orc.encoder(q, k, v, S=1, scale=scale)
    ref = _sdpa(q, k, v, scale, causal=True)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    causal = np.tril(np.ones((L, L), dtype=bool))
    np.testing.assert_allclose(lse, _torch_lse(q, k, scale, causal), rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------------------
# 3. Block size L is full diffusion ([BD3LM blog, sec. 2]): the encoder is bidirectional;
#    the decoder sees no encoder key (no earlier block) and its whole own block, i.e. plain
#    bidirectional attention over the decoder keys.
# ---------------------------------------------------------------------------------------
def pin_block_size_L_is_bidirectional(orc):
    L, d, B, H = 20, 8, 1, 3
    assert orc.mask_encoder(L, L).all()
    md = orc.mask_decoder(L, L)
    assert not md[:, :L].any() and md[:, L:].all()
    q, k, v, ke, ve = (_rand((B, H, L, d), 910 + t) for t in range(5))
    scale = 0.5
    out, lse = orc.encoder(q, k, v, S=L, scale=scale)
    np.testing.assert_allclose(out, _sdpa(q, k, v, scale), rtol=0, atol=1e-12)
    full = np.ones((L, L), dtype=bool)
    np.testing.assert_allclose(lse, _torch_lse(q, k, scale, full), rtol=0, atol=1e-12)
    out, lse = orc.decoder_train(q, ke, ve, k, v, S=L, scale=scale)
    np.testing.assert_allclose(out, _sdpa(q, k, v, scale), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, _torch_lse(q, k, scale, full), rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------------------
# 4. Intermediate block sizes against torch's attention with a mask built here from the
#    mask words of [E2D2 notes, sec. 4] (block ids compared with numpy broadcasting).
# ---------------------------------------------------------------------------------------
def _block_ids(L, S):
    return np.arange(L) // S


def pin_masked_against_torch(orc):
    B, Hq, Hkv, L, S, d = 2, 4, 2, 24, 4, 8
    G = Hq // Hkv
    q = _rand((B, Hq, L, d), 920)
    k, v, ke, ve = (_rand((B, Hkv, L, d), 921 + t) for t in range(4))
    scale = 0.4
    bid = _block_ids(L, S)
    enc_mask = bid[None, :] <= bid[:, None]
    kr, vr = np.repeat(k, G, axis=1), np.repeat(v, G, axis=1)
    out, lse = orc.encoder(q, k, v, S=S, scale=scale)
    np.testing.assert_allclose(out, _sdpa(q, kr, vr, scale, mask=enc_mask), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, _torch_lse(q, kr, scale, enc_mask), rtol=0, atol=1e-12)
    # decoder: keys = [encoder keys | decoder keys]
    dec_mask = np.concatenate([bid[None, :] < bid[:, None], bid[None, :] == bid[:, None]], axis=1)
    kcat = np.concatenate([np.repeat(ke, G, 1), kr], axis=2)
    vcat = np.concatenate([np.repeat(ve, G, 1), vr], axis=2)
    out, lse = orc.decoder_train(q, ke, ve, k, v, S=S, scale=scale)
    np.testing.assert_allclose(out, _sdpa(q, kcat, vcat, scale, mask=dec_mask), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, _torch_lse(q, kcat, scale, dec_mask), rtol=0, atol=1e-12)
    # scale <= 0 selects the default softmax scale; torch's routine defaults to 1/sqrt(d).
    out, _ = orc.encoder(q, k, v, S=S, scale=0.0)
    np.testing.assert_allclose(out, _sdpa(q, kr, vr, None, mask=enc_mask), rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------------------
# 5. Brute force on tiny inputs: allowed keys listed as index ranges (not compared element
#    by element), scores and sums with math.fsum, one query at a time.
# ---------------------------------------------------------------------------------------
def _brute_row(qrow, keys, vals, scale):
    scores = [scale * math.fsum(a * b for a, b in zip(qrow, kk)) for kk in keys]
    m = max(scores)
    w = [math.exp(s - m) for s in scores]
    tot = math.fsum(w)
    d = len(vals[0])
    out = [math.fsum(wi * vv[c] for wi, vv in zip(w, vals)) / tot for c in range(d)]
    return out, m + math.log(tot)


def pin_brute_force(orc):
    B, Hq, Hkv, L, S, d = 1, 2, 1, 12, 3, 4
    q = _rand((B, Hq, L, d), 930).astype(np.float64)
    k, v, ke, ve = (_rand((B, Hkv, L, d), 931 + t).astype(np.float64) for t in range(4))
    scale = 0.7
    out_e, lse_e = orc.encoder(q, k, v, S=S, scale=scale)
    out_d, lse_d = orc.decoder_train(q, ke, ve, k, v, S=S, scale=scale)
    for h in range(Hq):
        g = h // (Hq // Hkv)
        for i in range(L):
            b0 = (i // S) * S  # first position of the query's block
            enc_keys = list(range(0, b0 + S))  # own block and every earlier block
            o, l = _brute_row(q[0, h, i], [k[0, g, j] for j in enc_keys], [v[0, g, j] for j in enc_keys], scale)
            np.testing.assert_allclose(out_e[0, h, i], o, rtol=0, atol=1e-12)
            assert abs(lse_e[0, h, i] - l) < 1e-12
            keys = [ke[0, g, j] for j in range(0, b0)] + [k[0, g, j] for j in range(b0, b0 + S)]
            vals = [ve[0, g, j] for j in range(0, b0)] + [v[0, g, j] for j in range(b0, b0 + S)]
            o, l = _brute_row(q[0, h, i], keys, vals, scale)
            np.testing.assert_allclose(out_d[0, h, i], o, rtol=0, atol=1e-12)
            assert abs(lse_d[0, h, i] - l) < 1e-12
    # sampling step: every query sees the P prefix rows and the S own rows
    P, cap = 5, 9
    qs = _rand((B, Hq, S, d), 940).astype(np.float64)
    kc, vc = (_rand((B, Hkv, cap, d), 941 + t).astype(np.float64) for t in range(2))
    kb, vb = (_rand((B, Hkv, S, d), 943 + t).astype(np.float64) for t in range(2))
    out_s, lse_s = orc.decoder_sample(qs, kc, vc, P, kb, vb, scale=scale)
    for h in range(Hq):
        g = h // (Hq // Hkv)
        keys = [kc[0, g, j] for j in range(P)] + [kb[0, g, j] for j in range(S)]
        vals = [vc[0, g, j] for j in range(P)] + [vb[0, g, j] for j in range(S)]
        for i in range(S):
            o, l = _brute_row(qs[0, h, i], keys, vals, scale)
            np.testing.assert_allclose(out_s[0, h, i], o, rtol=0, atol=1e-12)
            assert abs(lse_s[0, h, i] - l) < 1e-12


# ---------------------------------------------------------------------------------------
# 6. Closed form with all-zero keys: every allowed score is 0, so lse_i = ln(n_i) and out_i
#    is the mean of the allowed values.  n_i = (block(i) + 1) S for both train passes
#    ([E2D2 notes, sec. 4]: own block plus every earlier block, from one side or the other)
#    and P + S for the sampling step.
# ---------------------------------------------------------------------------------------
def pin_zero_keys_closed_form(orc):
    B, H, L, S, d = 1, 2, 16, 4, 4
    q = _rand((B, H, L, d), 950)
    v, ve = _rand((B, H, L, d), 951), _rand((B, H, L, d), 952)
    z = np.zeros((B, H, L, d), dtype=np.float32)
    out, lse = orc.encoder(q, z, v, S=S)
    for i in range(L):
        n = (i // S + 1) * S
        np.testing.assert_allclose(lse[:, :, i], math.log(n), rtol=0, atol=1e-13)
        np.testing.assert_allclose(out[:, :, i], v[:, :, :n].astype(np.float64).mean(axis=2), rtol=0, atol=1e-12)
    out, lse = orc.decoder_train(q, z, ve, z, v, S=S)
    for i in range(L):
        b0 = (i // S) * S
        n = b0 + S
        mean = (ve[:, :, :b0].astype(np.float64).sum(axis=2) + v[:, :, b0:b0 + S].astype(np.float64).sum(axis=2)) / n
        np.testing.assert_allclose(lse[:, :, i], math.log(n), rtol=0, atol=1e-13)
        np.testing.assert_allclose(out[:, :, i], mean, rtol=0, atol=1e-12)
    P, cap = 7, 11
    qs = _rand((B, H, S, d), 953)
    vc, vb = _rand((B, H, cap, d), 954), _rand((B, H, S, d), 955)
    out, lse = orc.decoder_sample(qs, np.zeros((B, H, cap, d), np.float32), vc, P,
                                  np.zeros((B, H, S, d), np.float32), vb)
    mean = (vc[:, :, :P].astype(np.float64).sum(axis=2) + vb.astype(np.float64).sum(axis=2)) / (P + S)
    np.testing.assert_allclose(lse, math.log(P + S), rtol=0, atol=1e-13)
    np.testing.assert_allclose(out, np.repeat(mean[:, :, None, :], S, axis=2), rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------------------
# 7. Invariants: constant values give that constant; GQA equals MHA with repeated kv heads.
# ---------------------------------------------------------------------------------------
def pin_constant_values(orc):
    B, H, L, S, d = 1, 2, 16, 4, 8
    q, k = _rand((B, H, L, d), 960), _rand((B, H, L, d), 961)
    c = np.full((B, H, L, d), 0.375, dtype=np.float32)
    out, _ = orc.encoder(q, k, c, S=S)
    np.testing.assert_allclose(out, 0.375, rtol=0, atol=1e-14)
    out, _ = orc.decoder_train(q, k, c, k, c, S=S)
    np.testing.assert_allclose(out, 0.375, rtol=0, atol=1e-14)


def pin_gqa_is_repeated_heads(orc):
    B, Hq, Hkv, L, S, d = 1, 6, 2, 16, 4, 8
    G = Hq // Hkv
    q = _rand((B, Hq, L, d), 970)
    k, v, ke, ve = (_rand((B, Hkv, L, d), 971 + t) for t in range(4))
    rep = lambda t: np.repeat(t, G, axis=1)
    a = orc.encoder(q, k, v, S=S)
    b = orc.encoder(q, rep(k), rep(v), S=S)
    np.testing.assert_array_equal(a[0], b[0])
    a = orc.decoder_train(q, ke, ve, k, v, S=S)
    b = orc.decoder_train(q, rep(ke), rep(ve), rep(k), rep(v), S=S)
    np.testing.assert_array_equal(a[0], b[0])
    P, cap = 6, 8
    kc, vc = _rand((B, Hkv, cap, d), 975), _rand((B, Hkv, cap, d), 976)
    qs = _rand((B, Hq, S, d), 977)
    a = orc.decoder_sample(qs, kc, vc, P, k[:, :, :S], v[:, :, :S])
    b = orc.decoder_sample(qs, rep(kc), rep(vc), P, rep(k[:, :, :S]), rep(v[:, :, :S]))
    np.testing.assert_array_equal(a[0], b[0])


# ---------------------------------------------------------------------------------------
# 8. Sampling step == the matching rows of the training pass ([E2D2 notes, sec. 3 vs 4]):
#    the noised block b with the encoder cache of blocks < b gives the decoder-train rows of
#    block b; the encoder rows of block b are a sampling-shaped call over prefix [0, bS)
#    plus the block itself.
# ---------------------------------------------------------------------------------------
def pin_sample_is_train_slice(orc):
    B, Hq, Hkv, L, S, d = 2, 4, 2, 20, 5, 8
    q = _rand((B, Hq, L, d), 980)
    k, v, ke, ve = (_rand((B, Hkv, L, d), 981 + t) for t in range(4))
    scale = 0.3
    out_d, lse_d = orc.decoder_train(q, ke, ve, k, v, S=S, scale=scale)
    out_e, lse_e = orc.encoder(q, k, v, S=S, scale=scale)
    for blk in range(L // S):
        r = slice(blk * S, blk * S + S)
        o, l = orc.decoder_sample(q[:, :, r], ke, ve, blk * S, k[:, :, r], v[:, :, r], scale=scale)
        np.testing.assert_allclose(o, out_d[:, :, r], rtol=0, atol=1e-13)
        np.testing.assert_allclose(l, lse_d[:, :, r], rtol=0, atol=1e-13)
        o, l = orc.decoder_sample(q[:, :, r], k, v, blk * S, k[:, :, r], v[:, :, r], scale=scale)
        np.testing.assert_allclose(o, out_e[:, :, r], rtol=0, atol=1e-13)
        np.testing.assert_allclose(l, lse_e[:, :, r], rtol=0, atol=1e-13)


# ---------------------------------------------------------------------------------------
# 9. KV-cache append is array concatenation ([E2D2 notes, sec. 3]: the cache grows by the
#    decoded block); rows outside [P, P+S_new) are untouched.
# ---------------------------------------------------------------------------------------
def pin_append_is_concatenation(orc):
    B, Hkv, cap, d = 2, 3, 12, 8
    rng = np.random.default_rng(990)
    kc = rng.integers(0, 65535, size=(B, Hkv, cap, d), dtype=np.uint16)
    vc = rng.integers(0, 65535, size=(B, Hkv, cap, d), dtype=np.uint16)
    P = 0
    kc0, vc0 = kc.copy(), vc.copy()
    pieces_k, pieces_v = [], []
    for S_new in (3, 4, 2):
        kn = rng.integers(0, 65535, size=(B, Hkv, S_new, d), dtype=np.uint16)
        vn = rng.integers(0, 65535, size=(B, Hkv, S_new, d), dtype=np.uint16)
        orc.kv_append(kc, vc, P, kn, vn)
        pieces_k.append(kn)
        pieces_v.append(vn)
        P += S_new
    np.testing.assert_array_equal(kc[:, :, :P], np.concatenate(pieces_k, axis=2))
    np.testing.assert_array_equal(vc[:, :, :P], np.concatenate(pieces_v, axis=2))
    np.testing.assert_array_equal(kc[:, :, P:], kc0[:, :, P:])
    np.testing.assert_array_equal(vc[:, :, P:], vc0[:, :, P:])


# ---------------------------------------------------------------------------------------
# 12. Short last block (the block-diffusion page lets the last block be shorter when S does not
#     divide L): with L = n S + r, 0 < r < S, full block b has S rows attending (b + 1) S keys and
#     the r rows of the last block attend all L keys, so both masks hold S^2 n (n+1)/2 + r L
#     pairs; S >= L is one block (n = 0, r = L: L^2 pairs).  A brute-force check on a tiny case
#     takes the block rule with the last block clipped at L.
# ---------------------------------------------------------------------------------------
def pin_short_last_block(orc):
    for L, S in ((10, 4), (13, 5), (7, 3), (100, 16), (200, 48), (5, 8), (9, 9)):
        n, r = L // S, L % S
        closed = S * S * n * (n + 1) // 2 + r * L
        assert int(orc.mask_encoder(L, S).sum()) == closed, ("encoder", L, S)
        assert int(orc.mask_decoder(L, S).sum()) == closed, ("decoder", L, S)
    B, Hq, Hkv, L, S, d = 1, 2, 2, 10, 4, 4
    q = _rand((B, Hq, L, d), 970).astype(np.float64)
    k, v, ke, ve = (_rand((B, Hkv, L, d), 971 + t).astype(np.float64) for t in range(4))
    scale = 0.6
    out_e, lse_e = orc.encoder(q, k, v, S=S, scale=scale)
    out_d, lse_d = orc.decoder_train(q, ke, ve, k, v, S=S, scale=scale)
    for h in range(Hq):
        for i in range(L):
            b0 = (i // S) * S
            end = min(L, b0 + S)  # the last block stops at L
            o, l = _brute_row(q[0, h, i], [k[0, h, j] for j in range(end)], [v[0, h, j] for j in range(end)], scale)
            np.testing.assert_allclose(out_e[0, h, i], o, rtol=0, atol=1e-12)
            assert abs(lse_e[0, h, i] - l) < 1e-12
            keys = [ke[0, h, j] for j in range(b0)] + [k[0, h, j] for j in range(b0, end)]
            vals = [ve[0, h, j] for j in range(b0)] + [v[0, h, j] for j in range(b0, end)]
            o, l = _brute_row(q[0, h, i], keys, vals, scale)
            np.testing.assert_allclose(out_d[0, h, i], o, rtol=0, atol=1e-12)
            assert abs(lse_d[0, h, i] - l) < 1e-12


# ---------------------------------------------------------------------------------------
# 13. Decoder-only block diffusion (BD3LM) for comparison: its training forward takes the clean
#     and the noised sequence together (2L tokens) at attention cost 4ND(L^2 + LS) ([E2D2 notes],
#     sec. 1 and the FLOPs table of sec. 4).  Read as: noised tokens see the noised tokens of their
#     own block and the clean tokens of earlier blocks, clean tokens are block-causal.  That mask
#     has L^2 + LS pairs (twice one E2D2 pass), and it is the decoder mask on the noised rows and
#     the encoder mask on the clean rows; attention over the 2L tokens (torch SDPA on the explicit
#     mask) equals one encoder call plus one decoder-train call with the same network's K/V.
# ---------------------------------------------------------------------------------------
def pin_bd3lm_vectorized_mask(orc):
    for L, S in ((8, 2), (12, 3), (16, 4), (64, 8), (48, 16)):
        blk = np.arange(L) // S
        nn = blk[:, None] == blk[None, :]  # noised -> noised: own block
        nc = blk[None, :] < blk[:, None]   # noised -> clean: earlier blocks
        cc = blk[None, :] <= blk[:, None]  # clean -> clean: block-causal
        full = np.block([[nn, nc], [np.zeros((L, L), dtype=bool), cc]])
        assert int(full.sum()) == L * L + L * S, (L, S)
        dec = orc.mask_decoder(L, S).astype(bool)  # columns 0..L-1 clean (encoder), L..2L-1 noised
        assert (dec[:, :L] == nc).all() and (dec[:, L:] == nn).all(), (L, S)
        assert (orc.mask_encoder(L, S).astype(bool) == cc).all(), (L, S)
    B, H, L, S, d = 1, 2, 12, 4, 8
    qn, kn, vn, qc, kc, vc = (_rand((B, H, L, d), 990 + t).astype(np.float64) for t in range(6))
    blk = np.arange(L) // S
    full = np.block([[blk[:, None] == blk[None, :], blk[None, :] < blk[:, None]],
                     [np.zeros((L, L), dtype=bool), blk[None, :] <= blk[:, None]]])
    q2, k2, v2 = (torch.from_numpy(np.concatenate(x, axis=2)) for x in ((qn, qc), (kn, kc), (vn, vc)))
    ref = torch.nn.functional.scaled_dot_product_attention(q2, k2, v2, attn_mask=torch.from_numpy(full)).numpy()
    out_n, _ = orc.decoder_train(qn, kc, vc, kn, vn, S=S)
    out_c, _ = orc.encoder(qc, kc, vc, S=S)
    np.testing.assert_allclose(out_n, ref[:, :, :L], rtol=0, atol=1e-10)
    np.testing.assert_allclose(out_c, ref[:, :, L:], rtol=0, atol=1e-10)


# ---------------------------------------------------------------------------------------
# 13b. BD3LM's attention over its 2L training tokens as its own oracle function (the comparison
#      point of the FLOPs table): (a) pair count L^2 + LS, the table's 4ND(L^2+LS) per layer over
#      4D; (b) the mask equals one built here from numpy block ids; (c) the output equals torch's
#      SDPA in fp64 on that mask (GQA through repeated kv heads); (d) the noised rows equal the
#      decoder-train call and the clean rows the encoder call on the same tensors (two definitions
#      that must agree); (e) S = L: every row attends bidirectionally within its own copy.
# ---------------------------------------------------------------------------------------
def _bd3lm_mask(L, S):
    blk = np.arange(L) // S
    return np.block([[blk[:, None] == blk[None, :], blk[None, :] < blk[:, None]],
                     [np.zeros((L, L), dtype=bool), blk[None, :] <= blk[:, None]]])


def pin_bd3lm_train(orc):
    for L, S in ((8, 1), (8, 2), (12, 3), (16, 4), (64, 8), (48, 16), (32, 32)):
        m = orc.mask_bd3lm(L, S)
        assert int(m.sum()) == L * L + L * S, (L, S)
        assert (m == _bd3lm_mask(L, S)).all(), (L, S)
    B, Hq, Hkv, L, S, d, scale = 2, 4, 2, 20, 5, 8, 0.4
    G = Hq // Hkv
    qn, qc = (_rand((B, Hq, L, d), 1200 + t) for t in range(2))
    kn, vn, kc, vc = (_rand((B, Hkv, L, d), 1202 + t) for t in range(4))
    q2, k2, v2 = (np.concatenate(x, axis=2) for x in ((qn, qc), (kn, kc), (vn, vc)))
    out, lse = orc.bd3lm_train(q2, k2, v2, S, scale=scale)
    m = _bd3lm_mask(L, S)
    kr, vr = np.repeat(k2, G, axis=1), np.repeat(v2, G, axis=1)
    np.testing.assert_allclose(out, _sdpa(q2, kr, vr, scale, mask=m), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, _torch_lse(q2, kr, scale, np.broadcast_to(m, lse.shape + (2 * L,))),
                               rtol=0, atol=1e-12)
    on, ln = orc.decoder_train(qn, kc, vc, kn, vn, S=S, scale=scale)
    oc, lc = orc.encoder(qc, kc, vc, S=S, scale=scale)
    np.testing.assert_allclose(out[:, :, :L], on, rtol=0, atol=1e-13)
    np.testing.assert_allclose(out[:, :, L:], oc, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse[:, :, :L], ln, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse[:, :, L:], lc, rtol=0, atol=1e-13)
    out, _ = orc.bd3lm_train(q2, k2, v2, L, scale=scale)
    np.testing.assert_allclose(out[:, :, :L], _sdpa(qn, np.repeat(kn, G, 1), np.repeat(vn, G, 1), scale),
                               rtol=0, atol=1e-12)
    np.testing.assert_allclose(out[:, :, L:], _sdpa(qc, np.repeat(kc, G, 1), np.repeat(vc, G, 1), scale),
                               rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------------------
# 14. Backward of the train calls ([E2D2 notes, sec. 4]: one encoder and one decoder pass, forward
#     and backward).  (a) torch autograd in fp64 through SDPA on masks built here from the block
#     rule (GQA through repeated kv heads, whose gradients autograd sums; a short last block);
#     (b) central differences of the oracle's forward on exactly representable inputs;
#     (c) constant values: out does not depend on q or k (dq = dk = 0) and the dv rows sum to the
#     dout rows (every softmax row sums to one).
# ---------------------------------------------------------------------------------------
def _block_masks(L, S):
    blk = np.arange(L) // S
    enc = blk[None, :] <= blk[:, None]
    dec = np.concatenate([blk[None, :] < blk[:, None], blk[None, :] == blk[:, None]], axis=1)
    return enc, dec


def pin_backward_against_autograd(orc):
    B, Hq, Hkv, L, S, d, scale = 2, 4, 2, 20, 6, 8, 0.5
    G = Hq // Hkv
    q, dout = (_rand((B, Hq, L, d), 1000 + t) for t in range(2))
    k, v, ke, ve = (_rand((B, Hkv, L, d), 1002 + t) for t in range(4))
    enc_m, dec_m = (torch.from_numpy(m) for m in _block_masks(L, S))
    t64 = lambda a: torch.tensor(np.asarray(a, dtype=np.float64), requires_grad=True)
    rep = lambda t: t.repeat_interleave(G, dim=1)
    sdpa = torch.nn.functional.scaled_dot_product_attention
    g = torch.from_numpy(np.asarray(dout, dtype=np.float64))
    # encoder
    tq, tk, tv = t64(q), t64(k), t64(v)
    (sdpa(tq, rep(tk), rep(tv), attn_mask=enc_m, scale=scale) * g).sum().backward()
    dq, dk, dv = orc.encoder_backward(q, k, v, dout, S=S, scale=scale)
    for mine, ref in ((dq, tq), (dk, tk), (dv, tv)):
        np.testing.assert_allclose(mine, ref.grad.numpy(), rtol=0, atol=1e-10)
    # decoder-train: keys are the encoder-side rows, then the decoder-side rows
    tq, tke, tve, tkd, tvd = t64(q), t64(ke), t64(ve), t64(k), t64(v)
    kk, vv = torch.cat([rep(tke), rep(tkd)], dim=2), torch.cat([rep(tve), rep(tvd)], dim=2)
    (sdpa(tq, kk, vv, attn_mask=dec_m, scale=scale) * g).sum().backward()
    grads = orc.decoder_train_backward(q, ke, ve, k, v, dout, S=S, scale=scale)
    for mine, ref in zip(grads, (tq, tke, tve, tkd, tvd)):
        np.testing.assert_allclose(mine, ref.grad.numpy(), rtol=0, atol=1e-10)


def pin_backward_finite_differences(orc):
    B, Hq, Hkv, L, S, d, scale = 1, 1, 1, 5, 2, 3, 0.8
    rng = np.random.default_rng(1010)
    grid = lambda shape: (rng.integers(-512, 512, size=shape) / 1024.0).astype(np.float32)  # exact in fp32
    q, k, v, ke, ve, dout = (grid((B, Hq, L, d)) for _ in range(6))
    h = np.float32(2.0 ** -8)

    def f_enc(qq, kk, vv):
        return float((orc.encoder(qq, kk, vv, S=S, scale=scale)[0] * dout).sum())

    def f_dec(qq, kke, vve, kkd, vvd):
        return float((orc.decoder_train(qq, kke, vve, kkd, vvd, S=S, scale=scale)[0] * dout).sum())

    grads_e = orc.encoder_backward(q, k, v, dout, S=S, scale=scale)
    grads_d = orc.decoder_train_backward(q, ke, ve, k, v, dout, S=S, scale=scale)
    for f, args, grads in ((f_enc, [q, k, v], grads_e), (f_dec, [q, ke, ve, k, v], grads_d)):
        for a, ga in zip(range(len(args)), grads):
            for idx in ((0, 0, 0, 0), (0, 0, 2, 1), (0, 0, L - 1, d - 1), (0, 0, 3, 2)):
                plus = [x.copy() for x in args]
                minus = [x.copy() for x in args]
                plus[a][idx] += h
                minus[a][idx] -= h
                num = (f(*plus) - f(*minus)) / (2.0 * float(h))
                assert abs(num - ga[idx]) <= 2e-4 + 2e-3 * abs(ga[idx]), (f.__name__, a, idx, num, ga[idx])
    # constant values
    vc = np.full_like(v, 0.375)
    dq, dk, dv = orc.encoder_backward(q, k, vc, dout, S=S, scale=scale)
    assert np.abs(dq).max() < 1e-12 and np.abs(dk).max() < 1e-12
    np.testing.assert_allclose(dv.sum(axis=2), dout.astype(np.float64).sum(axis=2), rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------------------
# Ragged prefixes: a batch whose entries have decoded different numbers of clean tokens.  The
# plainest reading of the sampling step of [E2D2 notes, sec. 3] for such a batch: entry b sees
# the first P[b] rows of its own cache and its own block.  Pinned against torch's attention
# routine with an explicit per-entry mask over [whole cache ; block], the cache rows at or past
# each entry's prefix filled with large values that must not matter, and entry by entry against
# the single-prefix step (itself pinned above).
# ---------------------------------------------------------------------------------------
def pin_ragged_prefix_against_torch(orc):
    B, Hq, Hkv, S, cap, d = 5, 4, 2, 5, 23, 8
    G = Hq // Hkv
    P = [0, 7, 23, 12, 5]   # empty prefix, unaligned, full capacity, unaligned, one block
    q = _rand((B, Hq, S, d), 1100)
    kc, vc = _rand((B, Hkv, cap, d), 1101), _rand((B, Hkv, cap, d), 1102)
    kb, vb = _rand((B, Hkv, S, d), 1103), _rand((B, Hkv, S, d), 1104)
    for b, pb in enumerate(P):
        kc[b, :, pb:] = 8192.0
        vc[b, :, pb:] = -8192.0
    scale = 0.4
    out, lse = orc.decoder_sample_ragged(q, kc, vc, P, kb, vb, scale=scale)
    keys = np.repeat(np.concatenate([kc, kb], axis=2), G, axis=1)
    vals = np.repeat(np.concatenate([vc, vb], axis=2), G, axis=1)
    mask = np.zeros((B, 1, S, cap + S), dtype=bool)
    for b, pb in enumerate(P):
        mask[b, :, :, :pb] = True
        mask[b, :, :, cap:] = True
    np.testing.assert_allclose(out, _sdpa(q, keys, vals, scale, mask=mask), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, _torch_lse(q, keys, scale, mask), rtol=0, atol=1e-12)
    for b, pb in enumerate(P):
        sl = slice(b, b + 1)
        o, l = orc.decoder_sample(q[sl], kc[sl], vc[sl], pb, kb[sl], vb[sl], scale=scale)
        np.testing.assert_allclose(out[sl], o, rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse[sl], l, rtol=0, atol=1e-13)


ALL_PINS = [pin_pair_count, pin_golden_pairs, pin_block_size_one_is_causal,
            pin_block_size_L_is_bidirectional, pin_masked_against_torch, pin_brute_force,
            pin_zero_keys_closed_form, pin_constant_values, pin_gqa_is_repeated_heads,
            pin_sample_is_train_slice, pin_append_is_concatenation, pin_short_last_block,
            pin_bd3lm_vectorized_mask, pin_bd3lm_train, pin_backward_against_autograd,
            pin_backward_finite_differences, pin_ragged_prefix_against_torch]
