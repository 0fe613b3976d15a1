"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle, element by element.

Shapes span several 128-row tiles, ragged tails (L or P not a multiple of 128, S not a
multiple of 16), block sizes from 1 (causal) to L (bidirectional), head_dim 32/64/128, GQA
ratios 1/2/4, split-KV sampling with P = 0 and with several query tiles per kv head.  The full
sizes of the E2D2 train pass and sampling step are checked on sampled heads (exact: heads are
independent)."""
import numpy as np
import pytest
import torch

from block_discrete_diffusion_tcgen05_b200 import attn, synth, workloads
import gpu_helpers as H

pytestmark = pytest.mark.gpu

TRAIN_CASES = [
    # B, Hq, Hkv, L, S, d, sigma
    (1, 2, 2, 64, 8, 32, 1.0),       # tiny check workload
    (2, 4, 4, 256, 16, 64, 64 ** -0.25),
    (1, 2, 2, 200, 8, 64, 1.0),      # ragged L
    (1, 2, 1, 384, 1, 64, 1.0),      # S = 1: causal; GQA 2
    (1, 2, 2, 256, 256, 64, 1.0),    # S = L: bidirectional
    (1, 2, 2, 320, 64, 128, 1.0),    # d = 128
    (1, 4, 2, 192, 48, 32, 1.0),     # S does not divide the 128-key tile
    (1, 8, 2, 256, 32, 64, 3.0),     # sharp softmax, GQA 4
    (1, 2, 2, 130, 130, 64, 1.0),    # S = L, ragged
    (2, 2, 2, 512, 4, 64, 1.0),      # translation-shaped block size
    (1, 1, 1, 1024, 16, 64, 1.0),    # many tiles per row
    # short last block (S does not divide L) and S > L (one block)
    (1, 2, 2, 200, 48, 64, 1.0),     # blocks of 48, last one 8 rows
    (1, 4, 2, 300, 7, 32, 1.0),      # last block 6 rows, GQA 2, d 32
    (2, 2, 2, 130, 16, 128, 1.0),    # last block 2 rows, d 128
    (1, 2, 1, 100, 160, 64, 1.0),    # S > L
]


@pytest.mark.parametrize("B,Hq,Hkv,L,S,d,sigma", TRAIN_CASES)
def test_encoder_parity(oracle, B, Hq, Hkv, L, S, d, sigma):
    H.run_encoder_case(oracle, B, Hq, Hkv, L, S, d, sigma)


@pytest.mark.parametrize("B,Hq,Hkv,L,S,d,sigma", TRAIN_CASES)
def test_decoder_train_parity(oracle, B, Hq, Hkv, L, S, d, sigma):
    H.run_decoder_case(oracle, B, Hq, Hkv, L, S, d, sigma)


SAMPLE_CASES = [
    # B, Hq, Hkv, S, P, cap, d
    (2, 4, 2, 16, 0, 64, 128),        # first block: no prefix
    (2, 4, 2, 16, 5, 64, 128),
    (2, 4, 2, 16, 128, 160, 128),     # prefix = one tile
    (2, 16, 8, 16, 1000, 1100, 128),
    (4, 32, 8, 16, 2048, 2064, 128),  # long-context loop shape (G = 4)
    (2, 4, 1, 64, 300, 400, 128),     # G*S = 256: two query tiles per kv head
    (3, 4, 4, 4, 700, 800, 64),
    (2, 2, 2, 16, 333, 400, 32),
    (1, 8, 2, 100, 513, 600, 128),    # S not a multiple of 16; 4 query tiles
    (1, 2, 2, 1, 129, 130, 64),       # S = 1
    # d = 128 with G*S <= 64: the keys-on-lanes kernel (S^T = K Q^T)
    (2, 8, 8, 8, 700, 720, 128),      # G*S = 8: 16 packed columns, 8 of them padding
    (3, 6, 2, 5, 260, 300, 128),      # G*S = 15, S not a multiple of 16
    (1, 12, 4, 16, 400, 420, 128),    # G*S = 48: 64 columns, 16 of them padding
    (1, 4, 4, 16, 5000, 5000, 128),   # 4 units of 41 key tiles, each split over 5 CTAs
    # schedule corners on a 148-SM part: more units than CTAs
    (75, 4, 2, 16, 300, 320, 128),    # 150 units: 148 whole, 2 split over 10 CTAs (keys-on-lanes kernel)
    (40, 8, 4, 8, 200, 210, 64),      # 160 units: 148 whole, 12 split over 60 CTAs (generic kernel)
]


@pytest.mark.parametrize("B,Hq,Hkv,S,P,cap,d", SAMPLE_CASES)
def test_decoder_sample_parity(oracle, B, Hq, Hkv, S, P, cap, d):
    H.run_sample_case(oracle, B, Hq, Hkv, S, P, cap, d)


@pytest.mark.parametrize("B,Hq,Hkv,S,P,cap,d", [(2, 8, 4, 16, 900, 1000, 128), (1, 8, 2, 16, 700, 700, 128),
                                                 (2, 4, 2, 32, 600, 640, 128)])
def test_decoder_sample_sharp_softmax(oracle, B, Hq, Hkv, S, P, cap, d):
    """Q and K with sigma 3: running maxima move by more than the rescale threshold mid-unit,
    so O is rescaled (and, split over CTAs, merged with unequal maxima)."""
    H.run_sample_case(oracle, B, Hq, Hkv, S, P, cap, d, sigma=3.0, seed0=900)


def test_train_pass_full_size_sampled_heads(oracle):
    """E2D2 train pass at full size (B8 L1024 S16 H16 d64), the launch the benchmark times;
    the oracle recomputes three (batch, head) pairs."""
    w = workloads.TRAIN
    B, Hq, L, d, S = w.batch, w.q_heads, w.L, w.head_dim, w.S
    q = H.gen((B, Hq, L, d), synth.seed_for(2, 0, "q"), w.sigma)
    k = H.gen((B, Hq, L, d), synth.seed_for(2, 0, "k"), w.sigma)
    v = H.gen((B, Hq, L, d), synth.seed_for(2, 0, "v"), w.sigma)
    ke = H.gen((B, Hq, L, d), synth.seed_for(2, 0, "k_enc"), w.sigma)
    ve = H.gen((B, Hq, L, d), synth.seed_for(2, 0, "v_enc"), w.sigma)
    out_e, lse_e = attn.encoder_blockcausal(q[1], k[1], v[1], S)
    out_d, lse_d = attn.decoder_train(q[1], ke[1], ve[1], k[1], v[1], S)
    torch.cuda.synchronize()
    for b, h in ((0, 0), (7, 15), (3, 9)):
        sl = (slice(b, b + 1), slice(h, h + 1))
        ro, rl = oracle.encoder(q[0].f32[sl], k[0].f32[sl], v[0].f32[sl], S)
        H.compare(out_e[sl], lse_e[sl], ro, rl, f"train-pass encoder b{b} h{h}")
        ro, rl = oracle.decoder_train(q[0].f32[sl], ke[0].f32[sl], ve[0].f32[sl], k[0].f32[sl], v[0].f32[sl], S)
        H.compare(out_d[sl], lse_d[sl], ro, rl, f"train-pass decoder b{b} h{h}")


def test_sampling_step_full_size_sampled_batches(oracle):
    """E2D2 sampling step at full size (B32 P2048 S16 Hq16 Hkv8 d128) in the benchmark's launch
    configuration; the oracle recomputes two batch entries."""
    w = workloads.SAMPLE
    B, Hq, Hkv, S, P, d = w.batch, w.q_heads, w.kv_heads, w.S, w.P, w.head_dim
    cap = P + S
    q, kc, vc, kb, vb = H.sample_inputs(B, Hq, Hkv, S, cap, d, 1.0, 3000)
    out, lse = attn.decoder_sample(q[1], kc[1], vc[1], P, kb[1], vb[1])
    torch.cuda.synchronize()
    for b in (0, 17, 31):
        sl = slice(b, b + 1)
        ro, rl = oracle.decoder_sample(q[0].f32[sl], kc[0].f32[sl], vc[0].f32[sl], P, kb[0].f32[sl], vb[0].f32[sl])
        H.compare(out[sl], lse[sl], ro, rl, f"sampling step b{b}")


def test_translation_train_full_size_sampled_heads(oracle):
    """Translation-shaped train pass at full size (B16 L512 S4 H16 d64: the shape of the 28 encoder
    and 4 decoder calls of one step); the oracle recomputes two (batch, head) pairs per call."""
    w = workloads.TRAIN_CHAIN
    B, Hq, L, d, S = w.batch, w.q_heads, w.L, w.head_dim, w.S
    q = H.gen((B, Hq, L, d), synth.seed_for(4, 0, "q"), w.sigma)
    k = H.gen((B, Hq, L, d), synth.seed_for(4, 0, "k"), w.sigma)
    v = H.gen((B, Hq, L, d), synth.seed_for(4, 0, "v"), 1.0)
    ke = H.gen((B, Hq, L, d), synth.seed_for(4, 0, "k_enc"), w.sigma)
    ve = H.gen((B, Hq, L, d), synth.seed_for(4, 0, "v_enc"), 1.0)
    out_e, lse_e = attn.encoder_blockcausal(q[1], k[1], v[1], S)
    out_d, lse_d = attn.decoder_train(q[1], ke[1], ve[1], k[1], v[1], S)
    torch.cuda.synchronize()
    for b, h in ((0, 0), (15, 11)):
        bs, hs = slice(b, b + 1), slice(h, h + 1)
        qq, kk, vv = q[0].f32[bs, hs], k[0].f32[bs, hs], v[0].f32[bs, hs]
        ro, rl = oracle.encoder(qq, kk, vv, S)
        H.compare(out_e[bs, hs], lse_e[bs, hs], ro, rl, f"translation encoder b{b} h{h}")
        ro, rl = oracle.decoder_train(qq, ke[0].f32[bs, hs], ve[0].f32[bs, hs], kk, vv, S)
        H.compare(out_d[bs, hs], lse_d[bs, hs], ro, rl, f"translation decoder b{b} h{h}")


@pytest.mark.parametrize("P", [0, 16, 1008, 4080, 8176])
def test_long_sample_loop_shapes(oracle, P):
    """Sampling calls of the long-context loop (B4 S16 Hq32 Hkv8 d128) at prefix lengths of its
    blocks 0, 1, 63, 255 and 511, full size; the oracle recomputes two batch entries."""
    w = workloads.SAMPLE_LOOP
    B, Hq, Hkv, S, d = w["batch"], w["q_heads"], w["kv_heads"], w["S"], w["head_dim"]
    cap = w["P_max"] + S
    q, kc, vc, kb, vb = H.sample_inputs(B, Hq, Hkv, S, cap, d, 1.0, 5000 + P)
    out, lse = attn.decoder_sample(q[1], kc[1], vc[1], P, kb[1], vb[1])
    torch.cuda.synchronize()
    for b in (0, 3):
        sl = slice(b, b + 1)
        ro, rl = oracle.decoder_sample(q[0].f32[sl], kc[0].f32[sl], vc[0].f32[sl], P, kb[0].f32[sl], vb[0].f32[sl])
        H.compare(out[sl], lse[sl], ro, rl, f"long loop P{P} b{b}")


@pytest.mark.parametrize("B,Hq,Hkv,S,b,d", [(2, 4, 2, 16, 5, 128), (1, 8, 2, 16, 200, 128), (2, 4, 4, 8, 20, 64),
                                           (1, 2, 2, 16, 0, 128)])
def test_encoder_block_step_matches_encoder_rows(oracle, B, Hq, Hkv, S, b, d):
    """Encoder block step for block b (cache holding blocks 0..b-1) reproduces block b's rows of
    the encoder over the whole (b+1) S tokens, and leaves the cache equal to the concatenation:
    block b in rows bS..bS+S-1 bit for bit, earlier rows unchanged, later rows untouched."""
    L, P = (b + 1) * S, b * S
    cap = P + S + 24
    q = H.gen((B, Hq, L, d), 7100 + b, 1.0)
    k = H.gen((B, Hkv, L, d), 7101 + b, 1.0)
    v = H.gen((B, Hkv, L, d), 7102 + b, 1.0)
    kc = torch.full((B, Hkv, cap, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    vc = torch.full_like(kc, float("nan"))
    kc[:, :, :P] = k[1][:, :, :P]
    vc[:, :, :P] = v[1][:, :, :P]
    out, lse = attn.encoder_block_step(q[1][:, :, P:].contiguous(), kc, vc, P, k[1][:, :, P:].contiguous(),
                                       v[1][:, :, P:].contiguous())
    torch.cuda.synchronize()
    ro, rl = oracle.encoder(q[0].f32, k[0].f32, v[0].f32, S)
    H.compare(out, lse, ro[:, :, P:], rl[:, :, P:], f"encoder block step b{b} S{S} d{d}")
    for cache, src in ((kc, k[1]), (vc, v[1])):
        assert torch.equal(cache[:, :, :L].view(torch.int16), src.view(torch.int16))
        assert torch.isnan(cache[:, :, L:].float()).all()


def test_sample_equals_train_rows():
    """On the GPU: a sampling call for block b over the encoder prefix [0, bS) reproduces the
    decoder-train rows of block b (same inputs)."""
    B, Hq, Hkv, L, S, d = 1, 4, 2, 256, 16, 64
    q, ks = H.train_inputs(B, Hq, Hkv, L, d, 1.0, 700)
    (ke, ket), (ve, vet), (kd, kdt), (vd, vdt) = ks
    out_t, lse_t = attn.decoder_train(q[1], ket, vet, kdt, vdt, S)
    for blk in (0, 5, 15):
        r = slice(blk * S, blk * S + S)
        o, l = attn.decoder_sample(q[1][:, :, r].contiguous(), ket, vet, blk * S,
                                   kdt[:, :, r].contiguous(), vdt[:, :, r].contiguous())
        torch.cuda.synchronize()
        assert (o.float() - out_t[:, :, r].float()).abs().max().item() <= 2e-2
        assert (l - lse_t[:, :, r]).abs().max().item() <= 1e-3


def test_kv_append_bitwise(oracle):
    B, Hkv, cap, d = 3, 4, 100, 64
    rng = np.random.default_rng(5)
    kc = rng.integers(0, 65535, size=(B, Hkv, cap, d), dtype=np.uint16)
    vc = rng.integers(0, 65535, size=(B, Hkv, cap, d), dtype=np.uint16)
    to_dev = lambda a: torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16).cuda()
    kg, vg = to_dev(kc), to_dev(vc)
    P = 0
    for S_new in (16, 1, 33, 16):
        kn = rng.integers(0, 65535, size=(B, Hkv, S_new, d), dtype=np.uint16)
        vn = rng.integers(0, 65535, size=(B, Hkv, S_new, d), dtype=np.uint16)
        oracle.kv_append(kc, vc, P, kn, vn)
        P = attn.kv_cache_append(kg, vg, P, to_dev(kn), to_dev(vn))
    torch.cuda.synchronize()
    np.testing.assert_array_equal(kg.cpu().view(torch.int16).numpy().view(np.uint16), kc)
    np.testing.assert_array_equal(vg.cpu().view(torch.int16).numpy().view(np.uint16), vc)


def test_outputs_fully_written_deterministic_and_bounded():
    """NaN-poisoned outputs are fully overwritten, a guard band after the output is untouched,
    and two runs are bitwise identical (catches unwritten rows, stray writes and races)."""
    B, Hq, Hkv, L, S, d = 2, 4, 2, 200, 8, 64
    q, ks = H.train_inputs(B, Hq, Hkv, L, d, 1.0, 800)
    n = B * Hq * L * d
    res = []
    for _ in range(2):
        buf = torch.full((n + 4096,), float("nan"), dtype=torch.bfloat16, device="cuda")
        out = buf[:n].view(B, Hq, L, d)
        lse = torch.full((B, Hq, L), float("nan"), device="cuda")
        attn.decoder_train(q[1], ks[0][1], ks[1][1], ks[2][1], ks[3][1], S, out=out, lse=lse)
        torch.cuda.synchronize()
        assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
        assert torch.isnan(buf[n:].float()).all()
        res.append((out.clone(), lse.clone()))
    assert torch.equal(res[0][0], res[1][0]) and torch.equal(res[0][1], res[1][1])
    # sampling path
    qs, kc, vc, kb, vb = H.sample_inputs(2, 8, 2, 16, 800, 128, 1.0, 900)
    res = []
    for _ in range(2):
        o, l = attn.decoder_sample(qs[1], kc[1], vc[1], 700, kb[1], vb[1])
        torch.cuda.synchronize()
        res.append((o, l))
    assert torch.equal(res[0][0], res[1][0]) and torch.equal(res[0][1], res[1][1])


def test_no_device_wait_timed_out():
    assert attn.last_device_error() == 0


def test_sampling_loop_with_appends_matches_oracle(oracle):
    """The long-context sampling loop's structure at a reduced size: per block, two layers each
    run a sampling call over the cached prefix (P grows by S per block, from 0), then the block
    is appended to that layer's cache.  One workspace serves every call (its tickets must come
    back to zero).  Every call is checked against the oracle; the caches bit for bit at the end."""
    B, Hq, Hkv, S, d, blocks, layers = 2, 8, 2, 16, 128, 10, 2
    cap = blocks * S
    rng_seed = 5000
    caches = []
    for layer in range(layers):
        kc = torch.zeros((B, Hkv, cap, d), dtype=torch.bfloat16, device="cuda")
        vc = torch.zeros_like(kc)
        caches.append([kc, vc, np.zeros((B, Hkv, cap, d), np.uint16), np.zeros((B, Hkv, cap, d), np.uint16)])
    q0 = torch.empty((B, Hq, S, d), dtype=torch.bfloat16, device="cuda")
    ws = attn.sample_workspace(q0, caches[0][0])
    P = 0
    for blk in range(blocks):
        for layer in range(layers):
            kc, vc, kbits, vbits = caches[layer]
            seed = rng_seed + 100 * blk + 10 * layer
            q = H.gen((B, Hq, S, d), seed)
            kb = H.gen((B, Hkv, S, d), seed + 1)
            vb = H.gen((B, Hkv, S, d), seed + 2)
            out, lse = attn.decoder_sample(q[1], kc, vc, P, kb[1], vb[1], workspace=ws)
            torch.cuda.synchronize()
            ref_o, ref_l = oracle.decoder_sample(q[0].f32, synth.bf16_bits_to_f32(kbits),
                                                 synth.bf16_bits_to_f32(vbits), P, kb[0].f32, vb[0].f32)
            H.compare(out, lse, ref_o, ref_l, f"loop block {blk} layer {layer} P{P}")
            attn.kv_cache_append(kc, vc, P, kb[1], vb[1])
            oracle.kv_append(kbits, vbits, P, kb[0].bits, vb[0].bits)
        P += S
    torch.cuda.synchronize()
    for kc, vc, kbits, vbits in caches:
        np.testing.assert_array_equal(kc.cpu().view(torch.int16).numpy().view(np.uint16), kbits)
        np.testing.assert_array_equal(vc.cpu().view(torch.int16).numpy().view(np.uint16), vbits)
    assert int(ws[:1024].view(torch.int32).abs().sum().item()) == 0  # tickets back to zero
