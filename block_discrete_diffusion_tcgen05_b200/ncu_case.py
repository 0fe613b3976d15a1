"""Runs one attention call of a named workload a few times, for profiler captures (ncu).

    python -m block_discrete_diffusion_tcgen05_b200.ncu_case \
        {encoder|decoder_train|encoder_backward|decoder_backward|decoder_sample|kv_append} [repeats]

Shapes are the benchmark's: E2D2 train pass (B8 L1024 S16 H16 d64) for the two train calls and
their backward (one forward call, then `repeats` backward calls),
E2D2 sampling step (B32 P2048 S16 Hq16 Hkv8 d128) for the sampling call and the append.
Inputs are seeded normals drawn on the device (the values do not change the work)."""
from __future__ import annotations

import sys

import torch

from . import attn, workloads


def main(argv):
    which = argv[1] if len(argv) > 1 else "encoder"
    reps = int(argv[2]) if len(argv) > 2 else 3
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev)
    g.manual_seed(1234)

    def rnd(*shape, sigma=1.0):
        return (torch.randn(*shape, generator=g, device=dev) * sigma).to(torch.bfloat16)

    tw, sw = workloads.TRAIN, workloads.SAMPLE
    if which in ("encoder", "decoder_train"):
        shp = (tw.batch, tw.q_heads, tw.L, tw.head_dim)
        q, k, v, ke, ve = (rnd(*shp, sigma=tw.sigma) for _ in range(5))
        for _ in range(reps):
            if which == "encoder":
                attn.encoder_blockcausal(q, k, v, tw.S)
            else:
                attn.decoder_train(q, ke, ve, k, v, tw.S)
    elif which in ("encoder_backward", "decoder_backward"):
        shp = (tw.batch, tw.q_heads, tw.L, tw.head_dim)
        q, k, v, ke, ve = (rnd(*shp, sigma=tw.sigma) for _ in range(5))
        go = rnd(*shp)
        ws = torch.empty(attn.train_backward_workspace_bytes(tw.batch, tw.q_heads, tw.kv_heads, tw.head_dim, tw.L),
                         dtype=torch.uint8, device=dev)
        if which == "encoder_backward":
            o, lse = attn.encoder_blockcausal(q, k, v, tw.S)
            for _ in range(reps):
                attn.encoder_backward(q, k, v, o, lse, go, tw.S, workspace=ws)
        else:
            o, lse = attn.decoder_train(q, ke, ve, k, v, tw.S)
            for _ in range(reps):
                attn.decoder_train_backward(q, ke, ve, k, v, o, lse, go, tw.S, workspace=ws)
    elif which in ("decoder_sample", "kv_append"):
        cap = sw.P + sw.S
        q = rnd(sw.batch, sw.q_heads, sw.S, sw.head_dim)
        kc, vc = (rnd(sw.batch, sw.kv_heads, cap, sw.head_dim) for _ in range(2))
        kb, vb = (rnd(sw.batch, sw.kv_heads, sw.S, sw.head_dim) for _ in range(2))
        ws = attn.sample_workspace(q, kc)
        for _ in range(reps):
            if which == "decoder_sample":
                attn.decoder_sample(q, kc, vc, sw.P, kb, vb, workspace=ws)
            else:
                attn.kv_cache_append(kc, vc, sw.P, kb, vb)
    else:
        raise SystemExit(f"unknown call {which}")
    torch.cuda.synchronize()
    assert attn.last_device_error() == 0
    print(f"{which}: {reps} calls ok")


if __name__ == "__main__":
    main(sys.argv)
