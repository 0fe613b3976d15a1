"""The sampling entry point that allocates nothing (e2d2_attn_decoder_sample_noalloc).

It serves callers that cannot allocate device memory -- an engine that hands all of HBM to its
own pool and gives plugins no allocator, or a hot path that may not call cudaMalloc because it
can synchronise the device.  Its split-KV scratch is a fixed device array inside the library.
These tests call it through the C ABI and check it against the workspace-taking entry point
(e2d2_attn_decoder_sample) within the parity tolerances, on consecutive calls (the array keeps
the previous call's contents) that reach both sampling kernels and split their work over
different CTA counts, and check that a shape too large for the array is refused.
This file is collected last on purpose."""
import ctypes

import pytest
import torch

from block_discrete_diffusion_tcgen05_b200 import _lib, attn
import gpu_helpers as H

pytestmark = pytest.mark.gpu


def _noalloc(lib, q, kc, vc, P, kb, vb):
    B, Hq, S, d = q.shape
    Hkv, cap = kc.shape[1], kc.shape[2]
    out = torch.full_like(q, float("nan"))
    lse = torch.full((B, Hq, S), float("nan"), dtype=torch.float32, device=q.device)
    st = lib.e2d2_attn_decoder_sample_noalloc(q.data_ptr(), kc.data_ptr(), vc.data_ptr(), cap, P,
                                              kb.data_ptr(), vb.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                              _lib.Dims(B, Hq, Hkv, d, 0.0), S,
                                              torch.cuda.current_stream().cuda_stream)
    assert st == 0, _lib.STATUS.get(st, st)
    return out, lse


# Consecutive calls with different work plans: the keys-on-lanes kernel (head_dim 128, G*S <= 64),
# then the generic kernel (head_dim 64) with its units split over a different number of CTAs, so
# the second and third calls find the array holding the previous call's partials and tickets.
CALLS = [(4, 16, 8, 16, 700, 800, 128, 4100),
         (2, 16, 4, 16, 1000, 1040, 64, 4300),
         (2, 32, 8, 16, 2048, 2064, 128, 4200)]


def test_noalloc_matches_workspace_entry_point_on_consecutive_calls():
    lib = _lib.load()
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    plans = [attn.sample_plan(B, Hq, Hkv, d, S, P, sms) for (B, Hq, Hkv, S, P, cap, d, _) in CALLS]
    assert plans[1]["kernel"] == 0 and plans[1]["split_units"] > 0, plans[1]
    assert plans[0]["split_ctas"] != plans[1]["split_ctas"], plans
    for call, (B, Hq, Hkv, S, P, cap, d, seed) in enumerate(CALLS):
        q, kc, vc, kb, vb = H.sample_inputs(B, Hq, Hkv, S, cap, d, 1.0, seed)
        ref_o, ref_l = attn.decoder_sample(q[1], kc[1], vc[1], P, kb[1], vb[1])
        out, lse = _noalloc(lib, q[1], kc[1], vc[1], P, kb[1], vb[1])
        torch.cuda.synchronize()
        assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all(), f"call {call}"
        assert (out.float() - ref_o.float()).abs().max().item() <= H.OUT_TOL, f"call {call}"
        assert (lse - ref_l).abs().max().item() <= H.LSE_TOL, f"call {call}"
    assert attn.last_device_error() == 0


def test_noalloc_refuses_shapes_larger_than_its_array():
    lib = _lib.load()
    dims = _lib.Dims(1, 128, 1, 128, 0.0)  # 2048 packed rows per kv head at d = 128
    need = lib.e2d2_attn_decoder_sample_workspace(dims, 16, 64)
    assert need > _lib.SAMPLE_NOALLOC_MAX_BYTES
    p = 0x10000
    st = lib.e2d2_attn_decoder_sample_noalloc(p, p, p, 64, 32, p, p, p, None, dims, 16, None)
    assert st == 6  # E2D2_ERR_WORKSPACE, before anything is launched
