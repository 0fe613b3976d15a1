"""Failure handling and debugging aids, exercised on the GPU without any fault:

- the bounded device waits: a test hook shortens their limit to 1 ms and delays the load producer
  by 20 ms, so the consumers' waits run out; the kernel unwinds (the waits that guard freeing
  tensor memory and copies in flight keep their 2 s limit), returns, and e2d2_last_device_error()
  reports E2D2_ERR_TIMEOUT; the next normal call on the same stream is parity-green;
- the library built with E2D2_DEBUG (device-side bounds checks on TMA coordinates and work-unit
  indices): parity-green on every call family with no check failing;
- E2D2_SPLITS: other split counts of the sampling call give the oracle's result too."""
import os
import subprocess
import sys
from pathlib import Path

import numpy as np
import pytest
import torch

from block_discrete_diffusion_tcgen05_b200 import _lib, attn, build
import gpu_helpers as H

pytestmark = pytest.mark.gpu

ROOT = Path(__file__).resolve().parents[1]
E2D2_ERR_TIMEOUT = 8


def test_wait_timeout_is_reported_and_the_next_call_is_clean(oracle):
    lib = _lib.load()
    B, Hq, Hkv, L, S, d = 1, 2, 2, 256, 16, 64
    q, ks = H.train_inputs(B, Hq, Hkv, L, d, 1.0, 1800)
    (k, kt), (v, vt) = ks[0], ks[1]
    assert attn.last_device_error() == 0
    try:
        assert lib.e2d2_debug_set_wait_test(1_000_000, 20_000_000) == 0   # 1 ms waits, 20 ms delay
        attn.encoder_blockcausal(q[1], kt, vt, S)
        torch.cuda.synchronize()
        assert attn.last_device_error() == E2D2_ERR_TIMEOUT
    finally:
        assert lib.e2d2_debug_set_wait_test(0, 0) == 0
    out, lse = attn.encoder_blockcausal(q[1], kt, vt, S)
    torch.cuda.synchronize()
    ref_o, ref_l = oracle.encoder(q[0].f32, k.f32, v.f32, S)
    H.compare(out, lse, ref_o, ref_l, "encoder after a timed-out call")
    assert attn.last_device_error() == 0


def test_debug_library_parity(oracle):
    """Every call family through the E2D2_DEBUG library: results as the oracle's, no failed check."""
    dbg = _lib.load(build.build(debug=True))
    saved = _lib._lib
    _lib._lib = dbg
    try:
        H.run_encoder_case(oracle, 2, 4, 2, 200, 16, 64)
        H.run_decoder_case(oracle, 1, 4, 4, 130, 7, 32)
        H.run_sample_case(oracle, 4, 16, 8, 16, 700, 800, 128)
        H.run_sample_case(oracle, 2, 16, 4, 16, 1000, 1040, 64)
        # ragged prefixes
        B, Hq, Hkv, S, cap, d, P = 3, 16, 8, 16, 600, 128, [0, 600, 77]
        qs, kc, vc, kb, vb = H.sample_inputs(B, Hq, Hkv, S, cap, d, 1.0, 1900)
        out, lse = attn.decoder_sample_ragged(qs[1], kc[1], vc[1], torch.tensor(P, dtype=torch.int32, device="cuda"),
                                              kb[1], vb[1])
        torch.cuda.synchronize()
        H.compare(out, lse, *oracle.decoder_sample_ragged(qs[0].f32, kc[0].f32, vc[0].f32, P, kb[0].f32, vb[0].f32),
                  "debug ragged")
        # backward
        qq, kss = H.train_inputs(1, 2, 2, 130, 64, 1.0, 1950)
        (k, kt), (v, vt) = kss[0], kss[1]
        g = H.gen((1, 2, 130, 64), 1959)
        o, l = attn.encoder_blockcausal(qq[1], kt, vt, 16)
        grads = attn.encoder_backward(qq[1], kt, vt, o, l, g[1], 16)
        torch.cuda.synchronize()
        ref = oracle.encoder_backward(qq[0].f32, k.f32, v.f32, g[0].f32, 16)
        for a, r in zip(grads, ref):
            err = np.abs(a.float().cpu().numpy() - r)
            assert (err <= 2e-2 + 2.0 ** -7 * np.abs(r)).all()
        assert dbg.e2d2_last_device_error(torch.cuda.current_stream().cuda_stream) == 0
    finally:
        _lib._lib = saved


_SPLIT_RUN = r"""
import sys
sys.path.insert(0, {root!r}); sys.path.insert(0, {tests!r})
import numpy as np, torch
import oracle
from block_discrete_diffusion_tcgen05_b200 import attn
import gpu_helpers as H
orc = oracle.default()
sms = torch.cuda.get_device_properties(0).multi_processor_count
print("PLAN", attn.sample_plan(4, 32, 8, 128, 16, 2000, sms))
print("RESULT", H.run_sample_case(orc, 4, 32, 8, 16, 2000, 2064, 128, seed0=2000))
print("ERR", attn.last_device_error())
"""


@pytest.mark.parametrize("splits", ["32", "100", "148"])
def test_split_override_keeps_the_result(splits):
    """The long-context loop's shape at P = 2000 (32 units) with the split phase cut over 32, 100
    and every CTA: each run matches the oracle (run_sample_case asserts the bars)."""
    code = _SPLIT_RUN.format(root=str(ROOT), tests=str(ROOT / "tests"))
    env = dict(os.environ, E2D2_SPLITS=splits)
    res = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stdout + res.stderr
    plan = eval(res.stdout.split("PLAN", 1)[1].splitlines()[0].strip())
    assert plan["split_ctas"] == min(int(splits), plan["grid"])
    assert "ERR 0" in res.stdout
