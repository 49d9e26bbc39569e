"""GPU parity of the Temporal Delta Cache's reuse path (R-REUSE) against the CPU oracle.

At a computed step the module's residual D = bf16(y - x) is kept; at a skipped step the output is
bf16(x + D). Both are bit-exact against the oracle, and each writes only in its own case of the
module's skip decision, which is taken on the device by sb_tdc_step.
"""
import numpy as np
import pytest
import torch

import oracle
from video_diffusion_mixed_b200 import synth
from gpu_helpers import u16

pytestmark = pytest.mark.gpu


def skipping_state(sb, M, C, skip: bool):
    """A module state after two computed outputs and one decision: skip or compute."""
    ws = sb.Workspace(M, C)
    st = sb.alloc_state()
    y0 = synth.activations(M, C, seed=31, device="cuda")
    cache = torch.zeros_like(y0)
    sb.tdc_record(y0, cache, None, st, ws)
    sb.tdc_record(synth.noisy_copy(y0, 0.01, seed=32), cache, None, st, ws)
    sb.tdc_step(st, sb.config(tdc_thresh=1e30 if skip else -1.0))
    sb.check(ws)
    assert sb.decode_state(st)["skip"] == (1 if skip else 0)
    return st


@pytest.mark.parametrize("M,C", [(1, 8), (300, 72), (256, 3072), (17776, 3072)])
def test_refresh_then_reuse_bitexact(sbg, M, C):
    x = synth.activations(M, C, n_outlier=3, scale=40.0, seed=1, device="cuda")
    y = synth.noisy_copy(x, 0.3, seed=2)
    x2 = synth.noisy_copy(x, 0.05, seed=3)  # the next step's input
    st_compute = skipping_state(sbg, 64, 64, skip=False)
    st_skip = skipping_state(sbg, 64, 64, skip=True)
    delta = torch.full_like(x, 7.0)
    sbg.tdc_refresh(x, y, delta, st_compute)
    out = torch.full_like(x, 7.0)
    sbg.tdc_reuse(x2, delta, out, st_skip)
    torch.cuda.synchronize()
    ref_d = oracle.tdc_refresh(u16(x), u16(y))
    assert np.array_equal(u16(delta), ref_d)
    assert np.array_equal(u16(out), oracle.tdc_reuse(u16(x2), ref_d))


def test_each_call_writes_only_in_its_own_case(sbg):
    M, C = 128, 256
    x = synth.activations(M, C, seed=5, device="cuda")
    y = synth.noisy_copy(x, 0.3, seed=6)
    st_compute = skipping_state(sbg, 64, 64, skip=False)
    st_skip = skipping_state(sbg, 64, 64, skip=True)
    sentinel = torch.full_like(x, -3.0)
    d = sentinel.clone()
    sbg.tdc_refresh(x, y, d, st_skip)   # skipped step: the kept residual stays
    o = sentinel.clone()
    sbg.tdc_reuse(x, y, o, st_compute)  # computed step: the module's own output stays
    torch.cuda.synchronize()
    assert torch.equal(d, sentinel) and torch.equal(o, sentinel)
