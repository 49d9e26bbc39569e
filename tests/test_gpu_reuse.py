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


# ---- the residual kept in FP8 (R-REUSE-FP8) -----------------------------------------------------

@pytest.mark.parametrize("M,C", [(1, 16), (300, 80), (256, 3072), (17776, 3072), (3, 33024)])
def test_fp8_refresh_then_reuse_bitexact(sbg, M, C):
    """Codes, per-token scales and the reused output bit for bit against the oracle, with rows of
    very different scales and a zero row (scale 0, zero codes). 33024 channels take the two-pass
    refresh (rows wider than the register-resident kernel's 32768)."""
    x = synth.activations(M, C, n_outlier=3, scale=40.0, seed=11, device="cuda")
    y = synth.noisy_copy(x, 0.3, seed=12)
    if M > 2:
        y[M // 2] = x[M // 2]  # zero residual row
        y[1] = x[1] + (y[1] - x[1]) * 1e-3
    x2 = synth.noisy_copy(x, 0.05, seed=13)
    st_compute = skipping_state(sbg, 64, 64, skip=False)
    st_skip = skipping_state(sbg, 64, 64, skip=True)
    d = sbg.Fp8Residual(M, C)
    d.codes.fill_(0x55)
    sbg.tdc_refresh_fp8(x, y, d, st_compute)
    out = torch.full_like(x, 7.0)
    sbg.tdc_reuse_fp8(x2, d, out, st_skip)
    torch.cuda.synchronize()
    codes, scale = oracle.tdc_refresh_fp8(u16(x), u16(y))
    assert np.array_equal(d.codes.cpu().numpy(), codes)
    assert np.array_equal(d.scale.cpu().numpy().view(np.uint32), scale.view(np.uint32))
    assert np.array_equal(u16(out), oracle.tdc_reuse_fp8(u16(x2), codes, scale))


def test_fp8_tiny_row_saturates_like_the_oracle(sbg):
    """A row whose largest residual is a bf16 subnormal (448 / a overflows): nonzero residuals
    code as +-448, zeros as 0."""
    M, C = 4, 64
    x = torch.zeros((M, C), dtype=torch.bfloat16, device="cuda")
    y = x.clone()
    yv = y.view(torch.int16)
    yv[0, 3], yv[0, 9], yv[2, 5] = 1, -32767, 2  # +2^-133, -2^-133, +2^-132
    st_compute = skipping_state(sbg, 64, 64, skip=False)
    d = sbg.Fp8Residual(M, C)
    sbg.tdc_refresh_fp8(x, y, d, st_compute)
    torch.cuda.synchronize()
    codes, scale = oracle.tdc_refresh_fp8(u16(x), u16(y))
    assert np.array_equal(d.codes.cpu().numpy(), codes)
    assert np.array_equal(d.scale.cpu().numpy().view(np.uint32), scale.view(np.uint32))
    assert codes[0, 3] == 0x7E and codes[0, 9] == 0xFE


def test_fp8_each_call_writes_only_in_its_own_case(sbg):
    M, C = 64, 128
    x = synth.activations(M, C, seed=15, device="cuda")
    y = synth.noisy_copy(x, 0.3, seed=16)
    st_compute = skipping_state(sbg, 64, 64, skip=False)
    st_skip = skipping_state(sbg, 64, 64, skip=True)
    d = sbg.Fp8Residual(M, C)
    d.codes.fill_(0x33)
    d.scale.fill_(5.0)
    sbg.tdc_refresh_fp8(x, y, d, st_skip)   # skipped step: the kept residual stays
    o = torch.full_like(x, -3.0)
    sbg.tdc_reuse_fp8(x, d, o, st_compute)  # computed step: the module's own output stays
    torch.cuda.synchronize()
    assert bool((d.codes == 0x33).all()) and bool((d.scale == 5.0).all()) and bool((o == -3.0).all())
