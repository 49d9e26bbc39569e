"""GPU parity of sb_module_record, the module's output record in one pass: the difference
statistic of the output y against the module input x and the Temporal Delta Cache record of y.

It must give, bit for bit, what the two calls it replaces give (sb_prepass in statistics mode with
x as x_ref, then sb_tdc_record taking d from those statistics): the statistics record, the module
state and the refreshed cache, over two module steps (the first records without a cached output),
for every row tiling of the fused kernel; d and delta also against the oracle. Each part keeps its
own gate (a skipped layer flag, a skipped module).
"""
import numpy as np
import pytest
import torch

import oracle
from video_diffusion_mixed_b200 import synth
from gpu_helpers import u16

pytestmark = pytest.mark.gpu
STATE = 56  # bytes of sb_module_state; the binding's 64-byte buffer has 8 more that nothing writes


def two_steps(sb, M, C, fused, prec_value=0, update=True):
    x = synth.activations(M, C, n_outlier=3, scale=30.0, seed=21, device="cuda")
    ys = [synth.noisy_copy(x, 0.4, seed=22), None]
    ys[1] = synth.noisy_copy(ys[0], 0.05, seed=23)
    ws = sb.Workspace(M, C)
    st = sb.alloc_state()
    stats = sb.alloc_stats()
    cache = torch.zeros_like(x)
    prec = torch.tensor([prec_value], dtype=torch.int32, device="cuda")
    cfg = sb.config(block=min(128, C), force_prec=-1)  # the statistics do not depend on the block
    out = []
    for y in ys:
        if fused:
            sb.module_record(y, x, cache, prec, stats, st, ws, update_cache=update)
        else:
            sb.prepass(y, x, cfg, sb.PREPASS_STATS, prec, None, None, stats, ws)
            sb.tdc_record(y, cache, stats, st, ws, update_cache=update)
        sb.check(ws)
        out.append((stats.clone(), st.clone(), cache.clone()))
    return x, ys, out


# Row tilings (warps per row x 1024-element segments per warp): (1, 64) 1 x 1; 1920 1 x 2;
# 3072 1 x 3; 4096 2 x 2; 6144 2 x 3; 8192 4 x 2; 12288 4 x 3; 16384 8 x 2. 70001 rows: more than
# 4096 groups, so the last CTA folds the group sums in chunks.
@pytest.mark.parametrize("M,C", [(1, 64), (33, 1920), (256, 3072), (17776, 3072), (64, 4096), (48, 6144), (16, 8192),
                                 (100, 12288), (24, 16384), (70001, 64)])
def test_module_record_equals_the_two_calls(sbg, M, C):
    x, ys, sep = two_steps(sbg, M, C, fused=False)
    _, _, fus = two_steps(sbg, M, C, fused=True)
    for (s0, t0, c0), (s1, t1, c1) in zip(sep, fus):
        assert torch.equal(s0, s1), (sbg.decode_stats(s0), sbg.decode_stats(s1))
        assert torch.equal(t0[:STATE], t1[:STATE]), (sbg.decode_state(t0), sbg.decode_state(t1))
        assert torch.equal(c0, c1)
    # and the second step's d and delta against the oracle
    stats = sbg.decode_stats(fus[1][0])
    ref = oracle.prepass(u16(ys[1]), u16(x), min(128, C), want_rot=False)
    assert stats["d"] == ref["d"]
    assert sbg.decode_state(fus[1][1])["delta"] == oracle.tdc_delta(u16(ys[1]), u16(ys[0]))[0]
    assert torch.equal(fus[1][2], ys[1])


def test_module_record_without_cache_update(sbg):
    M, C = 96, 1024
    _, _, sep = two_steps(sbg, M, C, fused=False, update=False)
    _, _, fus = two_steps(sbg, M, C, fused=True, update=False)
    for (s0, t0, c0), (s1, t1, c1) in zip(sep, fus):
        assert torch.equal(s0, s1) and torch.equal(t0[:STATE], t1[:STATE]) and torch.equal(c0, c1)
    assert not fus[1][2].any()  # the cache was never written


def _skipping(sb, skip):
    """A module state after two recorded outputs and one TDC decision (skip or compute)."""
    ws = sb.Workspace(64, 64)
    st = sb.alloc_state()
    y0 = synth.activations(64, 64, seed=31, device="cuda")
    cache = torch.zeros_like(y0)
    sb.tdc_record(y0, cache, None, st, ws)
    sb.tdc_record(synth.noisy_copy(y0, 0.01, seed=32), cache, None, st, ws)
    sb.tdc_step(st, sb.config(tdc_thresh=1e30 if skip else -1.0))
    sb.check(ws)
    assert sb.decode_state(st)["skip"] == (1 if skip else 0)
    return st


@pytest.mark.parametrize("skip,prec", [(True, 3), (False, 3), (True, 0)], ids=["both_off", "stats_off", "record_off"])
def test_module_record_gates(sbg, skip, prec):
    """Each part runs only in its own case: the statistics unless the layer flag reads SB_SKIP, the
    TDC record unless the module is skipped; a part that does not run writes nothing."""
    M, C = 64, 512
    x = synth.activations(M, C, seed=41, device="cuda")
    y = synth.noisy_copy(x, 0.3, seed=42)
    p = torch.tensor([prec], dtype=torch.int32, device="cuda")
    outs = []
    for fused in (False, True):
        ws = sbg.Workspace(M, C)
        st = _skipping(sbg, skip)
        stats = sbg.alloc_stats()
        stats.fill_(0x5A)
        cache = torch.full_like(x, 3.0)
        if fused:
            sbg.module_record(y, x, cache, p, stats, st, ws)
        else:
            sbg.prepass(y, x, sbg.config(force_prec=-1), sbg.PREPASS_STATS, p, None, None, stats, ws)
            sbg.tdc_record(y, cache, stats, st, ws)
        sbg.check(ws)
        outs.append((stats, st, cache))
    (s0, t0, c0), (s1, t1, c1) = outs
    assert torch.equal(s0, s1) and torch.equal(t0[:STATE], t1[:STATE]) and torch.equal(c0, c1)
    if prec == 3:
        assert bool((s1 == 0x5A).all())  # no statistics written
    if skip:
        assert bool((c1 == 3.0).all())  # no cache refresh
