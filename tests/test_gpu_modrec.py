"""GPU parity of sb_linear_module_record: the module's last linear layer whose GEMM epilogue also
computes the module record's partial sums per row and 128-column chunk, a fold kernel finishing
the record.

It must give, bit for bit, what sb_linear followed by sb_module_record gives: the output, the
statistics record (the difference statistic d of the output against the module input), the module
state (the TDC record) and the refreshed cache, over three module steps (the first one without a
cached output), in NVFP4, INT8 and BF16, with and without the cache refresh, with ragged M-tiles;
d and delta also against the oracle. The gates: a skipped layer writes nothing; a skipped module
keeps its cache and state while the statistics still run.
"""
import numpy as np
import pytest
import torch

import oracle
from video_diffusion_mixed_b200 import synth
from gpu_helpers import u16

pytestmark = pytest.mark.gpu
STATE = 56  # bytes of sb_module_state; the binding's 64-byte buffer has 8 more that nothing writes


def module_steps(sb, M, N, K, prec, fused, update=True, nsteps=3, state=None):
    """nsteps module steps of one layer: H_t -> Y_t = H_t W^T + b, recorded against the module
    input x and the module's cache."""
    x = synth.activations(M, N, n_outlier=3, scale=30.0, seed=41, tensor_id=60, device="cuda")
    W = synth.weight(N, K, seed=42, tensor_id=61, device="cuda")
    bias = synth.bias(N, std=0.02, seed=43, tensor_id=62, device="cuda")
    ws = sb.Workspace(max(M, N), K)
    w = sb.Weight(W, bias, 128, ws)
    st = sb.alloc_state() if state is None else state.clone()
    stats = sb.alloc_stats()
    cache = torch.zeros_like(x)
    a4, a8 = sb.Fp4Tensor(M, K), sb.I8Tensor(M, K)
    p = torch.zeros(1, dtype=torch.int32, device="cuda")
    rec = torch.full((M * (N // 128) * 8,), float("nan"), dtype=torch.float32, device="cuda")
    out = []
    for t in range(nsteps):
        H = synth.activations(M, K, n_outlier=2, scale=8.0, seed=50 + t, tensor_id=63, device="cuda")
        p.fill_(prec)
        sb.prepass(H, None, sb.config(block=128, force_prec=prec), sb.PREPASS_QUANT, p, a4, a8, sb.alloc_stats(), ws)
        Y = torch.full((M, N), 7.0, dtype=torch.bfloat16, device="cuda")
        if fused:
            sb.linear_module_record(H, a4, a8, p, w, Y, x, cache, rec, stats, st, ws, update_cache=update)
        else:
            sb.linear(H, a4, a8, p, w, Y, ws=ws)
            sb.module_record(Y, x, cache, p, stats, st, ws, update_cache=update)
        sb.check(ws)
        out.append((Y.clone(), stats.clone(), st.clone(), cache.clone()))
    return x, out


SHAPES = [(300, 1024, 512), (130, 512, 256), (1, 256, 128), (17776, 3072, 12288)]


@pytest.mark.parametrize("prec", ["NVFP4", "INT8", "BF16"])
@pytest.mark.parametrize("M,N,K", SHAPES, ids=[f"{m}x{n}x{k}" for m, n, k in SHAPES])
def test_fused_module_record_equals_the_two_calls(sbg, M, N, K, prec):
    P = getattr(sbg, prec)
    nsteps = 2 if M > 10000 else 3
    x, sep = module_steps(sbg, M, N, K, P, fused=False, nsteps=nsteps)
    _, fus = module_steps(sbg, M, N, K, P, fused=True, nsteps=nsteps)
    for (y0, s0, t0, c0), (y1, s1, t1, c1) in zip(sep, fus):
        assert torch.equal(y0.view(torch.int16), y1.view(torch.int16))
        assert torch.equal(s0, s1), (sbg.decode_stats(s0), sbg.decode_stats(s1))
        assert torch.equal(t0[:STATE], t1[:STATE]), (sbg.decode_state(t0), sbg.decode_state(t1))
        assert torch.equal(c0.view(torch.int16), c1.view(torch.int16))
    # the last step's d and delta against the oracle, the cache against the output
    y_last, y_prev = fus[-1][0], fus[-2][0]
    stats = sbg.decode_stats(fus[-1][1])
    ref = oracle.prepass(u16(y_last), u16(x), 128, want_rot=False)
    assert stats["d"] == ref["d"]
    assert sbg.decode_state(fus[-1][2])["delta"] == oracle.tdc_delta(u16(y_last), u16(y_prev))[0]
    assert torch.equal(fus[-1][3], y_last)


def test_fused_module_record_without_cache_update(sbg):
    M, N, K = 200, 768, 384
    _, sep = module_steps(sbg, M, N, K, sbg.INT8, fused=False, update=False)
    _, fus = module_steps(sbg, M, N, K, sbg.INT8, fused=True, update=False)
    for (y0, s0, t0, c0), (y1, s1, t1, c1) in zip(sep, fus):
        assert torch.equal(y0, y1) and torch.equal(s0, s1) and torch.equal(t0[:STATE], t1[:STATE])
        assert torch.equal(c0, c1)
    assert not fus[-1][3].any()  # the cache was never written


def _skipped_state(sb):
    """A module state whose TDC check decided to skip (two recorded outputs, then the check)."""
    ws = sb.Workspace(64, 64)
    st = sb.alloc_state()
    y0 = synth.activations(64, 64, seed=31, device="cuda")
    cache = torch.zeros_like(y0)
    sb.tdc_record(y0, cache, None, st, ws)
    sb.tdc_record(synth.noisy_copy(y0, 0.01, seed=32), cache, None, st, ws)
    sb.tdc_step(st, sb.config(tdc_thresh=1e30))
    sb.check(ws)
    assert sb.decode_state(st)["skip"] == 1
    return st


def test_fused_module_record_skipped_module(sbg):
    """The module's skip flag is set but the layer runs (a caller's choice): the statistics run, the
    TDC record and the cache refresh do not -- as in the two separate calls."""
    M, N, K = 96, 512, 256
    st = _skipped_state(sbg)
    _, sep = module_steps(sbg, M, N, K, sbg.NVFP4, fused=False, nsteps=1, state=st)
    _, fus = module_steps(sbg, M, N, K, sbg.NVFP4, fused=True, nsteps=1, state=st)
    (y0, s0, t0, c0), (y1, s1, t1, c1) = sep[0], fus[0]
    assert torch.equal(y0, y1) and torch.equal(s0, s1) and torch.equal(t0[:STATE], t1[:STATE])
    assert torch.equal(c0, c1) and not c1.any()
    assert torch.equal(t1[:STATE], st[:STATE])


def test_fused_module_record_skipped_layer_writes_nothing(sbg):
    M, N, K = 64, 256, 128
    x = synth.activations(M, N, seed=44, device="cuda")
    W = synth.weight(N, K, seed=45, device="cuda")
    ws = sbg.Workspace(max(M, N), K)
    w = sbg.Weight(W, None, 128, ws)
    H = synth.activations(M, K, seed=46, device="cuda")
    a4, a8 = sbg.Fp4Tensor(M, K), sbg.I8Tensor(M, K)
    p = torch.tensor([sbg.INT8], dtype=torch.int32, device="cuda")
    sbg.prepass(H, None, sbg.config(force_prec=sbg.INT8), sbg.PREPASS_QUANT, p, a4, a8, sbg.alloc_stats(), ws)
    p.fill_(sbg.SKIP)
    st = sbg.alloc_state()
    st0 = st.clone()
    stats = sbg.alloc_stats()
    stats.fill_(0x5A)
    cache = torch.full_like(x, 3.0)
    Y = torch.full((M, N), 7.0, dtype=torch.bfloat16, device="cuda")
    rec = torch.zeros(M * (N // 128) * 8, dtype=torch.float32, device="cuda")
    sbg.linear_module_record(H, a4, a8, p, w, Y, x, cache, rec, stats, st, ws)
    sbg.check(ws)
    assert bool((Y == 7.0).all()) and bool((cache == 3.0).all()) and bool((stats == 0x5A).all())
    assert torch.equal(st[:STATE], st0[:STATE]) and not rec.any()
