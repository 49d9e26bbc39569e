"""Token sharding on one GPU, through the C ABI.

The shards of a tensor run one after another on the same GPU (nothing waits on another launch),
each writing the group slots of its rows into the whole tensor's slot array; the final reduction
over that array must give the statistics, the PDR verdict, the INT8 and NVFP4 codes and the TDC
state of the unsharded tensor, bit for bit and equal to the oracle. The exchange of the slot
arrays between GPUs is covered on CPU by tests/test_shard_gather.py.
"""
import numpy as np
import pytest
import torch

import oracle
from video_diffusion_mixed_b200 import synth
from gpu_helpers import npy, u16

pytestmark = pytest.mark.gpu

STATS = ("sum_abs", "sum_d2", "sum_ref2", "max_abs", "amax_rot", "ratio", "d")

CASES = [
    # (M, K, shard boundaries, x_ref given)
    (17776, 3072, [0, 8896, 17776], False),
    (300, 1920, [0, 112, 208, 300], True),
    (70, 12288, [0, 48, 70], False),
    (33, 256, [0, 16, 32, 33], True),
]


def _shards(cuts):
    return list(zip(cuts[:-1], cuts[1:]))


@pytest.mark.parametrize("M,K,cuts,with_ref", CASES, ids=[f"{c[0]}x{c[1]}-{len(c[2]) - 1}" for c in CASES])
def test_sharded_prepass_int8_matches_oracle(sbg, M, K, cuts, with_ref):
    X = synth.activations(M, K, n_outlier=max(1, K // 200), scale=30.0, seed=3, tensor_id=M, device="cuda")
    R = synth.activations(M, K, seed=4, tensor_id=M, device="cuda") if with_ref else None
    ref = oracle.prepass(u16(X), u16(R) if R is not None else None, 128)
    q, s = oracle.quant_int8(ref["y"], ref["row_amax"])
    cfg = sbg.config(rho=64.0, block=128, force_prec=sbg.INT8)
    ws = sbg.Workspace(M, K)
    slots = sbg.alloc_slots(M)
    prec = torch.tensor([sbg.INT8], dtype=torch.int32, device="cuda")
    codes = []
    for r0, r1 in _shards(cuts):
        a8 = sbg.I8Tensor(r1 - r0, K)
        sbg.prepass_partial(X[r0:r1], R[r0:r1] if R is not None else None, r0, M, cfg, sbg.PREPASS_QUANT, prec,
                            a8, slots, ws)
        codes.append(a8)
    stats = sbg.alloc_stats()
    sbg.prepass_finish(slots, M, K, with_ref, cfg, sbg.PREPASS_QUANT, prec, stats, ws)
    sbg.check(ws)
    st = sbg.decode_stats(stats)
    for k in STATS:
        assert st[k] == ref[k], (k, st[k], ref[k])
    assert int(prec.item()) == sbg.INT8
    assert np.array_equal(np.concatenate([npy(a.codes) for a in codes]), q)
    assert np.array_equal(np.concatenate([npy(a.scale) for a in codes]).view(np.uint32), s.view(np.uint32))


@pytest.mark.parametrize("M,K,cuts,with_ref", CASES[:3], ids=[f"{c[0]}x{c[1]}" for c in CASES[:3]])
def test_sharded_prepass_nvfp4_encodes_with_the_whole_tensor_scale(sbg, M, K, cuts, with_ref):
    X = synth.activations(M, K, n_outlier=max(1, K // 200), scale=30.0, seed=5, tensor_id=M, device="cuda")
    ref = oracle.prepass(u16(X), None, 128)
    cfg = sbg.config(rho=64.0, block=128, force_prec=sbg.NVFP4)
    ws = sbg.Workspace(M, K)
    slots = sbg.alloc_slots(M)
    prec = torch.tensor([sbg.NVFP4], dtype=torch.int32, device="cuda")
    for r0, r1 in _shards(cuts):
        sbg.prepass_partial(X[r0:r1], None, r0, M, cfg, sbg.PREPASS_QUANT, prec, sbg.I8Tensor(r1 - r0, K), slots, ws)
    stats = sbg.alloc_stats()
    sbg.prepass_finish(slots, M, K, False, cfg, sbg.PREPASS_QUANT, prec, stats, ws)
    assert sbg.decode_stats(stats)["amax_rot"] == ref["amax_rot"]
    for r0, r1 in _shards(cuts):
        a4 = sbg.Fp4Tensor(r1 - r0, K)
        sbg.nvfp4_encode(X[r0:r1], cfg, prec, stats, a4, ws)
        sbg.check(ws)
        codes, sfl, sft, sg = oracle.quant_nvfp4(ref["y"][r0:r1], ref["amax_rot"])
        assert np.float32(npy(a4.gscale)[0]) == sg
        assert np.array_equal(npy(a4.codes), codes)
        assert np.array_equal(npy(a4.sf), sft)


def test_sharded_pdr_verdict_matches_the_whole_tensor(sbg):
    """Outliers only in the second shard: each shard alone would decide differently, the finished
    reduction decides as the whole tensor does."""
    M, K = 64, 512
    X = synth.activations(M, K, seed=6, device="cuda")
    X[40:, 7] = 400.0
    ref = oracle.prepass(u16(X), None, 128)
    rho = 16.0
    cfg = sbg.config(rho=rho, block=128)
    ws = sbg.Workspace(M, K)
    slots = sbg.alloc_slots(M)
    prec = torch.tensor([sbg.NVFP4], dtype=torch.int32, device="cuda")
    for r0, r1 in ((0, 32), (32, 64)):
        sbg.prepass_partial(X[r0:r1], None, r0, M, cfg, sbg.PREPASS_QUANT, prec, sbg.I8Tensor(32, K), slots, ws)
    assert int(prec.item()) == sbg.NVFP4  # the shards leave the verdict to the finish
    stats = sbg.alloc_stats()
    sbg.prepass_finish(slots, M, K, False, cfg, sbg.PREPASS_QUANT, prec, stats, ws)
    sbg.check(ws)
    assert int(prec.item()) == oracle.apply_pdr(sbg.NVFP4, ref["ratio"], rho) == sbg.BF16


@pytest.mark.parametrize("M,C,cuts", [(17776, 3072, [0, 4448, 8896, 17776]), (100, 1920, [0, 48, 100])])
def test_sharded_tdc_record_matches_oracle(sbg, M, C, cuts):
    y0 = synth.activations(M, C, seed=1, device="cuda")
    y1 = synth.noisy_copy(y0, 0.05, seed=2)
    ws = sbg.Workspace(M, C)
    st = sbg.alloc_state()
    cache = torch.zeros_like(y0)
    for y in (y0, y1):
        slots = sbg.alloc_slots(M)
        for r0, r1 in _shards(cuts):
            sbg.tdc_record_partial(y[r0:r1], cache[r0:r1], r0, M, st, slots, ws)
        sbg.tdc_finish(slots, M, C, None, st, ws)
        sbg.check(ws)
    s = sbg.decode_state(st)
    assert s["delta"] == oracle.tdc_delta(u16(y1), u16(y0))[0]
    assert s["n_out"] == 2 and s["acc"] == 0.0 and s["have_d"] == 0
    assert torch.equal(cache, y1)


@pytest.mark.parametrize("block", [256, 64])
def test_sharded_prepass_other_block_sizes(sbg, block):
    """B = 256 runs the 32-element row engine, B = 64 the block-per-lane kernel with its B = 64
    instance: both stop at the group slots when asked to."""
    M, K = 100, 1024
    X = synth.activations(M, K, n_outlier=3, scale=25.0, seed=8, device="cuda")
    ref = oracle.prepass(u16(X), None, block)
    q, s = oracle.quant_int8(ref["y"], ref["row_amax"])
    cfg = sbg.config(rho=64.0, block=block, force_prec=sbg.INT8)
    ws = sbg.Workspace(M, K)
    slots = sbg.alloc_slots(M)
    prec = torch.tensor([sbg.INT8], dtype=torch.int32, device="cuda")
    parts = []
    for r0, r1 in ((0, 48), (48, 100)):
        a8 = sbg.I8Tensor(r1 - r0, K)
        sbg.prepass_partial(X[r0:r1], None, r0, M, cfg, sbg.PREPASS_QUANT, prec, a8, slots, ws)
        parts.append(a8)
    stats = sbg.alloc_stats()
    sbg.prepass_finish(slots, M, K, False, cfg, sbg.PREPASS_QUANT, prec, stats, ws)
    sbg.check(ws)
    st = sbg.decode_stats(stats)
    for k in STATS:
        assert st[k] == ref[k], k
    assert np.array_equal(np.concatenate([npy(a.codes) for a in parts]), q)


def test_sharded_difference_statistic(sbg):
    """The d of a module output against its input (STATS mode with x_ref, the row engine without
    rotation), sharded: the finished record equals the oracle's and leaves *prec alone."""
    M, K = 17776, 3072
    X, _ = synth.workload_inputs("ffn5b", seed=0, device="cuda")
    Y = synth.noisy_copy(X, 0.1, seed=1)
    ref = oracle.prepass(u16(Y), u16(X), 128, want_rot=False)
    cfg = sbg.config(rho=0.0, block=128)
    ws = sbg.Workspace(M, K)
    slots = sbg.alloc_slots(M)
    for r0, r1 in ((0, 6000), (6000, 12000), (12000, M)):
        sbg.prepass_partial(Y[r0:r1], X[r0:r1], r0, M, cfg, sbg.PREPASS_STATS, None, None, slots, ws)
    stats = sbg.alloc_stats()
    sbg.prepass_finish(slots, M, K, True, cfg, sbg.PREPASS_STATS, None, stats, ws)
    sbg.check(ws)
    st = sbg.decode_stats(stats)
    for k in ("sum_abs", "sum_d2", "sum_ref2", "max_abs", "ratio", "d"):
        assert st[k] == ref[k], (k, st[k], ref[k])
    assert st["prec_out"] == -1
