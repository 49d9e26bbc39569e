"""The pre-pass from chunk records (sb_prepass_chunks), against the oracle.

The records are the oracle's own (orc_chunk_stats, pinned on CPU against exact arithmetic and
against the pre-pass row statistics), so this checks the folding, the group slots, the final
reduction, the PDR verdict and both quantization passes: everything must equal the oracle's
pre-pass of the same tensor bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
from video_diffusion_mixed_b200 import synth
from gpu_helpers import npy, u16

pytestmark = pytest.mark.gpu

STATS = ("sum_abs", "max_abs", "amax_rot", "ratio")


def _records(X, B):
    cs = oracle.chunk_stats(u16(X), B)  # [M, K/128, 3]
    rec = np.zeros(cs.shape[:2] + (4,), dtype=np.float32)
    rec[..., :3] = cs
    return torch.from_numpy(rec).cuda()


def _run(sbg, X, chunks, prec0, block=128, rho=64.0, force=-1):
    M, K = X.shape
    ws = sbg.Workspace(M, K)
    a4, a8 = sbg.Fp4Tensor(M, K), sbg.I8Tensor(M, K)
    stats = sbg.alloc_stats()
    prec = torch.tensor([prec0], dtype=torch.int32, device="cuda")
    sbg.prepass_chunks(X, chunks, sbg.config(rho=rho, block=block, force_prec=force), sbg.PREPASS_QUANT, prec, a4,
                       a8, stats, ws)
    sbg.check(ws)
    return a4, a8, sbg.decode_stats(stats), int(prec.item())


SHAPES = [(17776, 12288, 128), (300, 1920, 128), (70, 12288, 128), (33, 640, 128), (50, 1024, 64), (17, 256, 16)]


@pytest.mark.parametrize("M,K,B", SHAPES, ids=[f"{m}x{k}-B{b}" for m, k, b in SHAPES])
def test_prepass_from_chunk_records_int8(sbg, M, K, B):
    X = synth.activations(M, K, n_outlier=max(1, K // 200), scale=25.0, seed=M, tensor_id=K, device="cuda")
    ref = oracle.prepass(u16(X), None, B)
    q, s = oracle.quant_int8(ref["y"], ref["row_amax"])
    a4, a8, st, p = _run(sbg, X, _records(X, B), sbg.INT8, block=B, force=sbg.INT8)
    for k in STATS:
        assert st[k] == ref[k], (k, st[k], ref[k])
    assert p == sbg.INT8
    assert np.array_equal(npy(a8.codes), q)
    assert np.array_equal(npy(a8.scale).view(np.uint32), s.view(np.uint32))


@pytest.mark.parametrize("M,K,B", SHAPES[1:4], ids=[f"{m}x{k}" for m, k, _ in SHAPES[1:4]])
def test_prepass_from_chunk_records_nvfp4(sbg, M, K, B):
    X = synth.activations(M, K, n_outlier=max(1, K // 200), scale=25.0, seed=M + 1, tensor_id=K, device="cuda")
    ref = oracle.prepass(u16(X), None, B)
    a4, a8, st, p = _run(sbg, X, _records(X, B), sbg.NVFP4, block=B, force=sbg.NVFP4)
    codes, sfl, sft, sg = oracle.quant_nvfp4(ref["y"], ref["amax_rot"])
    assert st["amax_rot"] == ref["amax_rot"] and p == sbg.NVFP4
    assert np.float32(npy(a4.gscale)[0]) == sg
    assert np.array_equal(npy(a4.codes), codes)
    assert np.array_equal(npy(a4.sf), sft)


def test_chunk_records_pdr_verdict_and_int8_codes(sbg):
    """A large outlier: PDR sends the layer to BF16; the INT8 codes are still written, as
    sb_prepass writes them when the flag said INT8 at the start."""
    M, K = 64, 1024
    X = synth.activations(M, K, seed=12, device="cuda")
    X[5, 300] = 3000.0
    ref = oracle.prepass(u16(X), None, 128)
    q, _ = oracle.quant_int8(ref["y"], ref["row_amax"])
    a4, a8, st, p = _run(sbg, X, _records(X, 128), sbg.INT8, rho=64.0)
    assert st["ratio"] == ref["ratio"] > 64.0
    assert p == oracle.apply_pdr(sbg.INT8, ref["ratio"], 64.0) == sbg.BF16
    assert np.array_equal(npy(a8.codes), q)


def test_chunk_records_stats_mode(sbg):
    """STATS mode: the records fold into the statistics record only; no quantization kernel
    runs, the precision flag may be absent, the quantized tensors are not touched."""
    M, K = 300, 3072
    X = synth.activations(M, K, n_outlier=15, scale=50.0, seed=41, device="cuda")
    ref = oracle.prepass(u16(X), None, 128)
    ws = sbg.Workspace(M, K)
    stats = sbg.alloc_stats()
    sbg.prepass_chunks(X, _records(X, 128), sbg.config(block=128), sbg.PREPASS_STATS, None, None, None, stats, ws)
    sbg.check(ws)
    st = sbg.decode_stats(stats)
    for k in STATS:
        assert st[k] == ref[k], (k, st[k], ref[k])
    assert st["numel"] == M * K and st["nonfinite"] == 0


def test_chunk_records_skip_writes_nothing(sbg):
    """*prec == SB_SKIP: every kernel exits at once -- no statistics, codes or scales are written
    -- and the workspace's last-CTA ticket stays clean for the next call, which must be exact."""
    M, K = 200, 1024
    X = synth.activations(M, K, seed=42, device="cuda")
    ws = sbg.Workspace(M, K)
    a4, a8 = sbg.Fp4Tensor(M, K), sbg.I8Tensor(M, K)
    a4.codes.fill_(0xAB)
    a8.codes.fill_(0x55)
    a8.scale.fill_(-1.0)
    stats = sbg.alloc_stats()
    stats.fill_(0xEE)
    prec = torch.tensor([sbg.SKIP], dtype=torch.int32, device="cuda")
    sbg.prepass_chunks(X, _records(X, 128), sbg.config(block=128), sbg.PREPASS_QUANT, prec, a4, a8, stats, ws)
    sbg.check(ws)
    assert int(prec.item()) == sbg.SKIP
    assert (npy(a4.codes) == 0xAB).all() and (npy(a8.codes) == 0x55).all() and (npy(a8.scale) == -1.0).all()
    assert (npy(stats) == 0xEE).all()
    ref = oracle.prepass(u16(X), None, 128)
    q, s = oracle.quant_int8(ref["y"], ref["row_amax"])
    a4, a8, st, p = _run(sbg, X, _records(X, 128), sbg.INT8, force=sbg.INT8)
    assert st["sum_abs"] == ref["sum_abs"] and p == sbg.INT8
    assert np.array_equal(npy(a8.codes), q)
