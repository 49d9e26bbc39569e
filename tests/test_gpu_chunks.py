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


# ---- the producers of the records: sb_chunk_records (a bf16 tensor in memory) and the GEMM's
# record epilogue (sb_linear_records), against the oracle's chunk statistics ----

REC_SHAPES = [(17776, 12288, 128), (300, 1920, 128), (33, 640, 64), (5, 256, 16), (1, 128, 32)]


def _nan_records(M, N):
    return torch.full((M, N // 128, 4), float("nan"), dtype=torch.float32, device="cuda")


def _assert_records(got, ref):
    """Bit-exact on every finite field; NaN where the oracle has NaN (payloads may differ)."""
    got3 = got[..., :3]
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got3), nan)
    assert np.array_equal(got3[~nan].view(np.uint32), ref[~nan].view(np.uint32))
    assert (got[..., 3] == 0).all()


@pytest.mark.parametrize("M,K,B", REC_SHAPES, ids=[f"{m}x{k}-B{b}" for m, k, b in REC_SHAPES])
def test_chunk_records_kernel_bitexact(sbg, M, K, B):
    X = synth.activations(M, K, n_outlier=max(1, K // 200), scale=25.0, seed=M + 3, tensor_id=K + 5, device="cuda")
    rec = _nan_records(M, K)
    sbg.chunk_records(X, rec, block=B)
    _assert_records(npy(rec), oracle.chunk_stats(u16(X), B))


def test_chunk_records_nonfinite(sbg):
    """One +Inf in a chunk (every rotated value is then infinite), +Inf and -Inf in another (some
    rotated values are NaN, which the maxima skip), a NaN in a third (the sum is NaN)."""
    M, K = 4, 512
    X = synth.activations(M, K, seed=9, device="cuda")
    X[0, 5] = float("inf")
    X[1, 130] = float("inf")
    X[1, 200] = float("-inf")
    X[2, 300] = float("nan")
    rec = _nan_records(M, K)
    sbg.chunk_records(X, rec)
    ref = oracle.chunk_stats(u16(X), 128)
    assert np.isinf(ref[0, 0, 0]) and np.isnan(ref[2, 2, 1])
    _assert_records(npy(rec), ref)


def _gelu_layer(sbg, M, N, K, seed):
    X = synth.activations(M, K, n_outlier=max(1, K // 200), scale=10.0, seed=seed, tensor_id=20, device="cuda")
    W = synth.weight(N, K, seed=seed, tensor_id=21, device="cuda")
    bias = synth.bias(N, std=0.02, seed=seed, tensor_id=22, device="cuda")
    ws = sbg.Workspace(max(M, N), K)
    return X, sbg.Weight(W, bias, 128, ws), ws


def _quantized(sbg, X, prec, ws):
    M, K = X.shape
    a4, a8 = sbg.Fp4Tensor(M, K), sbg.I8Tensor(M, K)
    p = torch.tensor([prec], dtype=torch.int32, device="cuda")
    sbg.prepass(X, None, sbg.config(block=128, force_prec=prec), sbg.PREPASS_QUANT, p, a4, a8, sbg.alloc_stats(), ws)
    return a4, a8, p


LIN = [(300, 1024, 512, 128), (130, 256, 1024, 128), (17776, 12288, 3072, 128)]


@pytest.mark.parametrize("prec", ["NVFP4", "INT8", "BF16"])
@pytest.mark.parametrize("M,N,K,B", LIN, ids=[f"{m}x{n}x{k}-B{b}" for m, n, k, b in LIN])
def test_linear_records(sbg, M, N, K, B, prec):
    """The record form of the GEMM stores the same bf16 output as sb_linear, and its records are
    the oracle's chunk statistics of that output (ragged M-tiles included)."""
    X, w, ws = _gelu_layer(sbg, M, N, K, seed=M + N)
    a4, a8, p = _quantized(sbg, X, getattr(sbg, prec), ws)
    Y0 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    sbg.linear(X, a4, a8, p, w, Y0, epilogue=sbg.EPI_GELU, ws=ws)
    Y = torch.full_like(Y0, 7.0)
    rec = _nan_records(M, N)
    sbg.linear_records(X, a4, a8, p, w, Y, rec, epilogue=sbg.EPI_GELU, block=B, ws=ws)
    sbg.check(ws)
    assert torch.equal(Y.view(torch.int16), Y0.view(torch.int16))
    _assert_records(npy(rec), oracle.chunk_stats(u16(Y), B))


@pytest.mark.parametrize("prec", ["INT8", "NVFP4"])
def test_ffn_pair_records_feed_the_prepass(sbg, prec):
    """H = GELU(X W1^T + b1) with its records from the GEMM's epilogue; the pre-pass of H from
    those records equals the oracle's pre-pass of H: statistics, verdict and codes."""
    M, N, K, B = 300, 1536, 512, 128
    X, w, ws = _gelu_layer(sbg, M, N, K, seed=77)
    a4, a8, p = _quantized(sbg, X, sbg.NVFP4, ws)
    H = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    rec = _nan_records(M, N)
    sbg.linear_records(X, a4, a8, p, w, H, rec, epilogue=sbg.EPI_GELU, block=B, ws=ws)
    sbg.check(ws)
    ref = oracle.prepass(u16(H), None, B)
    P = getattr(sbg, prec)
    a4h, a8h, st, ph = _run(sbg, H, rec, P, block=B, force=P)
    for k in STATS:
        assert st[k] == ref[k], (k, st[k], ref[k])
    assert ph == P
    if P == sbg.INT8:
        q, s = oracle.quant_int8(ref["y"], ref["row_amax"])
        assert np.array_equal(npy(a8h.codes), q)
        assert np.array_equal(npy(a8h.scale).view(np.uint32), s.view(np.uint32))
    else:
        codes, sfl, sft, sg = oracle.quant_nvfp4(ref["y"], ref["amax_rot"])
        assert np.float32(npy(a4h.gscale)[0]) == sg
        assert np.array_equal(npy(a4h.codes), codes)
        assert np.array_equal(npy(a4h.sf), sft)


def test_linear_records_skip_writes_nothing(sbg):
    M, N, K = 64, 512, 256
    X, w, ws = _gelu_layer(sbg, M, N, K, seed=5)
    a4, a8, p = _quantized(sbg, X, sbg.INT8, ws)
    p.fill_(sbg.SKIP)
    Y = torch.full((M, N), 7.0, dtype=torch.bfloat16, device="cuda")
    rec = _nan_records(M, N)
    sbg.linear_records(X, a4, a8, p, w, Y, rec, epilogue=sbg.EPI_GELU, ws=ws)
    sbg.check(ws)
    assert (npy(Y.float()) == 7.0).all() and np.isnan(npy(rec)).all()
