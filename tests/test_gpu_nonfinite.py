"""Non-finite input to the pre-pass: an Inf or a NaN anywhere in X is reported as SB_ENONFINITE by
sb_check (and in stats->nonfinite), on every pre-pass kernel path: the block-per-lane kernel (no
X_ref), the row engine (X_ref given), and the pre-pass from chunk records. A finite row whose FP32
sum of |x| overflows to +inf is finite input and is not reported. After a report the workspace is
clean: the next call on it succeeds and matches the oracle bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
from video_diffusion_mixed_b200 import synth
from gpu_helpers import u16

pytestmark = pytest.mark.gpu

BF16_MAX = 0x7F7F  # largest finite bf16, about 3.39e38


def _bits(X, m, k, bits):
    v = X.view(torch.int16)
    v[m, k] = bits - 65536 if bits >= 32768 else bits


def _prepass(sb, X, R, ws, force=1):
    M, K = X.shape
    a4, a8 = sb.Fp4Tensor(M, K), sb.I8Tensor(M, K)
    stats = sb.alloc_stats()
    prec = torch.tensor([force], dtype=torch.int32, device="cuda")
    sb.prepass(X, R, sb.config(block=128, force_prec=force), sb.PREPASS_QUANT, prec, a4, a8, stats, ws)
    return stats


@pytest.mark.parametrize("bits", [0x7F80, 0xFF80, 0x7FC0], ids=["+inf", "-inf", "nan"])
@pytest.mark.parametrize("with_ref", [False, True], ids=["block_kernel", "row_engine"])
def test_nonfinite_input_reported(sbg, bits, with_ref):
    M, K = 300, 3072
    X = synth.activations(M, K, seed=31, device="cuda")
    _bits(X, 137, 1000, bits)
    R = synth.activations(M, K, seed=32, device="cuda") if with_ref else None
    ws = sbg.Workspace(M, K)
    stats = _prepass(sbg, X, R, ws)
    with pytest.raises(sbg.SixbitError) as e:
        sbg.check(ws)
    assert e.value.status == sbg.SB_ENONFINITE
    assert sbg.decode_stats(stats)["nonfinite"] == 1
    # the error word was read and cleared: the same workspace serves a finite tensor again
    Xf = synth.activations(M, K, seed=33, device="cuda")
    stats = _prepass(sbg, Xf, None, ws)
    sbg.check(ws)
    st = sbg.decode_stats(stats)
    ref = oracle.prepass(u16(Xf), None, 128)
    assert st["nonfinite"] == 0 and st["sum_abs"] == ref["sum_abs"] and st["amax_rot"] == ref["amax_rot"]


@pytest.mark.parametrize("with_ref", [False, True], ids=["block_kernel", "row_engine"])
def test_finite_row_sum_overflow_not_reported(sbg, with_ref):
    """Two |x| = bf16 max in one row: the row's FP32 sum of |x| overflows to +inf, but every
    input is finite, so nothing is reported; the statistics equal the oracle's (sum |x| = +inf,
    outlier ratio 0)."""
    M, K = 64, 1024
    X = synth.activations(M, K, seed=34, device="cuda")
    _bits(X, 5, 3, BF16_MAX)
    _bits(X, 5, 700, BF16_MAX | 0x8000)
    R = synth.activations(M, K, seed=35, device="cuda") if with_ref else None
    ws = sbg.Workspace(M, K)
    stats = _prepass(sbg, X, R, ws)
    sbg.check(ws)
    st = sbg.decode_stats(stats)
    ref = oracle.prepass(u16(X), u16(R) if R is not None else None, 128)
    assert st["nonfinite"] == 0
    assert np.isinf(ref["sum_abs"]) and st["sum_abs"] == ref["sum_abs"]
    assert st["max_abs"] == ref["max_abs"] and st["ratio"] == ref["ratio"] == 0.0


@pytest.mark.parametrize("bits", [0x7F80, 0x7FC0], ids=["inf", "nan"])
def test_nonfinite_chunk_records_reported(sbg, bits):
    """sb_prepass_chunks over records of a tensor holding Inf / NaN (the records carry the
    non-finite maxima and sums the producer saw)."""
    M, K = 48, 1024
    X = synth.activations(M, K, seed=36, device="cuda")
    _bits(X, 20, 513, bits)
    cs = oracle.chunk_stats(u16(X), 128)
    rec = np.zeros(cs.shape[:2] + (4,), dtype=np.float32)
    rec[..., :3] = cs
    chunks = torch.from_numpy(rec).cuda()
    ws = sbg.Workspace(M, K)
    stats = sbg.alloc_stats()
    prec = torch.tensor([sbg.INT8], dtype=torch.int32, device="cuda")
    sbg.prepass_chunks(X, chunks, sbg.config(block=128), sbg.PREPASS_STATS, prec, None, None, stats, ws)
    with pytest.raises(sbg.SixbitError) as e:
        sbg.check(ws)
    assert e.value.status == sbg.SB_ENONFINITE
    assert sbg.decode_stats(stats)["nonfinite"] == 1
