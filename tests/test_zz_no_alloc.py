"""sb_prepass_static -- the pre-pass for callers that cannot allocate device memory.

Such callers (a plugin whose host program owns the whole device-memory pool, or a loop that must
never call cudaMalloc/cudaFree because they can synchronise the device) cannot provide the
workspace sb_prepass needs; sb_prepass_static keeps that scratch in an array built into the
library instead. These tests call it through the C ABI twice in a row and compare every output
with the workspace version's on the same inputs; both must agree exactly, as the pre-pass outputs
are bit-exact. The file is named so that pytest collects it last.
"""
import numpy as np
import pytest
import torch

from video_diffusion_mixed_b200 import synth

pytestmark = pytest.mark.gpu


def _run(sb, fn, X, R, force, ws=None):
    M, K = X.shape
    a4, a8 = sb.Fp4Tensor(M, K), sb.I8Tensor(M, K)
    a4.codes.zero_()
    a4.sf.zero_()
    a8.codes.zero_()
    stats = sb.alloc_stats()
    prec = torch.tensor([force], dtype=torch.int32, device="cuda")
    cfg = sb.config(rho=64.0, block=128, force_prec=force)
    if fn == "static":
        sb.prepass_static(X, R, cfg, sb.PREPASS_QUANT, prec, a4, a8, stats)
    else:
        sb.prepass(X, R, cfg, sb.PREPASS_QUANT, prec, a4, a8, stats, ws)
    torch.cuda.synchronize()
    return {"q8": a8.codes.cpu(), "s8": a8.scale.cpu(), "c4": a4.codes.cpu(), "sf4": a4.sf.cpu(),
            "g4": a4.gscale[:1].cpu(), "stats": stats.cpu(), "prec": int(prec.item())}


def test_static_scratch_matches_workspace_version_twice_in_a_row(sbg):
    M, K = 3000, 3072
    ws = sbg.Workspace(M, K)
    cases = [
        (synth.activations(M, K, n_outlier=15, scale=50.0, seed=21, device="cuda"), None, sbg.INT8),
        (synth.activations(M, K, seed=22, device="cuda"), synth.activations(M, K, seed=23, device="cuda"),
         sbg.NVFP4),
    ]
    for X, R, force in cases:  # two calls in a row on the shared static scratch
        got = _run(sbg, "static", X, R, force)
        ref = _run(sbg, "ws", X, R, force, ws)
        assert got["prec"] == ref["prec"] == force
        assert torch.equal(got["stats"], ref["stats"])  # every FP64 statistic, bit for bit
        if force == sbg.INT8:
            assert torch.equal(got["q8"], ref["q8"]) and torch.equal(got["s8"], ref["s8"])
        else:
            assert torch.equal(got["c4"], ref["c4"]) and torch.equal(got["sf4"], ref["sf4"])
            assert torch.equal(got["g4"], ref["g4"])
        st = sbg.decode_stats(got["stats"])
        assert st["nonfinite"] == 0 and st["numel"] == M * K
        assert st["error"] == sbg.SB_OK  # the static scratch's device error word, copied out


def test_static_scratch_reports_device_errors_in_stats(sbg):
    """There is no workspace for sb_check to read, so a device-side error of the call reaches the
    caller through stats->error: a NaN in X gives SB_ENONFINITE there. The next call starts from a
    cleared error word and reports SB_OK."""
    M, K = 256, 1024
    X = synth.activations(M, K, seed=24, device="cuda")
    X.view(torch.int16)[17, 99] = 0x7FC0  # a bf16 NaN
    got = _run(sbg, "static", X, None, sbg.INT8)
    st = sbg.decode_stats(got["stats"])
    assert st["error"] == sbg.SB_ENONFINITE and st["nonfinite"] == 1
    Xf = synth.activations(M, K, seed=25, device="cuda")
    got = _run(sbg, "static", Xf, None, sbg.INT8)
    ref = _run(sbg, "ws", Xf, None, sbg.INT8, sbg.Workspace(M, K))
    assert sbg.decode_stats(got["stats"])["error"] == sbg.SB_OK
    assert torch.equal(got["stats"], ref["stats"]) and torch.equal(got["q8"], ref["q8"])


def test_static_scratch_rejects_too_many_rows(sbg):
    import ctypes
    L = sbg.lib()
    cfg = sbg.config()
    M = 65536 + 1
    status = L.sb_prepass_static(ctypes.c_void_p(0x1000), None, M, 256, ctypes.byref(cfg), sbg.PREPASS_STATS,
                                 None, None, None, ctypes.c_void_p(0x2000), None)
    assert status == sbg.SB_ESHAPE
    assert "SB_STATIC_MAX_ROWS" in L.sb_last_error().decode()
