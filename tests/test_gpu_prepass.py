"""GPU parity of the activation pre-pass against the CPU oracle, through the C ABI.

Bit-exact: rotated values, every FP64 statistic (the reductions follow the same pairwise tree),
INT8 codes and per-token scales, NVFP4 codes, E4M3 block scales (tiled layout, padding
included), the tensor scale and the PDR precision decision.
"""
import numpy as np
import pytest
import torch

import oracle
from video_diffusion_mixed_b200 import synth
from gpu_helpers import npy, u16

pytestmark = pytest.mark.gpu

STATS = ("sum_abs", "sum_d2", "sum_ref2", "max_abs", "amax_rot", "ratio", "d")


def run_prepass(sb, X, R=None, *, force=-1, prec0=None, block=128, rho=64.0, mode=0):
    M, K = X.shape
    ws = sb.Workspace(M, K)
    a4 = sb.Fp4Tensor(M, K)
    a8 = sb.I8Tensor(M, K)
    a4.codes.fill_(0xAB)
    a4.sf.fill_(0xCD)
    a8.codes.fill_(0x55)
    stats = sb.alloc_stats()
    prec = torch.tensor([prec0 if prec0 is not None else (force if force >= 0 else sb.INT8)], dtype=torch.int32,
                        device="cuda")
    cfg = sb.config(rho=rho, block=block, force_prec=force)
    sb.prepass(X, R, cfg, mode, prec, a4, a8, stats, ws)
    sb.check(ws)
    return {"a4": a4, "a8": a8, "stats": sb.decode_stats(stats), "prec": int(prec.item())}


@pytest.mark.parametrize("B,M,K", [(16, 3, 256), (32, 40, 512), (64, 9, 1024), (128, 40, 1024), (256, 5, 1024),
                                   (128, 5, 1920)])
def test_rotate_bitexact(sbg, B, M, K):
    X = synth.activations(M, K, n_outlier=3, scale=20.0, seed=B, device="cuda")
    Y = torch.empty((M, K), dtype=torch.float32, device="cuda")
    sbg.rotate(X, Y, B)
    torch.cuda.synchronize()
    ref = oracle.rotate_rows(u16(X), B)
    assert np.array_equal(npy(Y).view(np.uint32), ref.view(np.uint32))


CASES = [
    # (name, M, K, with_ref, workload-like generator args)
    ("tiny", 256, 256, False, dict(n_outlier=4, scale=20.0)),
    ("ragged_1920", 33, 1920, True, dict(n_outlier=19, scale=30.0, student=True)),
    ("k3072_ref", 300, 3072, True, dict(n_outlier=15, scale=50.0)),
    ("k12288", 70, 12288, False, dict()),
    ("one_row", 1, 7680, True, dict()),
]


@pytest.mark.parametrize("name,M,K,with_ref,gen", CASES, ids=[c[0] for c in CASES])
def test_prepass_int8_bitexact(sbg, name, M, K, with_ref, gen):
    X = synth.activations(M, K, seed=1, tensor_id=1, device="cuda", **gen)
    R = synth.activations(M, K, seed=1, tensor_id=2, device="cuda") if with_ref else None
    out = run_prepass(sbg, X, R, force=sbg.INT8)
    ref = oracle.prepass(u16(X), u16(R) if R is not None else None, 128)
    for k in STATS:
        assert out["stats"][k] == ref[k], (k, out["stats"][k], ref[k])
    assert out["stats"]["has_ref"] == int(with_ref)
    q, s = oracle.quant_int8(ref["y"], ref["row_amax"])
    assert np.array_equal(npy(out["a8"].scale).view(np.uint32), s.view(np.uint32))
    assert np.array_equal(npy(out["a8"].codes), q)
    assert out["prec"] == sbg.INT8  # forced precision is kept


@pytest.mark.parametrize("name,M,K,with_ref,gen", CASES, ids=[c[0] for c in CASES])
def test_prepass_nvfp4_bitexact(sbg, name, M, K, with_ref, gen):
    X = synth.activations(M, K, seed=2, tensor_id=1, device="cuda", **gen)
    out = run_prepass(sbg, X, None, force=sbg.NVFP4)
    ref = oracle.prepass(u16(X), None, 128)
    codes, sfl, sft, sg = oracle.quant_nvfp4(ref["y"], ref["amax_rot"])
    assert np.float32(npy(out["a4"].gscale)[0]) == sg
    assert np.array_equal(npy(out["a4"].codes), codes)
    assert np.array_equal(npy(out["a4"].sf), sft)  # includes the zeroed padding rows
    assert out["stats"]["amax_rot"] == ref["amax_rot"]


@pytest.mark.parametrize("B", [16, 32, 64, 256])
def test_prepass_block_sizes(sbg, B):
    X = synth.activations(50, 1024, n_outlier=5, scale=10.0, seed=B, device="cuda")
    ref = oracle.prepass(u16(X), None, B)
    out8 = run_prepass(sbg, X, force=sbg.INT8, block=B)
    q, s = oracle.quant_int8(ref["y"], ref["row_amax"])
    assert np.array_equal(npy(out8["a8"].codes), q)
    out4 = run_prepass(sbg, X, force=sbg.NVFP4, block=B)
    codes, sfl, sft, sg = oracle.quant_nvfp4(ref["y"], ref["amax_rot"])
    assert np.array_equal(npy(out4["a4"].codes), codes)
    assert np.array_equal(npy(out4["a4"].sf), sft)


@pytest.mark.parametrize("rho", [8.0, 64.0, 1e9])
def test_pdr_decision_matches_oracle(sbg, rho):
    X = synth.activations(256, 256, n_outlier=4, scale=20.0, seed=0, device="cuda")
    ref = oracle.prepass(u16(X), None, 128)
    for p0 in (sbg.NVFP4, sbg.INT8):
        out = run_prepass(sbg, X, prec0=p0, rho=rho)
        assert out["prec"] == oracle.apply_pdr(p0, ref["ratio"], rho), (p0, rho, ref["ratio"])
        assert out["stats"]["prec_in"] == p0 and out["stats"]["prec_out"] == out["prec"]


def test_pdr_ratio_equal_rho_keeps_quantization(sbg):
    # all ones with one 64: max = 64, mean = (n - 1 + 64) / n; rho set to the exact ratio
    X = torch.ones((32, 256), dtype=torch.bfloat16, device="cuda")
    X[3, 17] = 64.0
    ref = oracle.prepass(u16(X), None, 128)
    out = run_prepass(sbg, X, prec0=sbg.NVFP4, rho=ref["ratio"])
    assert out["stats"]["ratio"] == ref["ratio"] and out["prec"] == sbg.NVFP4
    out = run_prepass(sbg, X, prec0=sbg.NVFP4, rho=np.nextafter(ref["ratio"], 0))
    assert out["prec"] == sbg.BF16


def test_skip_leaves_everything_untouched(sbg):
    X = synth.activations(64, 256, seed=3, device="cuda")
    out = run_prepass(sbg, X, prec0=sbg.SKIP)
    assert out["prec"] == sbg.SKIP
    assert (npy(out["a8"].codes) == 0x55).all() and (npy(out["a4"].codes) == 0xAB).all()
    assert all(v == 0 for v in out["stats"].values())


def test_zero_input(sbg):
    X = torch.zeros((40, 512), dtype=torch.bfloat16, device="cuda")
    out8 = run_prepass(sbg, X, force=sbg.INT8)
    assert out8["stats"]["ratio"] == float("inf") and out8["stats"]["sum_abs"] == 0.0
    assert not npy(out8["a8"].codes).any() and not npy(out8["a8"].scale).any()
    out4 = run_prepass(sbg, X, force=sbg.NVFP4)
    assert npy(out4["a4"].gscale)[0] == 1.0
    assert not npy(out4["a4"].codes).any() and not npy(out4["a4"].sf).any()


def test_stats_mode_does_not_touch_precision(sbg):
    X = synth.activations(64, 512, seed=4, device="cuda")
    R = synth.activations(64, 512, seed=5, device="cuda")
    ws = sbg.Workspace(64, 512)
    stats = sbg.alloc_stats()
    sbg.prepass(X, R, sbg.config(rho=0.0), sbg.PREPASS_STATS, None, None, None, stats, ws)
    sbg.check(ws)
    st = sbg.decode_stats(stats)
    ref = oracle.prepass(u16(X), u16(R), 128)
    assert st["d"] == ref["d"] and st["ratio"] == ref["ratio"] and st["prec_out"] == -1


@pytest.mark.parametrize("wl", ["attn2b", "ffn5b"])
def test_prepass_full_size(sbg, wl):
    """Full CogVideoX-sized activations (17776 tokens): statistics, INT8 and NVFP4 bit-exact."""
    X, _ = synth.workload_inputs(wl, seed=0, device="cuda")
    R = synth.noisy_copy(X, 0.1, seed=0)
    out8 = run_prepass(sbg, R, X, force=sbg.INT8)
    ref = oracle.prepass(u16(R), u16(X), 128)
    for k in STATS:
        assert out8["stats"][k] == ref[k], k
    q, s = oracle.quant_int8(ref["y"], ref["row_amax"])
    assert np.array_equal(npy(out8["a8"].codes), q)
    assert np.array_equal(npy(out8["a8"].scale), s)
    out8n = run_prepass(sbg, R, None, force=sbg.INT8)  # no x_ref: the block-per-lane kernel
    for k in ("sum_abs", "max_abs", "amax_rot", "ratio"):
        assert out8n["stats"][k] == ref[k], k
    assert np.array_equal(npy(out8n["a8"].codes), q)
    assert np.array_equal(npy(out8n["a8"].scale), s)
    del out8n
    out4 = run_prepass(sbg, R, None, force=sbg.NVFP4)
    codes, sfl, sft, sg = oracle.quant_nvfp4(ref["y"], ref["amax_rot"])
    assert np.array_equal(npy(out4["a4"].codes), codes)
    assert np.array_equal(npy(out4["a4"].sf), sft)


# Row shapes for every team shape of the block-per-lane pre-pass: several rows per warp (K = 128,
# 384, 1920, 2048), rows straddling warps (640, 3072, 12288, 16384), idle lanes (128, 384, 640,
# 1920, 7680) and a ragged last group of rows.
GEOMS = [(1, 128), (17, 384), (33, 640), (129, 3072), (300, 1920), (7, 12288), (40, 16384), (1000, 2048),
         (20, 7680)]


@pytest.mark.parametrize("M,K", GEOMS, ids=[f"{m}x{k}" for m, k in GEOMS])
def test_prepass_team_shapes(sbg, M, K):
    X = synth.activations(M, K, n_outlier=max(1, K // 200), scale=25.0, seed=M, tensor_id=K, device="cuda")
    ref = oracle.prepass(u16(X), None, 128)
    out8 = run_prepass(sbg, X, force=sbg.INT8)
    for k in ("sum_abs", "max_abs", "amax_rot", "ratio"):
        assert out8["stats"][k] == ref[k], (k, out8["stats"][k], ref[k])
    q, s = oracle.quant_int8(ref["y"], ref["row_amax"])
    assert np.array_equal(npy(out8["a8"].codes), q)
    assert np.array_equal(npy(out8["a8"].scale).view(np.uint32), s.view(np.uint32))
    out4 = run_prepass(sbg, X, force=sbg.NVFP4)
    codes, sfl, sft, sg = oracle.quant_nvfp4(ref["y"], ref["amax_rot"])
    assert np.array_equal(npy(out4["a4"].codes), codes)
    assert np.array_equal(npy(out4["a4"].sf), sft)


@pytest.mark.parametrize("B,with_ref", [(128, False), (256, False), (128, True)])
def test_int8_rows_below_overflow_threshold(sbg, B, with_ref):
    """Rows of subnormal magnitude: 127 / a_m overflows in FP32, so every nonzero code clamps to
    +-127 and zeros stay 0 (both pre-pass kernels, with and without x_ref)."""
    X = (synth.activations(24, 512, seed=11, device="cuda").float() * 1e-39).to(torch.bfloat16)
    X[3] = 0.0                 # an all-zero row: a_m = 0
    X[5, ::3] = 0.0            # zeros inside a tiny row
    X[7] = (X[7].double() * 1e40).to(torch.bfloat16)  # one ordinary row (1e40 overflows FP32)
    R = synth.activations(24, 512, seed=12, device="cuda") if with_ref else None
    ref = oracle.prepass(u16(X), u16(R) if R is not None else None, B)
    assert (ref["row_amax"][[0, 1, 2, 4, 5]] < np.float32(127.0) / np.finfo(np.float32).max).all()
    out8 = run_prepass(sbg, X, R, force=sbg.INT8, block=B)
    q, s = oracle.quant_int8(ref["y"], ref["row_amax"])
    assert np.array_equal(npy(out8["a8"].codes), q)
    assert np.array_equal(npy(out8["a8"].scale).view(np.uint32), s.view(np.uint32))


def test_prepass_hidden_full_size(sbg):
    """The FFN hidden tensor of CogVideoX-5B (17776 x 12288): statistics, INT8 and NVFP4 of the
    block-per-lane pre-pass, bit-exact over every element."""
    X = synth.activations(17776, 12288, n_outlier=61, scale=20.0, seed=0, tensor_id=7, device="cuda")
    ref = oracle.prepass(u16(X), None, 128)
    out8 = run_prepass(sbg, X, force=sbg.INT8)
    for k in ("sum_abs", "max_abs", "amax_rot", "ratio"):
        assert out8["stats"][k] == ref[k], k
    q, s = oracle.quant_int8(ref["y"], ref["row_amax"])
    assert np.array_equal(npy(out8["a8"].codes), q)
    assert np.array_equal(npy(out8["a8"].scale), s)
    del out8, q
    out4 = run_prepass(sbg, X, force=sbg.NVFP4)
    codes, sfl, sft, sg = oracle.quant_nvfp4(ref["y"], ref["amax_rot"])
    assert np.array_equal(npy(out4["a4"].codes), codes)
    assert np.array_equal(npy(out4["a4"].sf), sft)


@pytest.mark.parametrize("K,B,with_ref", [(128, 128, False), (256, 256, False), (128, 128, True)])
def test_prepass_many_groups(sbg, K, B, with_ref):
    """More than 4096 groups of 16 rows (70001 tokens): the last CTA folds the FP64 group sums in
    several chunks of its shared buffer (both pre-pass kernels, with and without x_ref)."""
    M = 70001
    X = synth.activations(M, K, n_outlier=1, scale=30.0, seed=9, device="cuda")
    R = synth.activations(M, K, seed=10, device="cuda") if with_ref else None
    ref = oracle.prepass(u16(X), u16(R) if R is not None else None, B)
    out = run_prepass(sbg, X, R, force=sbg.INT8, block=B)
    for k in STATS:
        assert out["stats"][k] == ref[k], (k, out["stats"][k], ref[k])
    q, s = oracle.quant_int8(ref["y"], ref["row_amax"])
    assert np.array_equal(npy(out["a8"].codes), q)
    assert np.array_equal(npy(out["a8"].scale).view(np.uint32), s.view(np.uint32))


def _block_scale_code(amax: np.float32, s_g: np.float32) -> int:
    """E4M3(RN(RN(amax / 6) / s_g)) with numpy's IEEE FP32 divisions and the oracle's E4M3 cast;
    used only to place inputs on the scale boundaries (expected values come from the oracle)."""
    with np.errstate(over="ignore"):
        q = np.float32(np.float32(amax) / np.float32(6.0))
        return oracle.e4m3_encode(float(np.float32(q / np.float32(s_g))))


def _scale_boundaries(s_g: np.float32) -> list:
    """For every block-scale code c >= 1 reachable from finite amax: the smallest FP32 amax whose
    scale code is >= c (bisection over the ordered bit patterns of non-negative floats)."""
    out = []
    top = _block_scale_code(np.float32(np.finfo(np.float32).max), s_g)
    for c in range(1, top + 1):
        lo, hi = 0, 0x7F7FFFFF
        while lo + 1 < hi:
            mid = (lo + hi) // 2
            if _block_scale_code(np.uint32(mid).view(np.float32), s_g) >= c:
                hi = mid
            else:
                lo = mid
        out.append(np.uint32(hi).view(np.float32))
    return out


def _bf16_parts(v: np.float32):
    """v = p0 + p1 + p2 exactly, each part a bf16 value (8 significant bits apiece)."""
    b = int(np.float32(v).view(np.uint32))
    e, m = (b >> 23) & 0xFF, (b & 0x7FFFFF) | (0x800000 if (b >> 23) & 0xFF else 0)
    scale = 2.0 ** ((e if e else 1) - 150)
    parts = [((m >> 16) << 16) * scale, (((m >> 8) & 0xFF) << 8) * scale, (m & 0xFF) * scale]
    assert sum(parts) == float(v)
    return parts


@pytest.mark.parametrize("A", [1000.0, 0.75, 24576.0])  # bf16-exact tensor maxima
def test_nvfp4_block_scales_on_every_boundary(sbg, A):
    """Group maxima placed exactly on, one ulp below and one ulp above every block-scale rounding
    boundary, for three tensor scales: with B = 16 a block with x0 + x1 + x2 in its first three
    channels (each part a bf16 value) rotates to a group whose amax is exactly the FP32 value
    x0 + x1 + x2. The encode's table-driven scale choice must match the oracle's plain arithmetic
    (two IEEE divisions, then the E4M3 cast) on every such group, codes and scales alike."""
    s_g = np.float32(np.float32(A) / np.float32(2688.0))
    targets = []
    for T in _scale_boundaries(s_g):
        for v in (np.nextafter(T, np.float32(0)), T, np.nextafter(T, np.float32(np.inf))):
            if 0 < v < A:
                targets.append(v)
    K = 2048  # 128 groups of 16 per row
    rows = (len(targets) + 127) // 128 + 1
    X = torch.zeros((rows, K), dtype=torch.float32)
    X[0, 0] = A  # the tensor amax: sets s_g
    for i, v in enumerate(targets):
        r, g = 1 + i // 128, i % 128
        for j, p in enumerate(_bf16_parts(v)):
            X[r, 16 * g + j] = p
    Xb = X.to(torch.bfloat16)
    assert torch.equal(Xb.float(), X)  # every part is bf16-exact
    Xb = Xb.cuda()
    ref = oracle.prepass(u16(Xb), None, 16)
    assert ref["amax_rot"] == A
    out = run_prepass(sbg, Xb, force=sbg.NVFP4, block=16)
    codes, sfl, sft, sg = oracle.quant_nvfp4(ref["y"], ref["amax_rot"])
    assert np.float32(npy(out["a4"].gscale)[0]) == sg == s_g
    # the groups really sit on distinct scale codes on both sides of each boundary
    assert len(np.unique(sfl[1:])) >= 100
    assert np.array_equal(npy(out["a4"].sf), sft)
    assert np.array_equal(npy(out["a4"].codes), codes)
