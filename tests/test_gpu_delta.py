"""GPU parity of the delta-token path (DeltaQuant page, abstract; readings R-DQ-* of the oracle).

sb_delta_split is compared bit for bit with the oracle: the core tokens' E4M3 codes and FP32
scales, their bf16 copies and every delta token. The linear layer built from it -- the delta
tokens through the pre-pass and the NVFP4 GEMM, the cores through the BF16 GEMM, the two added per
token by sb_delta_combine -- is compared with the oracle's FP64 result within the GEMM tolerance,
and the combine kernel itself bit for bit against the FP32 sum of the two GEMM outputs it reads.
"""
import numpy as np
import pytest
import torch

import oracle
from video_diffusion_mixed_b200 import synth
from gpu_helpers import assert_close, npy, sample_rows, u16

pytestmark = pytest.mark.gpu

LAYOUTS = [  # (id, text, frames, height, width, cube, K)
    ("tiny_2x2x2", 2, 3, 3, 3, (2, 2, 2), 128),
    ("ragged_2x2x2", 5, 3, 6, 10, (2, 2, 2), 1920),
    ("1x4x4", 0, 2, 8, 8, (1, 4, 4), 256),
    ("2x3x5_30tok", 3, 4, 6, 10, (2, 3, 5), 640),
    ("cogvideox_5b", 226, 13, 30, 45, (2, 2, 2), 3072),
]


def _grid(text, F, H, W, cube):
    return (text, F, H, W) + tuple(cube)


@pytest.mark.parametrize("name,text,F,H,W,cube,K", LAYOUTS, ids=[l[0] for l in LAYOUTS])
def test_delta_split_bitexact(sbg, name, text, F, H, W, cube, K):
    M = text + F * H * W
    X = synth.activations(M, K, n_outlier=max(1, K // 200), scale=30.0, seed=M, tensor_id=K, device="cuda")
    c = sbg.cubes(text, F, H, W, *cube)
    core = sbg.CoreTokens(c, M, K)
    delta = torch.empty_like(X)
    sbg.delta_split(X, c, core, delta)
    torch.cuda.synchronize()
    codes, scale, dec, dref = oracle.delta_split(u16(X), _grid(text, F, H, W, cube))
    assert core.n == len(scale)
    assert np.array_equal(npy(core.codes), codes)
    assert np.array_equal(npy(core.scale).view(np.uint32), scale.view(np.uint32))
    assert np.array_equal(u16(core.bf16), oracle.f32_to_bf16(dec))
    assert np.array_equal(u16(delta), dref)


def test_delta_split_special_values(sbg):
    """Cubes of zeros (scale 0, zero codes, deltas = the tokens), of identical tokens (exact mean),
    of -0 channels next to a nonzero one (the pairwise sum of -0 keeps its sign: E4M3 code 0x80),
    and a cube whose max |mean| is subnormal-small (448 / a overflows: nonzero means take +-448)."""
    text, F, H, W, cube, K = 0, 2, 4, 4, (2, 2, 2), 64
    M = F * H * W
    X = torch.zeros((M, K), dtype=torch.float32)
    g = _grid(text, F, H, W, cube)
    toks = [oracle.cube_tokens(k, g) for k in range(oracle.cube_count(M, g))]
    X[toks[1]] = torch.linspace(-3, 3, K)          # identical tokens
    X[toks[2]] = -0.0                                # negative zeros ...
    X[toks[2], 0] = 1.0                              # ... next to a channel that sets the scale
    X[toks[3], :3] = torch.tensor([1e-39, -2e-39, 0.0])  # tiny means: 448 / a overflows
    Xb = X.to(torch.bfloat16).cuda()
    c = sbg.cubes(text, F, H, W, *cube)
    core = sbg.CoreTokens(c, M, K)
    delta = torch.empty_like(Xb)
    sbg.delta_split(Xb, c, core, delta)
    torch.cuda.synchronize()
    codes, scale, dec, dref = oracle.delta_split(u16(Xb), g)
    assert np.array_equal(npy(core.codes), codes)
    assert np.array_equal(npy(core.scale).view(np.uint32), scale.view(np.uint32))
    assert np.array_equal(u16(delta), dref)
    assert scale[0] == 0.0 and (codes[0] == 0).all()
    assert codes[2, 0] == 0x7E and (codes[2, 1:] == 0x80).all()
    assert codes[3, 0] == 0x7E and codes[3, 1] == 0xFE and codes[3, 2] == 0


def _delta_linear(sbg, X, c, W, bias, gelu):
    """The delta-token linear layer through the C ABI; returns (Y bf16, Yd f32, Yc f32, core, delta)."""
    M, K = X.shape
    N = W.shape[0]
    ws = sbg.Workspace(max(M, N), K)
    w_nb = sbg.Weight(W, None, 128, ws)     # the delta GEMM: no bias
    w_b = sbg.Weight(W, bias, 128, ws)      # the core GEMM carries the bias
    core = sbg.CoreTokens(c, M, K)
    delta = torch.empty_like(X)
    sbg.delta_split(X, c, core, delta)
    a4, a8, st = sbg.Fp4Tensor(M, K), sbg.I8Tensor(M, K), sbg.alloc_stats()
    p4 = torch.tensor([sbg.NVFP4], dtype=torch.int32, device="cuda")
    sbg.prepass(delta, None, sbg.config(force_prec=sbg.NVFP4), sbg.PREPASS_QUANT, p4, a4, a8, st, ws)
    Yd = torch.empty((M, N), dtype=torch.float32, device="cuda")
    sbg.linear(delta, a4, a8, p4, w_nb, Yd, out_dtype=sbg.OUT_F32, ws=ws)
    pb = torch.tensor([sbg.BF16], dtype=torch.int32, device="cuda")
    Yc = torch.empty((core.n, N), dtype=torch.float32, device="cuda")
    sbg.linear(core.bf16, None, None, pb, w_b, Yc, out_dtype=sbg.OUT_F32, ws=ws)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    sbg.delta_combine(Yd, Yc, c, Y, epilogue=sbg.EPI_GELU if gelu else sbg.EPI_NONE)
    sbg.check(ws)
    return Y, Yd, Yc, core, delta


@pytest.mark.parametrize("gelu", [False, True], ids=["linear", "gelu"])
def test_delta_linear_against_oracle(sbg, gelu):
    text, F, H, W_, cube = 7, 4, 6, 10, (2, 2, 2)
    M, K, N = text + F * H * W_, 1920, 768
    X = synth.activations(M, K, n_outlier=19, scale=30.0, student=True, seed=3, device="cuda")
    Wt = synth.weight(N, K, seed=3, device="cuda")
    bias = synth.bias(N, std=0.02, seed=3, device="cuda")
    c = sbg.cubes(text, F, H, W_, *cube)
    Y, Yd, Yc, core, delta = _delta_linear(sbg, X, c, Wt, bias, gelu)
    g = _grid(text, F, H, W_, cube)
    codes, scale, dec, dref = oracle.delta_split(u16(X), g)
    dp = oracle.prepass(dref, None, 128)
    c4, sfl, _, sg = oracle.quant_nvfp4(dp["y"], dp["amax_rot"])
    wp = oracle.prepare_weight(u16(Wt), 128)
    yd_ref = oracle.gemm_nvfp4(c4, sfl, sg, wp["c4"], wp["sf4"], wp["sg4"], None, K, 128)
    ref = oracle.delta_linear(yd_ref, dec, u16(Wt), u16(bias), M, g, gelu=gelu)
    cube_of = np.array([oracle.cube_of_token(t, g) for t in range(M)])
    y32 = npy(Yd) + npy(Yc)[cube_of]  # the two GEMM outputs, added in FP32 as the combine does
    if not gelu:
        assert_close(y32, ref, 1e-3)
        # the combine kernel: the FP32 sum rounded to bf16, bit for bit
        assert np.array_equal(u16(Y), oracle.f32_to_bf16(y32.astype(np.float32)))
    else:
        y = oracle.bf16_to_f32(u16(Y)).astype(np.float64)
        assert_close(y, ref, 5e-3)  # bf16 output rounding (2^-9) on top of the GEMMs' 1e-3


def test_delta_linear_full_size_sampled(sbg):
    """The CogVideoX-2B attention projection shape with the CogVideoX token layout (226 text
    tokens, 13 x 30 x 45 latent grid, 17776 tokens), 2 x 2 x 2 cubes: sampled rows against the
    oracle."""
    text, F, H, W_, cube = 226, 13, 30, 45, (2, 2, 2)
    M, K, N = 17776, 1920, 1920
    X = synth.activations(M, K, n_outlier=19, scale=30.0, student=True, seed=4, device="cuda")
    Wt = synth.weight(N, K, seed=4, device="cuda")
    bias = synth.bias(N, std=0.02, seed=4, device="cuda")
    c = sbg.cubes(text, F, H, W_, *cube)
    Y, Yd, Yc, core, delta = _delta_linear(sbg, X, c, Wt, bias, False)
    g = _grid(text, F, H, W_, cube)
    codes, scale, dec, dref = oracle.delta_split(u16(X), g)
    assert np.array_equal(u16(delta), dref) and np.array_equal(npy(core.codes), codes)
    rows = sample_rows(M)
    dp = oracle.prepass(dref, None, 128)
    c4, sfl, _, sg = oracle.quant_nvfp4(dp["y"], dp["amax_rot"])
    wp = oracle.prepare_weight(u16(Wt), 128)
    yd_ref = oracle.gemm_nvfp4(c4, sfl, sg, wp["c4"], wp["sf4"], wp["sg4"], None, K, 128, rows=rows)
    ref = oracle.delta_linear(yd_ref, dec, u16(Wt), u16(bias), M, g, rows=rows)
    cube_of = np.array([oracle.cube_of_token(t, g) for t in rows])
    y32 = npy(Yd)[rows] + npy(Yc)[cube_of]
    assert_close(y32, ref, 1e-3)


def _fused_delta_linear(sbg, X, c, W, bias, gelu, prec, out_dtype):
    """sb_delta_linear: the cores' product without bias (BF16 GEMM, FP32), then the delta tokens'
    GEMM with the bias and the per-token core row added in its epilogue."""
    M, K = X.shape
    N = W.shape[0]
    ws = sbg.Workspace(max(M, N), K)
    w_nb = sbg.Weight(W, None, 128, ws)
    w_b = sbg.Weight(W, bias, 128, ws)
    core = sbg.CoreTokens(c, M, K)
    delta = torch.empty_like(X)
    sbg.delta_split(X, c, core, delta)
    a4, a8, st = sbg.Fp4Tensor(M, K), sbg.I8Tensor(M, K), sbg.alloc_stats()
    p = torch.tensor([prec], dtype=torch.int32, device="cuda")
    sbg.prepass(delta, None, sbg.config(force_prec=prec), sbg.PREPASS_QUANT, p, a4, a8, st, ws)
    pb = torch.tensor([sbg.BF16], dtype=torch.int32, device="cuda")
    Yc = torch.empty((core.n, N), dtype=torch.float32, device="cuda")
    sbg.linear(core.bf16, None, None, pb, w_nb, Yc, out_dtype=sbg.OUT_F32, ws=ws)
    Y = torch.full((M, N), 7.0, dtype=torch.float32 if out_dtype == sbg.OUT_F32 else torch.bfloat16, device="cuda")
    sbg.delta_linear(delta, a4, a8, p, w_b, Yc, c, Y, epilogue=sbg.EPI_GELU if gelu else sbg.EPI_NONE,
                     out_dtype=out_dtype, ws=ws)
    sbg.check(ws)
    return Y, delta


# N = 768 and 1920: 128- and 192-wide tiles (two accumulators, chunked epilogue); 3072: 256-wide
# NVFP4 tiles (one accumulator, the epilogue drains every column first); BF16: the raw delta tokens
@pytest.mark.parametrize("N,gelu,prec", [(768, False, 0), (768, True, 0), (1920, True, 0), (3072, False, 0),
                                         (1920, False, 1), (1920, False, 2)],
                         ids=["768", "768_gelu", "1920_gelu", "3072", "1920_int8", "1920_bf16"])
def test_fused_delta_linear_against_oracle(sbg, N, gelu, prec):
    text, F, H, W_, cube = 7, 4, 6, 10, (2, 2, 2)
    M, K = text + F * H * W_, 1920
    X = synth.activations(M, K, n_outlier=19, scale=30.0, student=True, seed=5, device="cuda")
    Wt = synth.weight(N, K, seed=5, device="cuda")
    bias = synth.bias(N, std=0.02, seed=5, device="cuda")
    c = sbg.cubes(text, F, H, W_, *cube)
    Y32, delta = _fused_delta_linear(sbg, X, c, Wt, bias, gelu, prec, sbg.OUT_F32)
    Y16, _ = _fused_delta_linear(sbg, X, c, Wt, bias, gelu, prec, sbg.OUT_BF16)
    g = _grid(text, F, H, W_, cube)
    _, _, dec, dref = oracle.delta_split(u16(X), g)
    if prec == 0:
        dp = oracle.prepass(dref, None, 128)
        c4, sfl, _, sg = oracle.quant_nvfp4(dp["y"], dp["amax_rot"])
        wp = oracle.prepare_weight(u16(Wt), 128)
        yd_ref = oracle.gemm_nvfp4(c4, sfl, sg, wp["c4"], wp["sf4"], wp["sg4"], None, K, 128)
    elif prec == 1:
        dp = oracle.prepass(dref, None, 128)
        q8, s8 = oracle.quant_int8(dp["y"], dp["row_amax"])
        wp = oracle.prepare_weight(u16(Wt), 128)
        yd_ref = oracle.gemm_int8(q8, s8, wp["q8"], wp["s8"], None, 128)
    else:
        yd_ref = oracle.gemm_bf16(dref, u16(Wt), None)
    ref = oracle.delta_linear(yd_ref, dec, u16(Wt), u16(bias), M, g, gelu=gelu)
    assert_close(npy(Y32).astype(np.float64), ref, 1e-3)
    # the bf16 output is the same epilogue value rounded to bf16
    assert np.array_equal(u16(Y16), oracle.f32_to_bf16(npy(Y32).astype(np.float32)))


def test_fused_delta_linear_full_size_sampled(sbg):
    """The CogVideoX-2B attention projection with the CogVideoX token layout (17776 tokens),
    sampled rows against the oracle."""
    text, F, H, W_, cube = 226, 13, 30, 45, (2, 2, 2)
    M, K, N = 17776, 1920, 1920
    X = synth.activations(M, K, n_outlier=19, scale=30.0, student=True, seed=6, device="cuda")
    Wt = synth.weight(N, K, seed=6, device="cuda")
    bias = synth.bias(N, std=0.02, seed=6, device="cuda")
    c = sbg.cubes(text, F, H, W_, *cube)
    Y32, delta = _fused_delta_linear(sbg, X, c, Wt, bias, False, 0, sbg.OUT_F32)
    g = _grid(text, F, H, W_, cube)
    _, _, dec, dref = oracle.delta_split(u16(X), g)
    rows = sample_rows(M)
    dp = oracle.prepass(dref, None, 128)
    c4, sfl, _, sg = oracle.quant_nvfp4(dp["y"], dp["amax_rot"])
    wp = oracle.prepare_weight(u16(Wt), 128)
    yd_ref = oracle.gemm_nvfp4(c4, sfl, sg, wp["c4"], wp["sf4"], wp["sg4"], None, K, 128, rows=rows)
    ref = oracle.delta_linear(yd_ref, dec, u16(Wt), u16(bias), M, g, rows=rows)
    assert_close(npy(Y32)[rows].astype(np.float64), ref, 1e-3)
