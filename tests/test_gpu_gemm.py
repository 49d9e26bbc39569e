"""GPU parity of the tcgen05 quantized linear layer against the CPU oracle, through the C ABI.

INT8 accumulators are compared bit-exactly (int32 vs the oracle's int64), at full size too on
sampled rows; NVFP4, INT8 and BF16 outputs within 1e-3 relative Frobenius error of the FP64
dequantized reference (FP32 output mode) and within the matching elementwise bound
(gpu_helpers.assert_close); bf16 outputs within one bf16 ulp of the rounded reference. The weight
preparation (rotation, NVFP4 and INT8 weight copies) is checked bit-exactly first.
"""
import numpy as np
import pytest
import torch

import oracle
from video_diffusion_mixed_b200 import synth
from gpu_helpers import assert_close, bf16_ulp_diff, npy, rel_fro, sample_rows, u16

pytestmark = pytest.mark.gpu
TOL = 1e-3


class Layer:
    def __init__(self, sb, M, N, K, *, seed=0, gen=None, bias_std=0.02, block=128):
        gen = gen or {}
        self.sb, self.M, self.N, self.K, self.block = sb, M, N, K, block
        self.X = synth.activations(M, K, seed=seed, tensor_id=10, device="cuda", **gen)
        self.W = synth.weight(N, K, seed=seed, tensor_id=11, device="cuda")
        self.bias = synth.bias(N, std=bias_std, seed=seed, tensor_id=12, device="cuda")
        self.ws = sb.Workspace(max(M, N), K)
        self.w = sb.Weight(self.W, self.bias, block, self.ws)
        self.a4 = sb.Fp4Tensor(M, K)
        self.a8 = sb.I8Tensor(M, K)
        self.stats = sb.alloc_stats()
        self.prec = torch.zeros(1, dtype=torch.int32, device="cuda")

    def quantize(self, prec):
        self.prec.fill_(prec)
        cfg = self.sb.config(block=self.block, force_prec=prec)
        self.sb.prepass(self.X, None, cfg, self.sb.PREPASS_QUANT, self.prec, self.a4, self.a8, self.stats, self.ws)

    def run(self, prec, out_dtype, gelu=False):
        self.quantize(prec)
        dt = {self.sb.OUT_BF16: torch.bfloat16, self.sb.OUT_F32: torch.float32, self.sb.OUT_RAW: torch.int32}[out_dtype]
        Y = torch.full((self.M, self.N), 7, dtype=dt, device="cuda")
        self.sb.linear(self.X, self.a4, self.a8, self.prec, self.w, Y,
                       epilogue=self.sb.EPI_GELU if gelu else self.sb.EPI_NONE, out_dtype=out_dtype, ws=self.ws)
        self.sb.check(self.ws)
        return Y

    # oracle operands (from the oracle's own quantization of the same bf16 inputs)
    def oracle_ops(self):
        wp = oracle.prepare_weight(u16(self.W), self.block)
        xp = oracle.prepass(u16(self.X), None, self.block)
        q8, s8 = oracle.quant_int8(xp["y"], xp["row_amax"])
        c4, sfl, sft, sg = oracle.quant_nvfp4(xp["y"], xp["amax_rot"])
        return wp, {"q8": q8, "s8": s8, "c4": c4, "sf4": sfl, "sg4": sg}


def test_weight_preparation_bitexact(sbg):
    L = Layer(sbg, 64, 1920, 3072, seed=1)
    torch.cuda.synchronize()
    wp = oracle.prepare_weight(u16(L.W), 128)
    assert np.array_equal(npy(L.w.w8.codes), wp["q8"])
    assert np.array_equal(npy(L.w.w8.scale), wp["s8"])
    assert np.array_equal(npy(L.w.w4.codes), wp["c4"])
    assert np.array_equal(npy(L.w.w4.sf), wp["sf4_tiled"])
    assert np.float32(npy(L.w.w4.gscale)[0]) == wp["sg4"]


SHAPES = [
    ("tiny", 256, 256, 256),
    ("ragged_m", 300, 256, 512),
    ("n1920_k1920", 200, 1920, 1920),   # 128-wide tiles (N % 256 != 0), NVFP4 half K-block
    ("n384_k640", 129, 384, 640),
    ("small_m", 96, 512, 768),          # the second CTA of each pair holds no rows at all
    ("multi_tile", 700, 1024, 1280),    # 3 x 4 tiles of 256 x 256, ragged last row tile
]


@pytest.mark.parametrize("name,M,N,K", SHAPES, ids=[s[0] for s in SHAPES])
def test_int8_accumulators_exact(sbg, name, M, N, K):
    L = Layer(sbg, M, N, K, seed=2)
    acc = L.run(sbg.INT8, sbg.OUT_RAW)
    wp, xp = L.oracle_ops()
    _, ref_acc = oracle.gemm_int8(xp["q8"], xp["s8"], wp["q8"], wp["s8"], None, 128, want_acc=True)
    assert np.array_equal(npy(acc).astype(np.int64), ref_acc)


@pytest.mark.parametrize("name,M,N,K", SHAPES, ids=[s[0] for s in SHAPES])
@pytest.mark.parametrize("gelu", [False, True], ids=["linear", "gelu"])
def test_int8_output(sbg, name, M, N, K, gelu):
    L = Layer(sbg, M, N, K, seed=3)
    Y = L.run(sbg.INT8, sbg.OUT_F32, gelu)
    wp, xp = L.oracle_ops()
    ref = oracle.gemm_int8(xp["q8"], xp["s8"], wp["q8"], wp["s8"], u16(L.bias), 128, gelu=gelu)
    assert_close(npy(Y), ref, TOL)


@pytest.mark.parametrize("name,M,N,K", SHAPES, ids=[s[0] for s in SHAPES])
def test_nvfp4_accumulators(sbg, name, M, N, K):
    L = Layer(sbg, M, N, K, seed=4)
    acc = L.run(sbg.NVFP4, sbg.OUT_RAW)
    wp, xp = L.oracle_ops()
    _, ref_acc = oracle.gemm_nvfp4(xp["c4"], xp["sf4"], xp["sg4"], wp["c4"], wp["sf4"], wp["sg4"], None, K, 128,
                                   want_acc=True)
    got = npy(acc).view(np.float32).astype(np.float64)
    assert rel_fro(got, ref_acc) <= 1e-5


@pytest.mark.parametrize("name,M,N,K", SHAPES, ids=[s[0] for s in SHAPES])
@pytest.mark.parametrize("gelu", [False, True], ids=["linear", "gelu"])
def test_nvfp4_output(sbg, name, M, N, K, gelu):
    L = Layer(sbg, M, N, K, seed=5)
    Y = L.run(sbg.NVFP4, sbg.OUT_F32, gelu)
    wp, xp = L.oracle_ops()
    ref = oracle.gemm_nvfp4(xp["c4"], xp["sf4"], xp["sg4"], wp["c4"], wp["sf4"], wp["sg4"], u16(L.bias), K, 128,
                            gelu=gelu)
    assert_close(npy(Y), ref, TOL)


@pytest.mark.parametrize("name,M,N,K", SHAPES, ids=[s[0] for s in SHAPES])
def test_bf16_output(sbg, name, M, N, K):
    L = Layer(sbg, M, N, K, seed=6)
    Y = L.run(sbg.BF16, sbg.OUT_F32)
    ref = oracle.gemm_bf16(u16(L.X), u16(L.W), u16(L.bias))
    assert_close(npy(Y), ref, TOL)


@pytest.mark.parametrize("prec", [0, 1, 2], ids=["nvfp4", "int8", "bf16"])
def test_bf16_output_mode_within_one_ulp(sbg, prec):
    L = Layer(sbg, 256, 512, 512, seed=7)
    Y = L.run(prec, sbg.OUT_BF16)
    Yf = L.run(prec, sbg.OUT_F32)
    # the bf16 store is the RNE rounding of the FP32 result the kernel computed
    d = bf16_ulp_diff(u16(Y), npy(Yf).astype(np.float64))
    assert d.max() == 0
    wp, xp = L.oracle_ops()
    if prec == 0:
        ref = oracle.gemm_nvfp4(xp["c4"], xp["sf4"], xp["sg4"], wp["c4"], wp["sf4"], wp["sg4"], u16(L.bias), 512, 128)
    elif prec == 1:
        ref = oracle.gemm_int8(xp["q8"], xp["s8"], wp["q8"], wp["s8"], u16(L.bias), 128)
    else:
        ref = oracle.gemm_bf16(u16(L.X), u16(L.W), u16(L.bias))
    d = bf16_ulp_diff(u16(Y), ref)
    assert np.mean(d <= 1) == 1.0


def test_skip_writes_nothing(sbg):
    L = Layer(sbg, 128, 256, 256, seed=8)
    L.quantize(sbg.INT8)
    L.prec.fill_(sbg.SKIP)
    Y = torch.full((128, 256), 3.0, dtype=torch.float32, device="cuda")
    sbg.linear(L.X, L.a4, L.a8, L.prec, L.w, Y, out_dtype=sbg.OUT_F32, ws=L.ws)
    sbg.check(L.ws)
    assert (npy(Y) == 3.0).all()


def test_missing_operands_reported(sbg):
    L = Layer(sbg, 128, 256, 256, seed=9)
    L.quantize(sbg.NVFP4)
    Y = torch.empty((128, 256), dtype=torch.float32, device="cuda")
    sbg.linear(L.X, None, L.a8, L.prec, L.w, Y, out_dtype=sbg.OUT_F32, ws=L.ws)  # NVFP4 chosen, no a4
    with pytest.raises(sbg.SixbitError) as e:
        sbg.check(L.ws)
    assert e.value.status == sbg.SB_EINVAL


FULL = [  # (id, N, K, GELU): CogVideoX-5B FFN, CogVideoX-2B attention projection and FFN
    ("5b_w1", 12288, 3072, True), ("5b_w2", 3072, 12288, False),
    ("2b_attn", 1920, 1920, False), ("2b_w1", 7680, 1920, True), ("2b_w2", 1920, 7680, False),
]


@pytest.mark.parametrize("name,N,K,gelu", FULL, ids=[f[0] for f in FULL])
@pytest.mark.parametrize("prec", [0, 1, 2], ids=["nvfp4", "int8", "bf16"])
def test_full_size_sampled(sbg, name, N, K, gelu, prec):
    """DiT layers at full shape (17776 tokens): every 64th row plus the last one against the
    oracle (FP32 output), and the bf16 output -- the TMA-store epilogue, last tile clipped at
    M -- equal to the RNE rounding of the kernel's FP32 result over every element. At 17776 tokens
    every layer has more output tiles than the persistent grid has CTA pairs (74), so each pair
    runs several tiles: the accumulator buffers alternate and the barrier phases wrap, for the
    BF16 fallback (K up to 12288, 192 K-blocks of 64) as for the quantized kinds."""
    M = synth.TOKENS
    L = Layer(sbg, M, N, K, seed=10, gen=dict(n_outlier=15, scale=50.0) if gelu else {})
    Y = L.run(prec, sbg.OUT_F32, gelu=gelu)
    Yb = L.run(prec, sbg.OUT_BF16, gelu=gelu)
    assert torch.equal(Yb, Y.to(torch.bfloat16))
    rows = sample_rows(M)
    wp, xp = L.oracle_ops() if prec != 2 else (None, None)
    if prec == 0:
        ref = oracle.gemm_nvfp4(xp["c4"], xp["sf4"], xp["sg4"], wp["c4"], wp["sf4"], wp["sg4"], u16(L.bias), K, 128,
                                gelu=gelu, rows=rows)
    elif prec == 1:
        ref = oracle.gemm_int8(xp["q8"], xp["s8"], wp["q8"], wp["s8"], u16(L.bias), 128, gelu=gelu, rows=rows)
    else:
        ref = oracle.gemm_bf16(u16(L.X), u16(L.W), u16(L.bias), gelu=gelu, rows=rows)
    assert_close(npy(Y)[rows], ref, TOL)


FULL_I8 = [("5b_w1", 12288, 3072), ("5b_w2", 3072, 12288), ("2b_w2", 1920, 7680)]


@pytest.mark.parametrize("name,N,K", FULL_I8, ids=[f[0] for f in FULL_I8])
def test_int8_accumulators_full_size_sampled(sbg, name, N, K):
    """The raw int32 accumulators of the INT8 kind at full shape (17776 tokens, K = 3072 / 12288 /
    7680: 24 / 96 / 60 K-blocks per tile, several tiles per CTA pair) equal the oracle's int64
    sums on every 64th row and the last one, bit for bit."""
    M = synth.TOKENS
    L = Layer(sbg, M, N, K, seed=11, gen=dict(n_outlier=15, scale=50.0))
    acc = L.run(sbg.INT8, sbg.OUT_RAW)
    rows = sample_rows(M)
    wp, xp = L.oracle_ops()
    _, ref_acc = oracle.gemm_int8(xp["q8"], xp["s8"], wp["q8"], wp["s8"], None, 128, rows=rows, want_acc=True)
    assert np.array_equal(npy(acc)[rows].astype(np.int64), ref_acc)
