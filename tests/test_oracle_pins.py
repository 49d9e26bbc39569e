"""Pins of the CPU oracle against what the formats, the mathematics and the pages fix.

None of these tests retypes an oracle formula: each checks a closed form, an invariant, a value
worked by hand (tests/golden/, with citations), an independent library routine (scipy's
Hadamard matrix, numpy matmul, ml_dtypes' OCP format casts, torch's GELU) or a brute-force
search, chosen so a dropped term, a wrong sign, a wrong index or a transposed operand fails.
"""
import math
import os

import numpy as np
import pytest
import torch

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    rows = []
    with open(os.path.join(GOLD, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


def _bf16(a):
    return torch.from_numpy(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)


# ------------------------------------------------------------------------------------------------
# Hadamard (R-H)
# ------------------------------------------------------------------------------------------------

@pytest.mark.parametrize("B", [16, 32, 64, 128, 256])
def test_fwht_matches_sylvester_matrix(orc, B):
    import scipy.linalg
    H = scipy.linalg.hadamard(B)  # Sylvester construction, natural order
    for i in range(B):
        e = np.zeros(B, np.float32)
        e[i] = 1.0
        col = orc.fwht(e, B)
        assert np.array_equal(col, H[:, i].astype(np.float32))
        for j in range(0, B, max(1, B // 8)):
            assert orc.hadamard_entry(j, i) == H[j, i]


@pytest.mark.parametrize("B", [16, 128, 256])
def test_fwht_orthogonality_and_involution(orc, B):
    rows = np.stack([orc.fwht(np.eye(B, dtype=np.float32)[i], B) for i in range(B)])
    assert np.array_equal(rows @ rows.T, B * np.eye(B))  # H H^T = B I exactly
    rng = np.random.default_rng(1)
    x = rng.integers(-8, 9, size=4 * B).astype(np.float32)
    assert np.array_equal(orc.fwht(orc.fwht(x, B), B), B * x)  # H (H x) = B x, exact
    xr = rng.standard_normal(B).astype(np.float32)
    y = orc.fwht(xr, B).astype(np.float64)
    # Parseval: |Hx|^2 = B |x|^2 within the FP32 butterfly's error bound (log2 B roundings)
    rel = abs(np.dot(y, y) - B * np.dot(xr.astype(np.float64), xr)) / (B * np.dot(xr, xr))
    assert rel < 4 * math.log2(B) * 2.0 ** -23


def test_rotate_rows_blockwise(orc):
    import scipy.linalg
    rng = np.random.default_rng(2)
    x = _bf16(rng.standard_normal((5, 384)))
    y = orc.rotate_rows(x, 128)
    H = scipy.linalg.hadamard(128).astype(np.float64)
    xf = x.float().numpy().astype(np.float64)
    for j in range(3):
        ref = xf[:, 128 * j:128 * (j + 1)] @ H.T
        assert np.allclose(y[:, 128 * j:128 * (j + 1)], ref, rtol=0, atol=1e-4)


# ------------------------------------------------------------------------------------------------
# Reductions (R-RED)
# ------------------------------------------------------------------------------------------------

def test_pairwise_order_hand_worked(orc):
    big = 2.0 ** 24
    # [2^24,1,1,1]: pairwise (2^24+1 -> 2^24 by ties-to-even) + (1+1) = 2^24+2;
    # a left-to-right sum would give 2^24.
    assert orc.pairwise_f32(np.array([big, 1, 1, 1], np.float32)) == np.float32(big + 2)
    # n=3 pads with one zero: (2^24+1 -> 2^24) + (1+0) -> 2^24+1 -> 2^24 (tie, even)
    assert orc.pairwise_f32(np.array([big, 1, 1], np.float32)) == np.float32(big)
    # n=5 pads to 8: ((2^24)+(2)) + ((1+0)+(0+0)) = 2^24+3 -> tie between +2 and +4 -> 2^24+4
    assert orc.pairwise_f32(np.array([big, 1, 1, 1, 1], np.float32)) == np.float32(big + 4)
    assert orc.pairwise_f32(np.zeros(0, np.float32)) == 0.0


def test_pairwise_f64_order_hand_worked(orc):
    """The FP64 tree across row groups: the same hand-worked cases one precision up, which a
    left-to-right (or right-to-left) FP64 fold gets wrong."""
    big = 2.0 ** 53
    # [2^53,1,1,1]: (2^53+1 -> 2^53, tie to even) + (1+1) = 2^53+2; a left-to-right sum gives 2^53
    assert orc.pairwise_f64(np.array([big, 1, 1, 1])) == big + 2
    # n=3 pads with one zero: 2^53 + (1+0) -> 2^53 (tie, even)
    assert orc.pairwise_f64(np.array([big, 1, 1])) == big
    # n=5 pads to 8: (2^53 + 2) + 1 = 2^53+3 -> tie between +2 and +4 -> 2^53+4
    assert orc.pairwise_f64(np.array([big, 1, 1, 1, 1])) == big + 4
    # right-to-left would give (1+1+1) + 2^53 = 2^53+4 for the first case; the tree gives +2
    assert orc.pairwise_f64(np.array([1, 1, 1, big])) == big + 2
    # [1, 2^53, 1, 1]: (1+2^53 -> 2^53) + (1+1) = 2^53+2
    assert orc.pairwise_f64(np.array([1, big, 1, 1])) == big + 2
    assert orc.pairwise_f64(np.zeros(0)) == 0.0


def test_f32_to_bf16_matches_ml_dtypes(orc):
    """The comparison helper that rounds FP64/FP32 references to bf16 agrees with ml_dtypes' own
    round-to-nearest-even cast on random values of every magnitude, on every tie (the 16 low bits
    exactly 0x8000, with an even and an odd kept bit), on subnormals, at the overflow edge and on
    infinities; a NaN stays a NaN."""
    ml = pytest.importorskip("ml_dtypes")
    rng = np.random.default_rng(17)
    bits = rng.integers(0, 2 ** 32, 200000, dtype=np.uint64).astype(np.uint32)
    ties = (rng.integers(0, 2 ** 16, 5000, dtype=np.uint64).astype(np.uint32) << 16) | 0x8000
    edge = np.array([0x7F7F7FFF, 0x7F7F8000, 0x7F7FFFFF, 0xFF7F8000, 0x00008000, 0x00018000, 0x0000FFFF,
                     0x80008000, 0x7F800000, 0xFF800000, 0x00000000, 0x80000000, 0x3F808000, 0x3F818000],
                    dtype=np.uint32)
    x = np.concatenate([bits, ties, edge]).view(np.float32)
    x = x[~np.isnan(x)]
    ref = x.astype(ml.bfloat16).view(np.uint16)
    assert np.array_equal(orc.f32_to_bf16(x), ref)
    nan = np.array([np.nan, -np.nan], dtype=np.float32)
    assert np.isnan(orc.bf16_to_f32(orc.f32_to_bf16(nan))).all()


def test_pairwise_accuracy(orc):
    rng = np.random.default_rng(3)
    t = rng.random(10007).astype(np.float32)
    exact = math.fsum(t.astype(np.float64))
    assert abs(float(orc.pairwise_f32(t)) - exact) / exact < 16 * 2.0 ** -24
    ti = rng.integers(0, 1000, 777).astype(np.float64)
    assert orc.pairwise_f64(ti) == float(ti.sum())


# ------------------------------------------------------------------------------------------------
# Number formats
# ------------------------------------------------------------------------------------------------

def test_e2m1_table_and_roundtrip(orc):
    for code, val in _golden("e2m1_table.txt"):
        c, v = int(code), float(val)
        assert orc.e2m1_decode(c) == v and math.copysign(1, orc.e2m1_decode(c)) == math.copysign(1, v)
        assert orc.e2m1_encode(np.float32(v)) == c  # encode(decode(c)) = c, incl. -0


def test_e4m3_table_and_roundtrip(orc):
    for code, val in _golden("e4m3_values.txt"):
        assert orc.e4m3_decode(int(code, 16)) == float(val)
    ref = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    for c in range(256):
        v = orc.e4m3_decode(c)
        if c & 0x7F == 0x7F:
            assert math.isnan(v) and math.isnan(ref[c])
            continue
        assert v == ref[c]
        assert orc.e4m3_encode(np.float32(v)) == c


def test_rounding_ties_golden(orc):
    for fmt, inp, code in _golden("rounding_ties.txt"):
        v = np.float32(float(inp))
        got = orc.e2m1_encode(v) if fmt == "e2m1" else orc.e4m3_encode(v)
        assert got == int(code, 16), (fmt, inp)


def test_encoders_match_ml_dtypes(orc):
    """ml_dtypes implements the OCP casts (round-to-nearest-even) independently of the oracle."""
    ml = pytest.importorskip("ml_dtypes")
    rng = np.random.default_rng(4)
    v = np.concatenate([rng.uniform(-7, 7, 4000), rng.standard_normal(2000) * 0.3,
                        np.arange(-6.5, 6.6, 0.125)]).astype(np.float32)
    ref = v.astype(ml.float4_e2m1fn).view(np.uint8) & 0xF
    got = np.array([orc.e2m1_encode(x) for x in v], np.uint8)
    assert np.array_equal(got, ref)
    s = np.concatenate([rng.uniform(0, 440, 3000), np.exp2(rng.uniform(-12, 8, 3000))]).astype(np.float32)
    ref = s.astype(ml.float8_e4m3fn).view(np.uint8)
    got = np.array([orc.e4m3_encode(x) for x in s], np.uint8)
    assert np.array_equal(got, ref)


def test_sf_tiled_layout_golden(orc):
    for m, g, K, off in _golden("sf_tiled_layout.txt"):
        assert orc.sf_tiled_offset(int(m), int(g), int(K)) == int(off)
    # bijection over the padded buffer for a ragged row count
    M, K = 300, 192
    seen = set()
    for m in range(((M + 127) // 128) * 128):
        for g in range(K // 16):
            seen.add(orc.sf_tiled_offset(m, g, K))
    assert seen == set(range(orc.sf_tiled_bytes(M, K)))


# ------------------------------------------------------------------------------------------------
# Quantizers
# ------------------------------------------------------------------------------------------------

def test_int8_quant_properties(orc):
    rng = np.random.default_rng(5)
    y = (rng.standard_normal((7, 256)) * rng.uniform(0.1, 50, (7, 1))).astype(np.float32)
    y[3] = 0.0
    amax = np.abs(y).max(1).astype(np.float32)
    q, s = orc.quant_int8(y, amax)
    assert s[3] == 0 and not q[3].any()
    for m in [0, 1, 2, 4, 5, 6]:
        i = int(np.argmax(np.abs(y[m])))
        assert q[m, i] == (127 if y[m, i] > 0 else -127)  # the amax element maps to +-127
        assert np.float32(s[m]) == np.float32(amax[m] / np.float32(127))
        err = np.abs(q[m].astype(np.float64) * s[m] - y[m])
        assert err.max() <= 0.5 * s[m] * (1 + 1e-5)
        # brute force: nearest integer in [-127, 127] of y * (127 / a), ties to even
        v = (y[m] * np.float32(np.float32(127) / amax[m])).astype(np.float64)
        cand = np.arange(-127, 128)
        d = np.abs(v[:, None] - cand[None, :])
        best = cand[np.argmin(d + 1e-9 * (cand[None, :] & 1), axis=1)]
        assert np.array_equal(q[m].astype(np.int64), best)


def test_int8_quant_overflowing_reciprocal(orc):
    """FP32 reading of R-INT8 when 127 / a overflows (a below 127 / FLT_MAX): the reciprocal is +inf,
    every nonzero y lands on +-127 (numpy's FP32 arithmetic gives the same +-inf products) and y = 0,
    whose exact product is 0, stays 0; s = a / 127 is still the correctly rounded quotient."""
    a = np.float32(1e-38)
    assert np.isinf(np.float32(127) / a)
    y = np.array([[a, a / 2, 0.0, -a / 4, -a, np.float32(1e-45)]], dtype=np.float32)
    y = np.pad(y, ((0, 0), (0, 128 - y.shape[1])))
    q, s = orc.quant_int8(y, np.array([a], dtype=np.float32))
    assert q[0, :6].tolist() == [127, 127, 0, -127, -127, 127] and not q[0, 6:].any()
    assert s[0] == np.float32(a / np.float32(127))


def test_chunk_stats_closed_forms(orc):
    """Chunk records against exact arithmetic: small integers make every FP32 sum exact, so the
    rotated amax is max |x H_B^T| from the explicit +-1 matrix and the sum is the integer sum."""
    rng = np.random.default_rng(21)
    M, K = 5, 512
    xi = rng.integers(-8, 9, size=(M, K))
    xi[2] = 0
    xi[3, :] = 1  # a constant row: the rotation puts 128 (B = 128) or B in the first slot of a block
    x = orc.f32_to_bf16(xi.astype(np.float32))
    for B in (16, 128):
        H = np.array([[orc.hadamard_entry(i, j) for j in range(B)] for i in range(B)], dtype=np.int64)
        cs = orc.chunk_stats(x, B)
        assert cs.shape == (M, K // 128, 3)
        for m in range(M):
            for c in range(K // 128):
                v = xi[m, 128 * c:128 * (c + 1)]
                rot = (v.reshape(-1, B) @ H.T).ravel()
                assert cs[m, c, 0] == np.abs(rot).max()
                assert cs[m, c, 1] == np.abs(v).sum()
                assert cs[m, c, 2] == np.abs(v).max()
        assert (cs[3, :, 0] == B).all() and (cs[3, :, 1] == 128).all() and not cs[2].any()


def test_chunk_stats_fold_to_the_row_statistics(orc):
    """The chunks are aligned subtrees of each row's pairwise tree: folding a row's chunk sums
    (zero-padded to a power of two) gives the pre-pass row sum bit for bit, and the chunk maxima
    give the per-token rotated amax and the raw max."""
    rng = np.random.default_rng(22)
    M, K = 7, 12288
    x = orc.f32_to_bf16((rng.standard_normal((M, K)) * rng.uniform(0.01, 40.0, (M, 1))).astype(np.float32))
    cs = orc.chunk_stats(x, 128)
    ref = orc.prepass(x, None, 128)
    for m in range(M):
        assert np.float32(orc.pairwise_f32(cs[m, :, 1])) == ref["row_part"][m, 0]
        assert cs[m, :, 0].max() == ref["row_amax"][m]
    assert float(cs[:, :, 2].max()) == ref["max_abs"]


def test_nvfp4_quant_properties(orc):
    rng = np.random.default_rng(6)
    y = (rng.standard_normal((9, 128)) * rng.uniform(0.01, 30, (9, 1))).astype(np.float32)
    y[4, 16:32] = 0.0
    A = float(np.abs(y).max())
    codes, sfl, sft, sg = orc.quant_nvfp4(y, A)
    assert sg == np.float32(np.float32(A) / np.float32(2688.0))
    t2 = orc.e2m1_table()
    t4 = orc.e4m3_table()
    dq = orc.nvfp4_dequant(codes, sfl)  # without s_g
    for m in range(9):
        for g in range(8):
            blk = y[m, 16 * g:16 * (g + 1)].astype(np.float64)
            sb = sfl[m, g]
            # the block scale is the nearest E4M3 of amax_g / 6 / s_g
            target = (np.float32(np.float32(np.abs(blk).max()) / np.float32(6.0)) / sg)
            cands = t4[:127]
            dist = np.abs(cands - float(target))
            assert dist[sb] == dist.min()
            den = float(np.float32(t4[sb]) * sg)
            if den == 0:
                assert not dq[m, 16 * g:16 * (g + 1)].any()
                continue
            vals = dq[m, 16 * g:16 * (g + 1)] / t4[sb]  # E2M1 values
            scaled = blk / den
            # each code is a nearest E2M1 value of y / den (within FP32 rounding of y * (1/den))
            grid = t2[:8]
            for v, s in zip(vals, scaled):
                s_clamped = max(-6.0, min(6.0, s))
                nearest = np.min(np.abs(grid - abs(s_clamped)))
                assert abs(abs(v) - abs(s_clamped)) <= nearest + 1e-6 * abs(s) + 1e-12
                assert v == 0 or np.sign(v) == np.sign(s)
    assert (sft.size == orc.sf_tiled_bytes(9, 128))
    for m in range(9):
        for g in range(8):
            assert sft[orc.sf_tiled_offset(m, g, 128)] == sfl[m, g]
    pad = np.ones(sft.size, bool)
    for m in range(9):
        for g in range(8):
            pad[orc.sf_tiled_offset(m, g, 128)] = False
    assert not sft[pad].any()  # padding rows of the tiled layout are zero


def test_nvfp4_zero_tensor(orc):
    codes, sfl, sft, sg = orc.quant_nvfp4(np.zeros((3, 64), np.float32), 0.0)
    assert sg == 1.0 and not codes.any() and not sfl.any() and not sft.any()


# ------------------------------------------------------------------------------------------------
# Pre-pass statistics: closed forms
# ------------------------------------------------------------------------------------------------

def test_prepass_closed_forms(orc):
    M, K = 33, 256
    x = np.ones((M, K), np.float32)
    x[7, 100] = 64.0
    xr = np.full((M, K), 2.0, np.float32)
    y = np.ones((M, K), np.float32) * 3.0  # y - xr = 1 everywhere
    st = orc.prepass(_bf16(x), None, 128)
    numel = M * K
    assert st["max_abs"] == 64.0
    assert st["sum_abs"] == numel - 1 + 64
    assert st["ratio"] == 64.0 / ((numel - 1 + 64) / numel)
    assert st["d"] == 0.0
    # amax of the rotated rows: an all-ones block rotates to (128, 0, ..., 0)
    assert st["row_amax"][0] == 128.0 and st["amax_rot"] == 128.0 + 63.0
    st2 = orc.prepass(_bf16(y), _bf16(xr), 128)
    assert st2["sum_d2"] == numel and st2["sum_ref2"] == 4.0 * numel
    assert st2["d"] == 0.5  # sqrt(n) / sqrt(4 n)


def test_prepass_sums_accuracy(orc):
    rng = np.random.default_rng(7)
    x = _bf16(rng.standard_normal((300, 384)))
    r = _bf16(rng.standard_normal((300, 384)))
    st = orc.prepass(x, r, 128)
    xf = x.float().numpy().astype(np.float64)
    rf = r.float().numpy().astype(np.float64)
    assert abs(st["sum_abs"] - math.fsum(np.abs(xf).ravel())) / st["sum_abs"] < 1e-5
    assert abs(st["sum_d2"] - math.fsum(((xf - rf) ** 2).ravel())) / st["sum_d2"] < 1e-5
    assert abs(st["d"] - np.linalg.norm(xf - rf) / np.linalg.norm(rf)) < 1e-6


# ------------------------------------------------------------------------------------------------
# GEMMs
# ------------------------------------------------------------------------------------------------

def test_gemm_int8_exact_and_epilogue(orc):
    rng = np.random.default_rng(8)
    qx = rng.integers(-127, 128, (37, 256)).astype(np.int8)
    qw = rng.integers(-127, 128, (24, 256)).astype(np.int8)
    sx = rng.uniform(0.01, 1, 37).astype(np.float32)
    sw = rng.uniform(0.01, 1, 24).astype(np.float32)
    b = _bf16(rng.standard_normal(24) * 0.1)
    Y, acc = orc.gemm_int8(qx, sx, qw, sw, b, 128, want_acc=True)
    ref_acc = qx.astype(np.int64) @ qw.astype(np.int64).T
    assert np.array_equal(acc, ref_acc)
    ref = ref_acc * sx[:, None].astype(np.float64) * sw[None, :].astype(np.float64) / 128 + b.float().numpy()
    assert np.allclose(Y, ref, rtol=1e-12, atol=1e-12)
    rows = np.array([0, 5, 36])
    Ys = orc.gemm_int8(qx, sx, qw, sw, b, 128, rows=rows)
    assert np.array_equal(Ys, Y[rows])


def test_gemm_nvfp4_integer_exact(orc):
    rng = np.random.default_rng(9)
    M, N, K = 20, 16, 128
    xc = rng.integers(0, 256, (M, K // 2)).astype(np.uint8)
    wc = rng.integers(0, 256, (N, K // 2)).astype(np.uint8)
    xs = np.full((M, K // 16), 0x38, np.uint8)  # scale 1.0
    ws = np.full((N, K // 16), 0x40, np.uint8)  # scale 2.0
    xs[3, 2] = 0x30  # 0.5
    Y = orc.gemm_nvfp4(xc, xs, 1.0, wc, ws, 1.0, None, K, 1)
    X = orc.nvfp4_dequant(xc, xs)
    W = orc.nvfp4_dequant(wc, ws)
    assert np.array_equal(Y, X @ W.T)  # half-integers: exact in FP64
    # transposition check: the result is not symmetric in the roles of x and w
    Yt = orc.gemm_nvfp4(wc, ws, 1.0, xc, xs, 1.0, None, K, 1)
    assert np.array_equal(Yt, Y.T)
    # nibble order: element 2i is the low nibble
    one = np.zeros((1, K // 2), np.uint8)
    one[0, 0] = 0x02  # element 0 = 1.0, element 1 = 0
    sel = np.zeros((2, K // 2), np.uint8)
    sel[0, 0] = 0x02  # w0 picks element 0
    sel[1, 0] = 0x20  # w1 picks element 1
    y = orc.gemm_nvfp4(one, np.full((1, K // 16), 0x38, np.uint8), 1.0, sel,
                       np.full((2, K // 16), 0x38, np.uint8), 1.0, None, K, 1)
    assert y[0, 0] == 1.0 and y[0, 1] == 0.0


def test_gemm_rotation_fold(orc):
    """(X H)(W H)^T / B = X W^T: rotating both operands and scaling by 1/B is exact algebra."""
    import scipy.linalg
    rng = np.random.default_rng(10)
    B, K = 128, 256
    X = rng.standard_normal((6, K))
    W = rng.standard_normal((5, K))
    H = scipy.linalg.block_diag(scipy.linalg.hadamard(B), scipy.linalg.hadamard(B)).astype(np.float64)
    lhs = (X @ H.T) @ (W @ H.T).T / B
    assert np.allclose(lhs, X @ W.T, rtol=0, atol=1e-12)
    # and the oracle's rotation applies H^T per block (H is symmetric): compare on bf16 data
    xb = _bf16(X)
    y = orc.rotate_rows(xb, B).astype(np.float64)
    assert np.allclose(y, xb.float().numpy().astype(np.float64) @ H.T, atol=1e-4)


def test_gemm_bf16_and_gelu(orc):
    rng = np.random.default_rng(11)
    x = _bf16(rng.standard_normal((9, 64)))
    w = _bf16(rng.standard_normal((7, 64)))
    b = _bf16(rng.standard_normal(7))
    Y = orc.gemm_bf16(x, w, b, gelu=True)
    lin = x.double() @ w.double().T + b.double()
    ref = torch.nn.functional.gelu(lin, approximate="tanh").numpy()
    assert np.allclose(Y, ref, rtol=1e-12, atol=1e-12)
    assert abs(orc.gelu_tanh(1.0) - 0.8411919906082768) < 1e-15


# ------------------------------------------------------------------------------------------------
# Temporal Delta Cache and decisions (closed-form schedules)
# ------------------------------------------------------------------------------------------------

def test_tdc_delta_closed_form(orc):
    a = _bf16(np.full((17, 96), 1.25))
    b = _bf16(np.full((17, 96), 1.0))
    d, s1, s2 = orc.tdc_delta(a, b)
    assert d == 0.25 and s1 == 0.25 * 17 * 96 and s2 == 17 * 96
    d0, _, _ = orc.tdc_delta(a, _bf16(np.zeros((17, 96))))
    assert d0 == math.inf


def test_tdc_reuse_matches_ml_dtypes_rounding(orc):
    """R-REUSE through an independent bf16 implementation: ml_dtypes' float32 -> bfloat16 cast
    (round to nearest even) of the FP32 difference / sum of the bf16 values."""
    ml = pytest.importorskip("ml_dtypes")
    rng = np.random.default_rng(11)
    # values of very different magnitude, so the FP32 difference and the bf16 rounding both bite
    x = (rng.standard_normal(6000) * np.exp2(rng.integers(-20, 20, 6000))).astype(np.float32).astype(ml.bfloat16)
    y = (rng.standard_normal(6000) * np.exp2(rng.integers(-20, 20, 6000))).astype(np.float32).astype(ml.bfloat16)
    xb, yb = x.view(np.uint16), y.view(np.uint16)
    ref_d = (y.astype(np.float32) - x.astype(np.float32)).astype(ml.bfloat16)
    d = orc.tdc_refresh(xb, yb)
    assert np.array_equal(d, ref_d.view(np.uint16))
    ref_y = (x.astype(np.float32) + ref_d.astype(np.float32)).astype(ml.bfloat16)
    assert np.array_equal(orc.tdc_reuse(xb, d), ref_y.view(np.uint16))


def test_tdc_reuse_closed_form(orc):
    """Small integers: every step is exact, so a reuse with the same input returns the output;
    a zero residual returns the input; equal input and output keep a +0 residual."""
    x = _bf16(np.arange(-64, 64, dtype=np.float64).reshape(8, 16))
    y = _bf16((np.arange(-64, 64, dtype=np.float64) * 3 + 5).reshape(8, 16))
    xb, yb = x.view(torch.int16).numpy().view(np.uint16), y.view(torch.int16).numpy().view(np.uint16)
    d = orc.tdc_refresh(xb, yb)
    assert np.array_equal(orc.tdc_reuse(xb, d), yb)
    assert np.array_equal(orc.tdc_reuse(xb, np.zeros_like(xb)), xb)
    assert np.array_equal(orc.tdc_refresh(xb, xb), np.zeros_like(xb))  # +0, not -0


def test_tdc_fp8_residual_closed_form(orc):
    """R-REUSE-FP8 on rows whose residuals are integers with row maximum 7: s = 7 / 448 = 2^-6 is
    exact, every d / s = 64 d is an E4M3 value, so codes decode exactly and a reuse with the same
    input returns the output bit for bit. A zero row keeps s = 0, zero codes and returns x."""
    rng = np.random.default_rng(12)
    M, C = 6, 40
    x = rng.integers(-50, 50, (M, C)).astype(np.float64)
    d = rng.integers(-7, 8, (M, C)).astype(np.float64)
    d[:, 0] = np.where(np.arange(M) % 2 == 0, 7, -7)  # row max |d| = 7, either sign
    d[M - 1] = 0.0
    xb = _bf16(x).view(torch.int16).numpy().view(np.uint16)
    yb = _bf16(x + d).view(torch.int16).numpy().view(np.uint16)
    codes, scale = orc.tdc_refresh_fp8(xb, yb)
    assert np.array_equal(scale[:M - 1], np.full(M - 1, 2.0 ** -6, dtype=np.float32))
    assert scale[M - 1] == 0.0 and not codes[M - 1].any()
    # 64 d: 0 -> 0x00, 64 -> 0x60 (2^6), 448 -> 0x7e, and the sign bit for negative d
    assert codes[0, 0] == 0x7E and codes[1, 0] == 0xFE
    dec = np.array([orc.e4m3_decode(int(c)) for c in codes.ravel()], dtype=np.float64).reshape(M, C)
    assert np.array_equal(dec * 2.0 ** -6, d)
    assert np.array_equal(orc.tdc_reuse_fp8(xb, codes, scale), yb)


def test_tdc_fp8_residual_matches_ml_dtypes_and_error_bound(orc):
    """R-REUSE-FP8 through independent implementations: the codes are ml_dtypes' E4M3 cast of the
    FP32 residual times 448 / a, the output is ml_dtypes' bf16 cast of x + dec; the decoded residual
    is within half an E4M3 step of d (2^-4 relative for normals, 2^-10 s absolute for subnormals)."""
    ml = pytest.importorskip("ml_dtypes")
    rng = np.random.default_rng(13)
    M, C = 24, 96
    xs = np.exp2(rng.integers(-8, 8, (M, 1)))
    x = (rng.standard_normal((M, C)) * xs).astype(np.float32).astype(ml.bfloat16)
    y = (x.astype(np.float32) + rng.standard_normal((M, C)).astype(np.float32) * 0.1 * xs.astype(np.float32)
         * np.exp2(rng.integers(-12, 1, (M, C))).astype(np.float32)).astype(ml.bfloat16)
    xb, yb = x.view(np.uint16), y.view(np.uint16)
    codes, scale = orc.tdc_refresh_fp8(xb, yb)
    d = y.astype(np.float32) - x.astype(np.float32)
    a = np.max(np.abs(d), axis=1)
    assert np.all(a > 0)
    ref = (d * (np.float32(448.0) / a)[:, None]).astype(np.float32).astype(ml.float8_e4m3fn)
    assert np.array_equal(codes, ref.view(np.uint8))
    dec = ref.astype(np.float32) * scale[:, None]
    err = np.abs(dec.astype(np.float64) - d.astype(np.float64))
    bound = np.maximum(2.0 ** -4 * np.abs(d), 2.0 ** -10 * scale[:, None]) * (1 + 2.0 ** -20) + 1e-44
    assert np.all(err <= bound)
    out = (x.astype(np.float32) + dec).astype(ml.bfloat16)
    assert np.array_equal(orc.tdc_reuse_fp8(xb, codes, scale), out.view(np.uint16))


def test_tdc_fp8_residual_overflow_row(orc):
    """A row whose largest residual is so small that 448 / a overflows FP32 codes every nonzero
    residual as +-448 (0x7e, 0xfe) and zeros as 0; s = a / 448 stays a positive subnormal."""
    x = np.zeros((1, 16), dtype=np.uint16)
    y = np.zeros((1, 16), dtype=np.uint16)
    y[0, 3] = 0x0001   # +2^-133 (the smallest bf16 subnormal)
    y[0, 9] = 0x8001   # -2^-133
    codes, scale = orc.tdc_refresh_fp8(x, y)
    assert 0.0 < scale[0] < 2.0 ** -133
    want = np.zeros(16, dtype=np.uint8)
    want[3], want[9] = 0x7E, 0xFE
    assert np.array_equal(codes[0], want)


def test_tdc_schedule_dyadic(orc):
    """delta = 1/32, threshold 1/8: after the two warm-up outputs, four skips then a compute."""
    s = orc.State()
    log = []
    for t in range(14):
        skip = orc.tdc_step(s, 0.125)
        log.append(skip)
        if not skip:
            orc.tdc_record(s, delta=(1 / 32 if s.n_out >= 1 else None), d=0.05)
    assert log == [0, 0, 1, 1, 1, 1, 0, 1, 1, 1, 1, 0, 1, 1]


def test_precision_rule_and_restart(orc):
    s = orc.State()
    orc.tdc_step(s, 0.1)
    assert orc.select_precision(s, 1.0, 0.0, 0.1) == orc.INT8  # no previous difference
    orc.tdc_record(s, None, d=0.05)
    orc.tdc_step(s, 0.1)
    assert orc.select_precision(s, 1.0, 0.0, 0.1) == orc.NVFP4  # 0.05 <= 0.1
    assert orc.select_precision(s, 2.0, 0.0, 0.1) == orc.NVFP4  # 0.1 == tau: tie -> NVFP4
    assert orc.select_precision(s, 2.0, 0.0625, 0.1) == orc.INT8
    assert orc.select_precision(s, -1.0, 0.0, -0.06) == orc.INT8  # sign of a matters
    assert orc.select_precision(s, 1.0, 0.0, 0.1, force=orc.BF16) == orc.BF16
    orc.tdc_record(s, 1 / 64, d=0.05)
    orc.tdc_step(s, 0.125)  # acc = 1/64 -> skip
    assert s.skip == 1 and orc.select_precision(s, 1.0, 0.0, 0.1) == orc.SKIP
    for _ in range(7):  # acc = 8/64 = threshold: still skipped
        orc.tdc_step(s, 0.125)
        assert s.skip == 1
    orc.tdc_step(s, 0.125)  # acc = 9/64 > 1/8
    assert s.skip == 0 and s.have_d == 0  # accumulator exceeded: restart
    assert orc.select_precision(s, 1.0, 0.0, 0.1) == orc.INT8


def test_pdr(orc):
    assert orc.apply_pdr(orc.NVFP4, 64.0, 64.0) == orc.NVFP4  # ratio == rho: no fallback
    assert orc.apply_pdr(orc.NVFP4, 64.0000001, 64.0) == orc.BF16
    assert orc.apply_pdr(orc.INT8, math.inf, 64.0) == orc.BF16
    assert orc.apply_pdr(orc.INT8, 1e9, 64.0, force=orc.INT8) == orc.INT8
    assert orc.apply_pdr(orc.SKIP, 1e9, 64.0) == orc.SKIP
