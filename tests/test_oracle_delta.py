"""Pins of the oracle's delta-token split (DeltaQuant page, abstract; readings R-DQ-* in
oracle/sixbit_oracle.c) against what the definitions and independent libraries fix: a hand-worked
cube map, exact means of cubes of identical tokens, the pairwise order of the token sum, FP8 core
codes against ml_dtypes' E4M3 cast, delta tokens against ml_dtypes' bf16 rounding, and the core
product against numpy on integer-valued cores."""
import numpy as np
import pytest

import oracle

GRID = (2, 3, 3, 3, 2, 2, 2)  # 2 text tokens, a 3 x 3 x 3 grid, 2 x 2 x 2 cubes


def test_cube_map_hand_worked():
    # text tokens 0, 1; grid token 2 + (f * 3 + h) * 3 + w; cubes in (f, h, w) order of first position
    expect = [[0], [1], [2, 3, 5, 6, 11, 12, 14, 15], [4, 7, 13, 16], [8, 9, 17, 18], [10, 19],
              [20, 21, 23, 24], [22, 25], [26, 27], [28]]
    assert oracle.cube_count(29, GRID) == len(expect)
    assert [oracle.cube_tokens(k, GRID) for k in range(len(expect))] == expect
    for k, toks in enumerate(expect):
        assert all(oracle.cube_of_token(t, GRID) == k for t in toks)
    assert oracle.cube_count(30, GRID) == -1  # the grid must cover the tokens exactly


def _bf16(a):
    return oracle.f32_to_bf16(np.asarray(a, dtype=np.float32))


def test_identical_tokens_have_exact_mean_and_zero_delta():
    """A cube of identical tokens: the pairwise sum is an exact multiple and the division exact,
    so the mean is the token; when the token is E4M3-exact after the per-core scale (here every
    channel a small power of two times the max) the core decodes to it and every delta is 0."""
    K = 32
    row = np.array([2.0 ** -(i % 5) * (1 if i % 3 else -1) for i in range(K)], dtype=np.float32)
    row[7] = 4.0  # the max |mean|: scale 4 / 448, and every other channel a power of two of it
    X = np.tile(row, (29, 1))
    codes, scale, dec, delta = oracle.delta_split(_bf16(X), GRID)
    assert np.array_equal(dec, np.tile(row, (len(scale), 1)))
    assert (delta == 0).all()
    assert (codes[:, 7] == 0x7E).all() and np.all(scale == np.float32(4.0) / np.float32(448.0))


def test_token_sum_is_pairwise_in_token_order():
    """A 4-token cube holding 2^24, 1, 1, 1 in one channel: the pairwise sum is 2^24 + 2 (a
    left-to-right sum gives 2^24), so the mean, and with it the core's scale max|mean| / 448,
    is 4194304.5 / 448, not 4194304 / 448."""
    grid = (0, 1, 2, 2, 1, 2, 2)  # one frame of 2 x 2 tokens, one cube of 4
    K = 16
    X = np.zeros((4, K), dtype=np.float32)
    X[:, 0] = [2.0 ** 24, 1.0, 1.0, 1.0]
    codes, scale, dec, delta = oracle.delta_split(_bf16(X), grid)
    a = np.float32(4194304.5)
    assert scale[0] == a / np.float32(448.0)
    assert codes[0, 0] == 0x7E and dec[0, 0] == np.float32(448.0) * scale[0]
    seq = np.float32(2.0 ** 24) / np.float32(4.0)
    assert scale[0] != seq / np.float32(448.0)


def test_core_codes_match_ml_dtypes_and_deltas_round_like_ml_dtypes():
    ml = pytest.importorskip("ml_dtypes")
    rng = np.random.default_rng(5)
    grid = (3, 4, 5, 6, 2, 2, 2)
    M, K = 3 + 4 * 5 * 6, 64
    X = (rng.standard_normal((M, K)) * np.exp(rng.uniform(-6, 6, (M, 1)))).astype(np.float32)
    Xb = _bf16(X)
    codes, scale, dec, delta = oracle.delta_split(Xb, grid)
    xf = oracle.bf16_to_f32(Xb)
    for k in range(len(scale)):
        toks = oracle.cube_tokens(k, grid)
        # the mean, recomputed in FP64 from the cube's values, is within a few FP32 ulps of the core
        m64 = xf[toks].astype(np.float64).mean(axis=0)
        a = np.float32(np.max(np.abs(m64)))
        assert abs(float(scale[k]) - float(a) / 448.0) <= 4e-7 * float(a) / 448.0 + 1e-45
        # codes: the E4M3 cast of mean * (448 / a), as ml_dtypes rounds it, for the oracle's mean
        mean32 = np.array([oracle.pairwise_f32(xf[toks, c]) / np.float32(len(toks)) for c in range(K)],
                          dtype=np.float32)
        am = np.max(np.abs(mean32))
        ref = (mean32 * (np.float32(448.0) / am)).astype(np.float32).astype(ml.float8_e4m3fn)
        assert np.array_equal(codes[k], ref.view(np.uint8))
        assert np.array_equal(dec[k], ref.astype(np.float32) * (am / np.float32(448.0)))
        for t in toks:  # the delta: FP32 difference rounded to bf16 by ml_dtypes
            d = (xf[t] - dec[k]).astype(np.float32).astype(ml.bfloat16).view(np.uint16)
            assert np.array_equal(delta[t], d)


def test_core_product_matches_numpy_on_integer_cores():
    """orc_delta_linear adds the core product, the bias and the delta GEMM's rows: with
    integer-valued cores, weights and rows the FP64 result is exact and numpy agrees."""
    rng = np.random.default_rng(9)
    T, F, H, W, ct, ch, cw = GRID
    M, K, N = 29, 32, 24
    n = oracle.cube_count(M, GRID)
    dec = rng.integers(-4, 5, (n, K)).astype(np.float32)
    Wt = _bf16(rng.integers(-3, 4, (N, K)).astype(np.float32))
    bias = _bf16(rng.integers(-2, 3, N).astype(np.float32))
    Yd = rng.integers(-50, 51, (M, N)).astype(np.float64)
    Y = oracle.delta_linear(Yd, dec, Wt, bias, M, GRID)
    cube = np.array([oracle.cube_of_token(t, GRID) for t in range(M)])
    ref = Yd + dec[cube].astype(np.float64) @ oracle.bf16_to_f32(Wt).astype(np.float64).T \
        + oracle.bf16_to_f32(bias).astype(np.float64)
    assert np.array_equal(Y, ref)
