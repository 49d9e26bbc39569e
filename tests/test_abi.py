"""The C-ABI library loads, exports every symbol include/sixbit.h declares, and validates
arguments on the host (no GPU needed: every case below fails before any CUDA call)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sixbit.h")


@pytest.fixture(scope="module")
def sb():
    from video_diffusion_mixed_b200 import build
    build.build()
    from video_diffusion_mixed_b200 import sixbit
    sixbit.lib()
    return sixbit


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(sb_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_expected_entry_points():
    names = declared_functions()
    for n in ("sb_prepass", "sb_linear", "sb_tdc_step", "sb_tdc_record", "sb_select_precision",
              "sb_prepare_weight", "sb_check"):
        assert n in names


def test_every_declared_symbol_is_exported(sb):
    L = sb.lib()
    for name in declared_functions():
        assert hasattr(L, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", sb.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (sb_\w+)", out))
    assert set(declared_functions()) <= exported
    assert set(sb.EXPORTED) == set(declared_functions())


def test_host_only_calls(sb):
    L = sb.lib()
    assert L.sb_version().decode().startswith("sixbit")
    n = ctypes.c_size_t(0)
    assert L.sb_workspace_size(17776, 3072, ctypes.byref(n)) == sb.SB_OK
    assert n.value >= 256 + 48 * 556 and n.value % 256 == 0
    assert L.sb_fp4_sf_bytes(17776, 3072) == 17792 * 192
    assert L.sb_fp4_sf_bytes(1, 64) == 128 * 4
    assert L.sb_workspace_size(1, 1, None) == sb.SB_EINVAL


def _fake(addr):
    return ctypes.c_void_p(addr)


def test_tdc_reuse_validation_without_gpu(sb):
    L = sb.lib()
    ok = (_fake(0x1000), _fake(0x2000), _fake(0x3000))
    assert L.sb_tdc_refresh(*ok, 4, 64, None, None) == sb.SB_EINVAL
    assert L.sb_tdc_reuse(_fake(0x1008), _fake(0x2000), _fake(0x3000), 4, 64, _fake(0x4000), None) == sb.SB_EALIGN
    assert L.sb_tdc_reuse(*ok, 4, 60, _fake(0x4000), None) == sb.SB_EUNSUPPORTED
    assert L.sb_tdc_refresh(*ok, 0, 64, _fake(0x4000), None) == sb.SB_ESHAPE


def test_tdc_fp8_validation_without_gpu(sb):
    L = sb.lib()
    x, y, q, s, st = _fake(0x1000), _fake(0x2000), _fake(0x3000), _fake(0x4000), _fake(0x5000)
    assert L.sb_tdc_refresh_fp8(None, y, q, s, 4, 64, st, None) == sb.SB_EINVAL
    assert L.sb_tdc_refresh_fp8(x, y, q, None, 4, 64, st, None) == sb.SB_EINVAL
    assert L.sb_tdc_refresh_fp8(x, y, _fake(0x3008), s, 4, 64, st, None) == sb.SB_EALIGN
    assert L.sb_tdc_reuse_fp8(x, q, _fake(0x4002), y, 4, 64, st, None) == sb.SB_EALIGN
    assert L.sb_tdc_reuse_fp8(x, q, s, y, 4, 72, st, None) == sb.SB_EUNSUPPORTED
    assert L.sb_tdc_reuse_fp8(x, q, s, y, 0, 64, st, None) == sb.SB_ESHAPE


def test_module_record_validation_without_gpu(sb):
    L = sb.lib()
    y, x, c, s, st, ws = (_fake(a) for a in (0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 0x6000))
    assert L.sb_module_record(None, x, c, 4, 64, None, 1, s, st, ws, None) == sb.SB_EINVAL
    assert L.sb_module_record(y, x, c, 4, 64, None, 1, s, None, ws, None) == sb.SB_EINVAL
    assert L.sb_module_record(y, _fake(0x2008), c, 4, 64, None, 1, s, st, ws, None) == sb.SB_EALIGN
    assert L.sb_module_record(y, x, c, 4, 64, _fake(0x7002), 1, s, st, ws, None) == sb.SB_EALIGN
    assert L.sb_module_record(y, x, c, 0, 64, None, 1, s, st, ws, None) == sb.SB_ESHAPE
    assert L.sb_module_record(y, x, c, 4, 96, None, 1, s, st, ws, None) == sb.SB_EUNSUPPORTED
    assert L.sb_module_record(y, x, c, 4, 16448, None, 1, s, st, ws, None) == sb.SB_EUNSUPPORTED


def test_workspace_holds_two_slot_arrays(sb):
    n = ctypes.c_size_t(0)
    assert sb.lib().sb_workspace_size(17776, 3072, ctypes.byref(n)) == sb.SB_OK
    assert n.value >= 256 + 2 * 48 * ((17776 + 15) // 16)


def test_wait_flag_validation_without_gpu(sb):
    L = sb.lib()
    assert L.sb_wait_flag(None, 1, 1000, _fake(0x100), None) == sb.SB_EINVAL
    assert L.sb_wait_flag(_fake(0x1002), 1, 1000, _fake(0x100), None) == sb.SB_EALIGN
    assert L.sb_wait_flag(_fake(0x1000), 1, 0, _fake(0x100), None) == sb.SB_EINVAL
    assert L.sb_wait_flag(_fake(0x1000), 1, 10_000_000_001, _fake(0x100), None) == sb.SB_EINVAL
    assert L.sb_drill_gemm_stall(-1, 1_000_000) == sb.SB_EINVAL
    assert L.sb_drill_gemm_stall(0, 99_999) == sb.SB_EINVAL
    assert L.sb_drill_gemm_stall(0, 10_000_000_001) == sb.SB_EINVAL
    assert "limit_ns" in L.sb_last_error().decode()


def test_argument_validation_without_gpu(sb):
    L = sb.lib()
    cfg = sb.config()
    a4 = sb.Fp4(0x1000, 0x2000, 0x3000, 64, 256)
    a8 = sb.I8(0x4000, 0x5000, 64, 256)
    s = None
    # null X
    assert L.sb_prepass(None, None, 64, 256, ctypes.byref(cfg), 0, _fake(0x100), ctypes.byref(a4),
                        ctypes.byref(a8), _fake(0x200), _fake(0x300), s) == sb.SB_EINVAL
    # misaligned X
    assert L.sb_prepass(_fake(0x1008), None, 64, 256, ctypes.byref(cfg), 0, _fake(0x100), ctypes.byref(a4),
                        ctypes.byref(a8), _fake(0x200), _fake(0x300), s) == sb.SB_EALIGN
    assert "aligned" in L.sb_last_error().decode()
    # K not a multiple of the block / of 64, bad block
    bad = sb.config(block=96)
    assert L.sb_prepass(_fake(0x1000), None, 64, 256, ctypes.byref(bad), 0, _fake(0x100), ctypes.byref(a4),
                        ctypes.byref(a8), _fake(0x200), _fake(0x300), s) == sb.SB_EUNSUPPORTED
    assert L.sb_prepass(_fake(0x1000), None, 64, 200, ctypes.byref(cfg), 0, _fake(0x100), ctypes.byref(a4),
                        ctypes.byref(a8), _fake(0x200), _fake(0x300), s) == sb.SB_EUNSUPPORTED
    assert L.sb_prepass(_fake(0x1000), None, 0, 256, ctypes.byref(cfg), 0, _fake(0x100), ctypes.byref(a4),
                        ctypes.byref(a8), _fake(0x200), _fake(0x300), s) == sb.SB_ESHAPE
    # shape mismatch between X and the a4 descriptor
    a4b = sb.Fp4(0x1000, 0x2000, 0x3000, 65, 256)
    assert L.sb_prepass(_fake(0x1000), None, 64, 256, ctypes.byref(cfg), 0, _fake(0x100), ctypes.byref(a4b),
                        ctypes.byref(a8), _fake(0x200), _fake(0x300), s) == sb.SB_ESHAPE
    # QUANT mode needs the quantized outputs
    assert L.sb_prepass(_fake(0x1000), None, 64, 256, ctypes.byref(cfg), 0, _fake(0x100), None, None,
                        _fake(0x200), _fake(0x300), s) == sb.SB_EINVAL
    # K above the supported maximum
    assert L.sb_prepass(_fake(0x1000), None, 64, 16384 + 64, ctypes.byref(cfg), 1, None, None, None,
                        _fake(0x200), _fake(0x300), s) == sb.SB_EUNSUPPORTED
    # linear: N not a multiple of 32, K not a multiple of 128
    w = sb.WeightC()
    w.N, w.K, w.block = 100, 256, 128
    assert L.sb_linear(_fake(0x1000), None, None, _fake(0x100), ctypes.byref(w), 0, 0, _fake(0x2000), 64,
                       _fake(0x300), s) == sb.SB_EUNSUPPORTED
    w.N, w.K = 128, 192
    assert L.sb_linear(_fake(0x1000), None, None, _fake(0x100), ctypes.byref(w), 0, 0, _fake(0x2000), 64,
                       _fake(0x300), s) == sb.SB_EUNSUPPORTED
    w.N, w.K = 128, 256
    assert L.sb_linear(None, None, None, _fake(0x100), ctypes.byref(w), 0, 0, _fake(0x2000), 64,
                       _fake(0x300), s) == sb.SB_EINVAL
    assert L.sb_linear(_fake(0x1000), None, None, _fake(0x100), ctypes.byref(w), 7, 0, _fake(0x2000), 64,
                       _fake(0x300), s) == sb.SB_EINVAL
    # tdc record: C not a multiple of 8
    assert L.sb_tdc_record(_fake(0x1000), _fake(0x2000), 4, 12, None, 1, _fake(0x300), _fake(0x400),
                           s) == sb.SB_EUNSUPPORTED
    # select: bad force value
    rule = sb.Rule(1.0, 0.0, 0.1)
    assert L.sb_select_precision(_fake(0x100), ctypes.byref(rule), ctypes.byref(sb.config(force_prec=5)),
                                 _fake(0x200), s) == sb.SB_EINVAL


def test_shard_validation_without_gpu(sb):
    """The token-sharding entry points check the shard rules before any launch."""
    L = sb.lib()
    cfg = sb.config()
    a8 = sb.I8(0x4000, 0x5000, 32, 256)
    assert L.sb_group_slots_bytes(17776) == 1111 * 48
    assert L.sb_group_slots_bytes(17) == 2 * 48
    assert L.sb_group_slots_bytes(0) == -1
    X, slots, ws, prec = _fake(0x1000), _fake(0x8000), _fake(0x9000), _fake(0x100)
    # row0 not on a 16-row group boundary
    assert L.sb_prepass_partial(X, None, 32, 256, 8, 64, ctypes.byref(cfg), 1, None, None, slots, ws,
                                None) == sb.SB_ESHAPE
    assert "multiple of 16" in L.sb_last_error().decode()
    # a shard that does not end the tensor must hold whole groups
    assert L.sb_prepass_partial(X, None, 20, 256, 0, 64, ctypes.byref(cfg), 1, None, None, slots, ws,
                                None) == sb.SB_ESHAPE
    # rows past the tensor
    assert L.sb_prepass_partial(X, None, 32, 256, 48, 64, ctypes.byref(cfg), 1, None, None, slots, ws,
                                None) == sb.SB_ESHAPE
    # QUANT needs prec and a8; misaligned slots
    assert L.sb_prepass_partial(X, None, 32, 256, 32, 64, ctypes.byref(cfg), 0, None, None, slots, ws,
                                None) == sb.SB_EINVAL
    assert L.sb_prepass_partial(X, None, 32, 256, 32, 64, ctypes.byref(cfg), 0, prec, ctypes.byref(a8),
                                _fake(0x8008), ws, None) == sb.SB_EALIGN
    # finish and TDC partial / finish
    assert L.sb_prepass_finish(None, 64, 256, 0, ctypes.byref(cfg), 1, None, _fake(0x200), ws, None) == sb.SB_EINVAL
    assert L.sb_prepass_finish(slots, 64, 256, 0, ctypes.byref(cfg), 0, None, _fake(0x200), ws, None) == sb.SB_EINVAL
    assert L.sb_tdc_record_partial(X, _fake(0x2000), 32, 64, 16, 40, 1, _fake(0x300), slots, ws,
                                   None) == sb.SB_ESHAPE
    assert L.sb_tdc_finish(slots, 0, 64, None, _fake(0x300), ws, None) == sb.SB_ESHAPE
    assert L.sb_nvfp4_encode(X, 64, 256, ctypes.byref(cfg), prec, _fake(0x200), None, ws, None) == sb.SB_EINVAL


def test_module_decide_validation_without_gpu(sb):
    L = sb.lib()
    cfg = sb.config()
    rules = (sb.Rule * 2)(sb.Rule(1.0, 0.0, 0.1), sb.Rule(1.0, 0.0, 0.2))
    precs = (ctypes.c_void_p * 2)(0x100, 0x200)
    r, p = ctypes.cast(rules, ctypes.c_void_p), ctypes.cast(precs, ctypes.c_void_p)
    st = _fake(0x1000)
    assert L.sb_module_decide(st, ctypes.byref(cfg), 0, r, p, None) == sb.SB_EINVAL
    assert L.sb_module_decide(st, ctypes.byref(cfg), 9, r, p, None) == sb.SB_EINVAL
    assert L.sb_module_decide(None, ctypes.byref(cfg), 2, r, p, None) == sb.SB_EINVAL
    bad = (ctypes.c_void_p * 2)(0x100, 0x202)
    assert L.sb_module_decide(st, ctypes.byref(cfg), 2, r, ctypes.cast(bad, ctypes.c_void_p), None) == sb.SB_EALIGN
    null = (ctypes.c_void_p * 2)(0x100, None)
    assert L.sb_module_decide(st, ctypes.byref(cfg), 2, r, ctypes.cast(null, ctypes.c_void_p), None) == sb.SB_EINVAL


def test_prepass_chunks_validation_without_gpu(sb):
    L = sb.lib()
    cfg = sb.config()
    a4 = sb.Fp4(0x1000, 0x2000, 0x3000, 64, 1024)
    a8 = sb.I8(0x4000, 0x5000, 64, 1024)
    X, chunks, stats, ws, prec = _fake(0x10000), _fake(0x20000), _fake(0x200), _fake(0x300), _fake(0x100)
    ok = (ctypes.byref(a4), ctypes.byref(a8), stats, ws, None)
    assert L.sb_prepass_chunks(X, None, 64, 1024, ctypes.byref(cfg), 0, prec, *ok) == sb.SB_EINVAL
    assert L.sb_prepass_chunks(X, _fake(0x20008), 64, 1024, ctypes.byref(cfg), 0, prec, *ok) == sb.SB_EALIGN
    # chunk records need whole 128-channel chunks and a Hadamard block that fits one
    big = sb.config(block=256)
    assert L.sb_prepass_chunks(X, chunks, 64, 1024, ctypes.byref(big), 0, prec, *ok) == sb.SB_EUNSUPPORTED
    assert L.sb_prepass_chunks(X, chunks, 64, 960, ctypes.byref(cfg), 0, prec, *ok) == sb.SB_EUNSUPPORTED
    assert "128" in L.sb_last_error().decode()
    assert L.sb_prepass_chunks(X, chunks, 64, 1024, ctypes.byref(cfg), 0, prec, None, None, stats, ws,
                               None) == sb.SB_EINVAL


def test_delta_token_validation_without_gpu(sb):
    L = sb.lib()
    c = sb.cubes(226, 13, 30, 45)  # the CogVideoX token layout: 226 text tokens, 13 x 30 x 45 grid
    M = 226 + 13 * 30 * 45
    assert M == 17776
    assert L.sb_cube_count(ctypes.byref(c), M) == 226 + 7 * 15 * 23
    assert L.sb_cube_count(ctypes.byref(c), M + 1) == -1  # the grid must cover the tokens exactly
    big = sb.cubes(0, 4, 4, 4, 4, 4, 4)  # 64 tokens per cube: above the 32-token limit
    assert L.sb_cube_count(ctypes.byref(big), 64) == -1
    X, codes, scale, core, delta = (_fake(0x10000), _fake(0x20000), _fake(0x30000), _fake(0x40000),
                                    _fake(0x50000))
    assert L.sb_delta_split(None, M, 3072, ctypes.byref(c), codes, scale, core, delta, None) == sb.SB_EINVAL
    assert L.sb_delta_split(_fake(0x10008), M, 3072, ctypes.byref(c), codes, scale, core, delta,
                            None) == sb.SB_EALIGN
    assert L.sb_delta_split(X, M, 3000, ctypes.byref(c), codes, scale, core, delta, None) == sb.SB_EUNSUPPORTED
    assert L.sb_delta_split(X, M - 1, 3072, ctypes.byref(c), codes, scale, core, delta, None) == sb.SB_ESHAPE
    Yd, Yc, Y = _fake(0x60000), _fake(0x70000), _fake(0x80000)
    assert L.sb_delta_combine(Yd, Yc, M, 1924, ctypes.byref(c), 0, Y, None) == sb.SB_EUNSUPPORTED
    assert L.sb_delta_combine(Yd, Yc, M, 1920, ctypes.byref(c), 5, Y, None) == sb.SB_EINVAL
    assert L.sb_delta_combine(Yd, Yc, M - 2, 1920, ctypes.byref(c), 0, Y, None) == sb.SB_ESHAPE
    # the fused form: y_core and the cubes first, then sb_linear's own checks
    p, w, ws = _fake(0x90000), sb.WeightC(), _fake(0xA0000)
    assert L.sb_delta_linear(delta, None, None, p, ctypes.byref(w), None, ctypes.byref(c), 0, 0, Y, M, ws,
                             None) == sb.SB_EINVAL
    assert L.sb_delta_linear(delta, None, None, p, ctypes.byref(w), _fake(0x70004), ctypes.byref(c), 0, 0, Y, M,
                             ws, None) == sb.SB_EALIGN
    assert L.sb_delta_linear(delta, None, None, p, ctypes.byref(w), Yc, ctypes.byref(c), 0, 2, Y, M, ws,
                             None) == sb.SB_EINVAL  # raw accumulators are not an output of this form
    assert L.sb_delta_linear(delta, None, None, p, ctypes.byref(w), Yc, ctypes.byref(c), 0, 0, Y, M - 1, ws,
                             None) == sb.SB_ESHAPE


def test_chunk_record_validation_without_gpu(sb):
    L = sb.lib()
    X, rec, Y, p, ws = _fake(0x10000), _fake(0x20000), _fake(0x30000), _fake(0x100), _fake(0x300)
    assert L.sb_chunk_records(None, 4, 256, 128, rec, None) == sb.SB_EINVAL
    assert L.sb_chunk_records(X, 4, 256, 128, _fake(0x20008), None) == sb.SB_EALIGN
    assert L.sb_chunk_records(X, 0, 256, 128, rec, None) == sb.SB_ESHAPE
    assert L.sb_chunk_records(X, 4, 320, 128, rec, None) == sb.SB_EUNSUPPORTED
    assert L.sb_chunk_records(X, 4, 256, 256, rec, None) == sb.SB_EUNSUPPORTED
    assert L.sb_chunk_records(X, 4, 256, 8, rec, None) == sb.SB_EUNSUPPORTED
    w = sb.WeightC()
    w.N, w.K, w.block = 512, 256, 128
    assert L.sb_linear_records(X, None, None, p, ctypes.byref(w), 0, Y, 4, 128, None, ws, None) == sb.SB_EINVAL
    assert L.sb_linear_records(X, None, None, p, ctypes.byref(w), 0, Y, 4, 128, _fake(0x20004), ws,
                               None) == sb.SB_EALIGN
    assert L.sb_linear_records(X, None, None, p, ctypes.byref(w), 0, Y, 4, 64, rec, ws, None) == sb.SB_EUNSUPPORTED
    w.N = 384  # records need 256-wide output tiles
    assert L.sb_linear_records(X, None, None, p, ctypes.byref(w), 0, Y, 4, 128, rec, ws, None) == sb.SB_EUNSUPPORTED
    assert "256" in L.sb_last_error().decode()


def test_fused_module_record_validation_without_gpu(sb):
    L = sb.lib()
    X, Y, x, c, rec, stats, st, ws, p = (_fake(0x10000), _fake(0x20000), _fake(0x30000), _fake(0x40000),
                                         _fake(0x50000), _fake(0x60000), _fake(0x70000), _fake(0x80000),
                                         _fake(0x100))
    w = sb.WeightC()
    w.N, w.K, w.block = 512, 256, 128
    args = lambda **o: [o.get("X", X), None, None, p, ctypes.byref(o.get("w", w)), 0, Y, o.get("M", 4),
                        o.get("x", x), o.get("c", c), 1, o.get("rec", rec), o.get("stats", stats), o.get("st", st),
                        ws, None]
    assert L.sb_linear_module_record(*args(x=None)) == sb.SB_EINVAL
    assert L.sb_linear_module_record(*args(rec=None)) == sb.SB_EINVAL
    assert L.sb_linear_module_record(*args(st=None)) == sb.SB_EINVAL
    assert L.sb_linear_module_record(*args(c=_fake(0x40008))) == sb.SB_EALIGN
    assert L.sb_linear_module_record(*args(rec=_fake(0x50004))) == sb.SB_EALIGN
    assert L.sb_linear_module_record(*args(M=0)) == sb.SB_ESHAPE
    w2 = sb.WeightC()
    w2.N, w2.K, w2.block = 384, 256, 128  # the record's chunks need 256-wide output tiles
    assert L.sb_linear_module_record(*args(w=w2)) == sb.SB_EUNSUPPORTED
    assert "256" in L.sb_last_error().decode()
