"""CPU oracle of the 6Bit-Diffusion hot path (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
this package. It wraps ``sixbit_oracle.c`` (plain C loops, FP32 round-to-nearest-even where the
GPU path decides codes, FP64 elsewhere) through ctypes and numpy. It shares no code with the CUDA
library in ``video_diffusion_mixed_b200``.

Every function cites the passage of the source pages it follows; see the header of
``sixbit_oracle.c`` for the readings (R-*) that fill what the pages leave open.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sixbit_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

NVFP4, INT8, BF16, SKIP = 0, 1, 2, 3

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FP contraction, OpenMP over rows)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp", "-fPIC", "-shared",
               "-std=c11", "-Wall", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _P(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        vp, i64, i32, f32, f64 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_double
        sig = {
            "orc_f32_to_bf16": (ctypes.c_uint16, [f32]),
            "orc_hadamard_entry": (i32, [i32, i32]),
            "orc_fwht_f32": (None, [vp, i32]),
            "orc_rotate_rows": (None, [vp, i64, i64, i32, vp]),
            "orc_pairwise_f32": (f32, [vp, i64]),
            "orc_pairwise_f64": (f64, [vp, i64]),
            "orc_prepass": (None, [vp, vp, i64, i64, i32, vp, vp, vp, vp]),
            "orc_quant_int8": (None, [vp, i64, i64, vp, vp, vp]),
            "orc_chunk_stats": (None, [vp, i64, i64, i32, vp]),
            "orc_cube_count": (i64, [i64, i64, i64, i64, i64, i64, i64, i64]),
            "orc_cube_of_token": (i64, [i64, i64, i64, i64, i64, i64, i64, i64]),
            "orc_cube_tokens": (i64, [i64, i64, i64, i64, i64, i64, i64, i64, vp]),
            "orc_delta_split": (None, [vp, i64, i64, i64, i64, i64, i64, i64, i64, i64, vp, vp, vp, vp]),
            "orc_delta_linear": (None, [vp, vp, vp, vp, i64, i64, i64, i64, i64, i64, i64, i64, i64, i64, i32,
                                        vp, i64, vp]),
            "orc_e2m1_decode": (f32, [ctypes.c_uint8]),
            "orc_e2m1_encode": (ctypes.c_uint8, [f32]),
            "orc_e4m3_decode": (f32, [ctypes.c_uint8]),
            "orc_e4m3_encode": (ctypes.c_uint8, [f32]),
            "orc_sf_tiled_offset": (i64, [i64, i64, i64]),
            "orc_sf_tiled_bytes": (i64, [i64, i64]),
            "orc_nvfp4_tensor_scale": (f32, [f32]),
            "orc_quant_nvfp4": (None, [vp, i64, i64, f32, vp, vp, vp, vp]),
            "orc_gelu_tanh": (f64, [f64]),
            "orc_gemm_nvfp4": (None, [vp, vp, f32, vp, vp, f32, vp, i64, i64, i64, i32, i32, vp, i64, vp, vp]),
            "orc_gemm_int8": (None, [vp, vp, vp, vp, vp, i64, i64, i64, i32, i32, vp, i64, vp, vp]),
            "orc_gemm_bf16": (None, [vp, vp, vp, i64, i64, i64, i32, vp, i64, vp]),
            "orc_tdc_delta": (f64, [vp, vp, i64, i64, vp]),
            "orc_tdc_refresh": (None, [vp, vp, i64, vp]),
            "orc_tdc_reuse": (None, [vp, vp, i64, vp]),
            "orc_tdc_refresh_fp8": (None, [vp, vp, i64, i64, vp, vp]),
            "orc_tdc_reuse_fp8": (None, [vp, vp, vp, i64, i64, vp]),
            "orc_state_init": (None, [vp]),
            "orc_tdc_step": (None, [vp, f64]),
            "orc_select_precision": (i32, [vp, f64, f64, f64, i32]),
            "orc_apply_pdr": (i32, [i32, f64, f64, i32]),
            "orc_tdc_record": (None, [vp, i32, f64, i32, f64]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _u16(a):
    """View a bf16 tensor/array as contiguous uint16 numpy."""
    try:
        import torch
        if isinstance(a, torch.Tensor):
            return a.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
    except ImportError:  # pragma: no cover
        pass
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16
    return a


# ---------------------------------------------------------------------------------------------
# Number formats
# ---------------------------------------------------------------------------------------------

def f32_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even FP32 -> bf16 bit patterns (comparison helper)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    nan = np.isnan(x)
    r[nan] = ((u[nan] >> 16) | 0x40).astype(np.uint16)
    return r


def bf16_to_f32(h: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(h, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def e2m1_decode(c: int) -> float:
    return lib().orc_e2m1_decode(c)


def e2m1_encode(v: float) -> int:
    return lib().orc_e2m1_encode(v)


def e4m3_decode(c: int) -> float:
    return lib().orc_e4m3_decode(c)


def e4m3_encode(v: float) -> int:
    return lib().orc_e4m3_encode(v)


E2M1_TABLE = None
E4M3_TABLE = None


def e2m1_table() -> np.ndarray:
    global E2M1_TABLE
    if E2M1_TABLE is None:
        E2M1_TABLE = np.array([e2m1_decode(c) for c in range(16)], dtype=np.float64)
    return E2M1_TABLE


def e4m3_table() -> np.ndarray:
    global E4M3_TABLE
    if E4M3_TABLE is None:
        E4M3_TABLE = np.array([e4m3_decode(c) for c in range(256)], dtype=np.float64)
    return E4M3_TABLE


# ---------------------------------------------------------------------------------------------
# Hadamard and reductions
# ---------------------------------------------------------------------------------------------

def hadamard_entry(i: int, j: int) -> int:
    return lib().orc_hadamard_entry(i, j)


def fwht(v: np.ndarray, B: int) -> np.ndarray:
    """Blockwise unnormalised FWHT (R-H) of a float32 vector whose length is a multiple of B."""
    v = np.array(v, dtype=np.float32, copy=True)
    for j in range(0, v.size, B):
        blk = np.ascontiguousarray(v[j:j + B])
        lib().orc_fwht_f32(_P(blk), B)
        v[j:j + B] = blk
    return v


def rotate_rows(x_bf16, B: int) -> np.ndarray:
    x = _u16(x_bf16)
    M, K = x.shape
    y = np.empty((M, K), dtype=np.float32)
    lib().orc_rotate_rows(_P(x), M, K, B, _P(y))
    return y


def pairwise_f32(t: np.ndarray) -> np.float32:
    t = np.ascontiguousarray(t, dtype=np.float32)
    return np.float32(lib().orc_pairwise_f32(_P(t), t.size))


def pairwise_f64(t: np.ndarray) -> float:
    t = np.ascontiguousarray(t, dtype=np.float64)
    return lib().orc_pairwise_f64(_P(t), t.size)


# ---------------------------------------------------------------------------------------------
# Pre-pass, quantization
# ---------------------------------------------------------------------------------------------

STAT_NAMES = ("sum_abs", "sum_d2", "sum_ref2", "max_abs", "amax_rot", "ratio", "d", "numel")


def prepass(x_bf16, xref_bf16=None, B: int = 128, want_rot: bool = True):
    """Pre-pass statistics ([VU] sections 一 and 三): rotated rows, per-token rotated amax,
    per-row FP32 partials and the FP64 statistics record (see ``STAT_NAMES``)."""
    x = _u16(x_bf16)
    M, K = x.shape
    r = _u16(xref_bf16) if xref_bf16 is not None else None
    y = np.empty((M, K), dtype=np.float32) if want_rot else None
    amax = np.empty(M, dtype=np.float32)
    part = np.empty((M, 3), dtype=np.float32)
    out = np.zeros(8, dtype=np.float64)
    lib().orc_prepass(_P(x), _P(r), M, K, B, _P(y), _P(amax), _P(part), _P(out))
    return {"y": y, "row_amax": amax, "row_part": part, **{n: float(out[i]) for i, n in enumerate(STAT_NAMES)}}


def chunk_stats(x_bf16, B: int = 128) -> np.ndarray:
    """Per aligned 128-channel chunk of every row: [M, K/128, 3] float32 of (max |H_B x|, canonical
    pairwise sum |x|, max |x|) -- the records the first FFN layer's epilogue hands to the second
    layer's pre-pass."""
    x = _u16(x_bf16)
    M, K = x.shape
    out = np.empty((M, K // 128, 3), dtype=np.float32)
    lib().orc_chunk_stats(_P(x), M, K, B, _P(out))
    return out


def quant_int8(y: np.ndarray, row_amax: np.ndarray):
    """R-INT8 per-token symmetric quantization of rotated rows ([VU] section 一: INT8)."""
    y = np.ascontiguousarray(y, dtype=np.float32)
    M, K = y.shape
    a = np.ascontiguousarray(row_amax, dtype=np.float32)
    q = np.empty((M, K), dtype=np.int8)
    s = np.empty(M, dtype=np.float32)
    lib().orc_quant_int8(_P(y), M, K, _P(a), _P(q), _P(s))
    return q, s


def sf_tiled_offset(m: int, g: int, K: int) -> int:
    return lib().orc_sf_tiled_offset(m, g, K)


def sf_tiled_bytes(M: int, K: int) -> int:
    return lib().orc_sf_tiled_bytes(M, K)


def quant_nvfp4(y: np.ndarray, A: float | None = None):
    """R-FP4 NVFP4 encode of rotated rows ([VU] section 一: NVFP4). Returns packed codes
    [M][K/2], logical scales [M][K/16], tiled scales (tensor-core layout) and the tensor scale."""
    y = np.ascontiguousarray(y, dtype=np.float32)
    M, K = y.shape
    if A is None:
        A = float(np.max(np.abs(y))) if y.size else 0.0
    codes = np.empty((M, K // 2), dtype=np.uint8)
    sfl = np.empty((M, K // 16), dtype=np.uint8)
    sft = np.empty(sf_tiled_bytes(M, K), dtype=np.uint8)
    sg = ctypes.c_float(0.0)
    lib().orc_quant_nvfp4(_P(y), M, K, ctypes.c_float(A), _P(codes), _P(sfl), _P(sft), ctypes.byref(sg))
    return codes, sfl, sft, np.float32(sg.value)


def nvfp4_dequant(codes: np.ndarray, sfl: np.ndarray, s_g: float | None = None) -> np.ndarray:
    """Decode packed NVFP4 codes and logical scales to FP64 (times s_g when given)."""
    M, Kh = codes.shape
    K = Kh * 2
    t2 = e2m1_table()
    t4 = e4m3_table()
    lo = codes & 15
    hi = codes >> 4
    c = np.empty((M, K), dtype=np.uint8)
    c[:, 0::2] = lo
    c[:, 1::2] = hi
    v = t2[c] * np.repeat(t4[sfl], 16, axis=1)
    return v * float(s_g) if s_g is not None else v


# ---------------------------------------------------------------------------------------------
# GEMMs (FP64)
# ---------------------------------------------------------------------------------------------

def _rows(M, rows):
    if rows is None:
        rows = np.arange(M, dtype=np.int64)
    return np.ascontiguousarray(rows, dtype=np.int64)


def gemm_nvfp4(xc, xsf, sgx, wc, wsf, sgw, bias, K: int, B: int, gelu=False, rows=None, want_acc=False):
    M, N = xc.shape[0], wc.shape[0]
    rows = _rows(M, rows)
    Y = np.empty((rows.size, N), dtype=np.float64)
    acc = np.empty((rows.size, N), dtype=np.float64) if want_acc else None
    b = _u16(bias) if bias is not None else None
    lib().orc_gemm_nvfp4(_P(np.ascontiguousarray(xc)), _P(np.ascontiguousarray(xsf)), ctypes.c_float(sgx),
                         _P(np.ascontiguousarray(wc)), _P(np.ascontiguousarray(wsf)), ctypes.c_float(sgw),
                         _P(b), M, N, K, B, int(gelu), _P(rows), rows.size, _P(Y), _P(acc))
    return (Y, acc) if want_acc else Y


def gemm_int8(qx, sx, qw, sw, bias, B: int, gelu=False, rows=None, want_acc=False):
    M, K = qx.shape
    N = qw.shape[0]
    rows = _rows(M, rows)
    Y = np.empty((rows.size, N), dtype=np.float64)
    acc = np.empty((rows.size, N), dtype=np.int64) if want_acc else None
    b = _u16(bias) if bias is not None else None
    lib().orc_gemm_int8(_P(np.ascontiguousarray(qx)), _P(np.ascontiguousarray(sx, dtype=np.float32)),
                        _P(np.ascontiguousarray(qw)), _P(np.ascontiguousarray(sw, dtype=np.float32)),
                        _P(b), M, N, K, B, int(gelu), _P(rows), rows.size, _P(Y), _P(acc))
    return (Y, acc) if want_acc else Y


def gemm_bf16(x_bf16, w_bf16, bias, gelu=False, rows=None):
    x = _u16(x_bf16)
    w = _u16(w_bf16)
    M, K = x.shape
    N = w.shape[0]
    rows = _rows(M, rows)
    Y = np.empty((rows.size, N), dtype=np.float64)
    b = _u16(bias) if bias is not None else None
    lib().orc_gemm_bf16(_P(x), _P(w), _P(b), M, N, K, int(gelu), _P(rows), rows.size, _P(Y))
    return Y


def gelu_tanh(v: float) -> float:
    return lib().orc_gelu_tanh(v)


# ---------------------------------------------------------------------------------------------
# Weights (offline): rotate rows along K, NVFP4 and INT8 copies ([VU] section 四: W4A6)
# ---------------------------------------------------------------------------------------------

def prepare_weight(w_bf16, B: int = 128):
    st = prepass(w_bf16, None, B)
    y = st["y"]
    q8, s8 = quant_int8(y, st["row_amax"])
    c4, sfl, sft, sg = quant_nvfp4(y, st["amax_rot"])
    return {"y": y, "q8": q8, "s8": s8, "c4": c4, "sf4": sfl, "sf4_tiled": sft, "sg4": sg,
            "amax_rot": st["amax_rot"]}


# ---------------------------------------------------------------------------------------------
# Temporal Delta Cache and decisions ([VU] sections 二 and 三; [GS] sections 3 and 4)
# ---------------------------------------------------------------------------------------------

def tdc_delta(ynew_bf16, ylast_bf16):
    a = _u16(ynew_bf16)
    b = _u16(ylast_bf16)
    M, C = a.shape
    out = np.zeros(2, dtype=np.float64)
    d = lib().orc_tdc_delta(_P(a), _P(b), M, C, _P(out))
    return d, float(out[0]), float(out[1])


def tdc_refresh(x_bf16, y_bf16):
    """R-REUSE: the residual kept at a computed step, D = bf16(y - x) (bf16 bit patterns)."""
    x = _u16(x_bf16)
    y = _u16(y_bf16)
    assert x.shape == y.shape
    d = np.empty_like(x)
    lib().orc_tdc_refresh(_P(x), _P(y), x.size, _P(d))
    return d


def tdc_reuse(x_bf16, d_bf16):
    """R-REUSE: the output of a skipped step, y = bf16(x + D) (bf16 bit patterns)."""
    x = _u16(x_bf16)
    d = _u16(d_bf16)
    assert x.shape == d.shape
    y = np.empty_like(x)
    lib().orc_tdc_reuse(_P(x), _P(d), x.size, _P(y))
    return y


def tdc_refresh_fp8(x_bf16, y_bf16):
    """R-REUSE-FP8: the residual kept in FP8, E4M3 codes [M][C] and one FP32 scale per row."""
    x = _u16(x_bf16)
    y = _u16(y_bf16)
    assert x.shape == y.shape and x.ndim == 2
    M, C = x.shape
    codes = np.zeros((M, C), dtype=np.uint8)
    scale = np.zeros(M, dtype=np.float32)
    lib().orc_tdc_refresh_fp8(_P(x), _P(y), M, C, _P(codes), _P(scale))
    return codes, scale


def tdc_reuse_fp8(x_bf16, codes, scale):
    """R-REUSE-FP8: the output of a skipped step, y = bf16(x + E4M3(code) * s) (bf16 bits)."""
    x = _u16(x_bf16)
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scale = np.ascontiguousarray(scale, dtype=np.float32)
    M, C = x.shape
    assert codes.shape == (M, C) and scale.shape == (M,)
    y = np.empty_like(x)
    lib().orc_tdc_reuse_fp8(_P(x), _P(codes), _P(scale), M, C, _P(y))
    return y


class State(ctypes.Structure):
    _fields_ = [("prev_d", ctypes.c_double), ("acc", ctypes.c_double), ("delta", ctypes.c_double),
                ("have_d", ctypes.c_int32), ("n_out", ctypes.c_int32),
                ("last_skipped", ctypes.c_int32), ("skip", ctypes.c_int32)]

    def __init__(self):
        super().__init__()
        lib().orc_state_init(ctypes.byref(self))

    def as_dict(self):
        return {n: getattr(self, n) for n, _ in self._fields_}


def tdc_step(s: State, thr: float) -> int:
    lib().orc_tdc_step(ctypes.byref(s), thr)
    return s.skip


def select_precision(s: State, a: float, b: float, tau: float, force: int = -1) -> int:
    return lib().orc_select_precision(ctypes.byref(s), a, b, tau, force)


def apply_pdr(prec: int, ratio: float, rho: float, force: int = -1) -> int:
    return lib().orc_apply_pdr(prec, ratio, rho, force)


def tdc_record(s: State, delta=None, d=None) -> None:
    lib().orc_tdc_record(ctypes.byref(s), int(delta is not None), float(delta or 0.0),
                         int(d is not None), float(d or 0.0))


# ---------------------------------------------------------------------------------------------
# Delta tokens (the DeltaQuant page, abstract; readings R-DQ-* in sixbit_oracle.c)
# ---------------------------------------------------------------------------------------------

def cube_count(M: int, grid) -> int:
    """Number of cubes of M tokens; grid = (T, F, H, W, ct, ch, cw); -1 if M != T + F H W."""
    return int(lib().orc_cube_count(M, *grid))


def cube_of_token(t: int, grid) -> int:
    return int(lib().orc_cube_of_token(t, *grid))


def cube_tokens(k: int, grid) -> list:
    T, F, H, W, ct, ch, cw = grid
    buf = np.zeros(ct * ch * cw, dtype=np.int64)
    n = lib().orc_cube_tokens(k, T, F, H, W, ct, ch, cw, _P(buf))
    return buf[:n].tolist()


def delta_split(x_bf16, grid):
    """R-DQ-MEAN / FP8 / DELTA: core codes [ncube][K] (E4M3), scales [ncube], dequantized cores
    [ncube][K] FP32 and the delta tokens [M][K] (bf16 bits)."""
    x = _u16(x_bf16)
    M, K = x.shape
    n = cube_count(M, grid)
    assert n > 0, "grid does not match the token count"
    codes = np.zeros((n, K), dtype=np.uint8)
    scale = np.zeros(n, dtype=np.float32)
    dec = np.zeros((n, K), dtype=np.float32)
    delta = np.zeros((M, K), dtype=np.uint16)
    lib().orc_delta_split(_P(x), M, K, *grid, _P(codes), _P(scale), _P(dec), _P(delta))
    return codes, scale, dec, delta


def delta_linear(Yd, dec, w_bf16, bias, M, grid, gelu=False, rows=None):
    """R-DQ-GEMM: the delta GEMM's rows Yd (FP64, no bias) plus the products of the bf16-rounded
    cores, the bias and the optional GELU."""
    w = _u16(w_bf16)
    N, K = w.shape
    rows = _rows(M, rows)
    Yd = np.ascontiguousarray(Yd, dtype=np.float64)
    Y = np.empty((rows.size, N), dtype=np.float64)
    b = _u16(bias) if bias is not None else None
    lib().orc_delta_linear(_P(Yd), _P(np.ascontiguousarray(dec, dtype=np.float32)), _P(w), _P(b), M, N, K,
                           *grid, int(gelu), _P(rows), rows.size, _P(Y))
    return Y
