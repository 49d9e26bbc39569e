"""ctypes binding of libsixbit.so (include/sixbit.h), argument marshalling only.

Every function here forwards torch tensors' device pointers and the current CUDA stream to the
C ABI; all computation happens in the library's sm_100a kernels. Importing this module fails
loudly when the library has not been built (there is no fallback path).

Allocation helpers (``alloc_fp4``, ``alloc_i8``, ``Workspace``, ``prepare_weight``...) create the
caller-owned device buffers with torch; the library itself never allocates.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsixbit.so")

SB_OK, SB_EINVAL, SB_ESHAPE, SB_EALIGN, SB_EUNSUPPORTED, SB_ECUDA, SB_ETIMEOUT, SB_ENONFINITE = range(8)
STATUS_NAMES = ["SB_OK", "SB_EINVAL", "SB_ESHAPE", "SB_EALIGN", "SB_EUNSUPPORTED", "SB_ECUDA", "SB_ETIMEOUT",
                "SB_ENONFINITE"]
NVFP4, INT8, BF16, SKIP = 0, 1, 2, 3
PREC_NAMES = {NVFP4: "nvfp4", INT8: "int8", BF16: "bf16", SKIP: "skip"}
OUT_BF16, OUT_F32, OUT_RAW = 0, 1, 2
EPI_NONE, EPI_GELU = 0, 1
PREPASS_QUANT, PREPASS_STATS = 0, 1


class SixbitError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES[status] if 0 <= status < len(STATUS_NAMES) else status}: {msg}")
        self.status = status


class Fp4(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("sf", ctypes.c_void_p), ("gscale", ctypes.c_void_p),
                ("rows", ctypes.c_int64), ("cols", ctypes.c_int64)]


class I8(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scale", ctypes.c_void_p), ("rows", ctypes.c_int64),
                ("cols", ctypes.c_int64)]


class WeightC(ctypes.Structure):
    _fields_ = [("w_bf16", ctypes.c_void_p), ("bias_bf16", ctypes.c_void_p), ("w4", Fp4), ("w8", I8),
                ("N", ctypes.c_int64), ("K", ctypes.c_int64), ("block", ctypes.c_int32)]


class Rule(ctypes.Structure):
    _fields_ = [("a", ctypes.c_double), ("b", ctypes.c_double), ("tau", ctypes.c_double)]


class Config(ctypes.Structure):
    _fields_ = [("rho", ctypes.c_double), ("tdc_thresh", ctypes.c_double), ("block", ctypes.c_int32),
                ("force_prec", ctypes.c_int32)]


class Cubes(ctypes.Structure):
    """sb_cubes: text tokens, the frames x height x width latent grid and the cube extent."""
    _fields_ = [("text", ctypes.c_int64), ("frames", ctypes.c_int64), ("height", ctypes.c_int64),
                ("width", ctypes.c_int64), ("ct", ctypes.c_int32), ("ch", ctypes.c_int32), ("cw", ctypes.c_int32)]


STATE_BYTES = 64
STATS_BYTES = 96
STATE_FIELDS = ("prev_d", "acc", "delta", "have_d", "n_out", "last_skipped", "skip", "steps")
STATS_FIELDS = ("sum_abs", "sum_d2", "sum_ref2", "max_abs", "amax_rot", "ratio", "d", "numel", "has_ref",
                "prec_in", "prec_out", "nonfinite", "error")

_lib = None


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m video_diffusion_mixed_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i64, i32, st = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_int
        P = ctypes.POINTER
        sig = {
            "sb_version": (ctypes.c_char_p, []),
            "sb_last_error": (ctypes.c_char_p, []),
            "sb_workspace_size": (st, [i64, i64, P(ctypes.c_size_t)]),
            "sb_workspace_init": (st, [vp, ctypes.c_size_t, vp]),
            "sb_fp4_sf_bytes": (i64, [i64, i64]),
            "sb_state_init": (st, [vp, vp]),
            "sb_rotate": (st, [vp, vp, i64, i64, i32, vp]),
            "sb_prepare_weight": (st, [vp, vp, i64, i64, i32, P(WeightC), vp, vp]),
            "sb_tdc_step": (st, [vp, P(Config), vp]),
            "sb_select_precision": (st, [vp, P(Rule), P(Config), vp, vp]),
            "sb_prepass": (st, [vp, vp, i64, i64, P(Config), i32, vp, P(Fp4), P(I8), vp, vp, vp]),
            "sb_linear": (st, [vp, P(Fp4), P(I8), vp, P(WeightC), i32, i32, vp, i64, vp, vp]),
            "sb_tdc_record": (st, [vp, vp, i64, i64, vp, i32, vp, vp, vp]),
            "sb_check": (st, [vp, vp]),
            "sb_prepass_static": (st, [vp, vp, i64, i64, P(Config), i32, vp, P(Fp4), P(I8), vp, vp]),
            "sb_wait_flag": (st, [vp, i32, ctypes.c_uint64, vp, vp]),
            "sb_drill_gemm_stall": (st, [i64, ctypes.c_uint64]),
            "sb_tdc_refresh_fp8": (st, [vp, vp, vp, vp, i64, i64, vp, vp]),
            "sb_module_record": (st, [vp, vp, vp, i64, i64, vp, i32, vp, vp, vp, vp]),
            "sb_delta_linear": (st, [vp, P(Fp4), P(I8), vp, P(WeightC), vp, P(Cubes), i32, i32, vp, i64, vp, vp]),
            "sb_linear_records": (st, [vp, P(Fp4), P(I8), vp, P(WeightC), i32, vp, i64, i32, vp, vp, vp]),
            "sb_chunk_records": (st, [vp, i64, i64, i32, vp, vp]),
            "sb_linear_module_record": (st, [vp, P(Fp4), P(I8), vp, P(WeightC), i32, vp, i64, vp, vp, i32, vp, vp, vp,
                                             vp, vp]),
            "sb_tdc_reuse_fp8": (st, [vp, vp, vp, vp, i64, i64, vp, vp]),
            "sb_tdc_refresh": (st, [vp, vp, vp, i64, i64, vp, vp]),
            "sb_tdc_reuse": (st, [vp, vp, vp, i64, i64, vp, vp]),
            "sb_group_slots_bytes": (i64, [i64]),
            "sb_prepass_partial": (st, [vp, vp, i64, i64, i64, i64, P(Config), i32, vp, P(I8), vp, vp, vp]),
            "sb_prepass_finish": (st, [vp, i64, i64, i32, P(Config), i32, vp, vp, vp, vp]),
            "sb_nvfp4_encode": (st, [vp, i64, i64, P(Config), vp, vp, P(Fp4), vp, vp]),
            "sb_tdc_record_partial": (st, [vp, vp, i64, i64, i64, i64, i32, vp, vp, vp, vp]),
            "sb_tdc_finish": (st, [vp, i64, i64, vp, vp, vp, vp]),
            "sb_module_decide": (st, [vp, P(Config), i32, vp, vp, vp]),
            "sb_prepass_chunks": (st, [vp, vp, i64, i64, P(Config), i32, vp, P(Fp4), P(I8), vp, vp, vp]),
            "sb_cube_count": (i64, [P(Cubes), i64]),
            "sb_delta_split": (st, [vp, i64, i64, P(Cubes), vp, vp, vp, vp, vp]),
            "sb_delta_combine": (st, [vp, vp, i64, i64, P(Cubes), i32, vp, vp]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


EXPORTED = ("sb_version", "sb_last_error", "sb_workspace_size", "sb_workspace_init", "sb_fp4_sf_bytes",
            "sb_state_init", "sb_rotate", "sb_prepare_weight", "sb_tdc_step", "sb_select_precision", "sb_prepass",
            "sb_linear", "sb_tdc_record", "sb_check", "sb_prepass_static", "sb_wait_flag", "sb_tdc_refresh",
            "sb_tdc_reuse", "sb_group_slots_bytes", "sb_prepass_partial", "sb_prepass_finish", "sb_nvfp4_encode",
            "sb_tdc_record_partial", "sb_tdc_finish", "sb_module_decide", "sb_prepass_chunks", "sb_cube_count",
            "sb_delta_split", "sb_delta_combine", "sb_drill_gemm_stall", "sb_tdc_refresh_fp8",
            "sb_tdc_reuse_fp8", "sb_module_record", "sb_delta_linear", "sb_linear_records",
            "sb_chunk_records", "sb_linear_module_record")


def _ck(status: int):
    if status != SB_OK:
        raise SixbitError(status, lib().sb_last_error().decode())


def _p(t):
    if t is None:
        return None
    assert t.is_cuda and t.is_contiguous(), "device tensors must be contiguous CUDA tensors"
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def version() -> str:
    return lib().sb_version().decode()


# ------------------------------------------------------------------------------------------------
# Caller-owned buffers
# ------------------------------------------------------------------------------------------------

class Workspace:
    def __init__(self, max_M: int, max_K: int, device="cuda", stream=None):
        n = ctypes.c_size_t(0)
        _ck(lib().sb_workspace_size(max_M, max_K, ctypes.byref(n)))
        self.bytes = n.value
        self.buf = torch.empty(self.bytes, dtype=torch.uint8, device=device)
        _ck(lib().sb_workspace_init(_p(self.buf), self.bytes, _stream(stream)))

    @property
    def ptr(self):
        return _p(self.buf)


class Fp4Tensor:
    def __init__(self, rows: int, cols: int, device="cuda"):
        self.rows, self.cols = rows, cols
        self.codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=device)
        self.sf = torch.empty(int(lib().sb_fp4_sf_bytes(rows, cols)), dtype=torch.uint8, device=device)
        self.gscale = torch.empty(4, dtype=torch.float32, device=device)  # 16-byte slot, element 0 used

    def c(self) -> Fp4:
        return Fp4(self.codes.data_ptr(), self.sf.data_ptr(), self.gscale.data_ptr(), self.rows, self.cols)


class I8Tensor:
    def __init__(self, rows: int, cols: int, device="cuda"):
        self.rows, self.cols = rows, cols
        self.codes = torch.empty((rows, cols), dtype=torch.int8, device=device)
        self.scale = torch.empty(rows, dtype=torch.float32, device=device)

    def c(self) -> I8:
        return I8(self.codes.data_ptr(), self.scale.data_ptr(), self.rows, self.cols)


class Weight:
    """A prepared linear layer: original bf16 weight + bias, rotated NVFP4 and INT8 copies."""

    def __init__(self, W: torch.Tensor, bias: torch.Tensor | None, block: int = 128, ws: Workspace | None = None,
                 stream=None):
        N, K = W.shape
        self.W, self.bias, self.N, self.K, self.block = W.contiguous(), bias, N, K, block
        self.w4 = Fp4Tensor(N, K, W.device)
        self.w8 = I8Tensor(N, K, W.device)
        self._c = WeightC()
        self._c.w4 = self.w4.c()
        self._c.w8 = self.w8.c()
        ws = ws or Workspace(N, K, W.device, stream)
        _ck(lib().sb_prepare_weight(_p(self.W), _p(bias), N, K, block, ctypes.byref(self._c), ws.ptr,
                                    _stream(stream)))

    def c(self) -> WeightC:
        return self._c


def alloc_state(device="cuda", stream=None) -> torch.Tensor:
    st = torch.empty(STATE_BYTES, dtype=torch.uint8, device=device)
    _ck(lib().sb_state_init(_p(st), _stream(stream)))
    return st


def state_init(state: torch.Tensor, stream=None):
    """Reset an existing module state (sb_state_init)."""
    _ck(lib().sb_state_init(_p(state), _stream(stream)))


def alloc_stats(device="cuda") -> torch.Tensor:
    return torch.zeros(STATS_BYTES, dtype=torch.uint8, device=device)


def decode_state(buf: torch.Tensor) -> dict:
    h = buf.detach().cpu()
    d = h[:24].view(torch.float64).tolist()
    i = h[24:44].view(torch.int32).tolist()
    return dict(zip(STATE_FIELDS, d + i))


def decode_stats(buf: torch.Tensor) -> dict:
    h = buf.detach().cpu()
    d = h[:64].view(torch.float64).tolist()
    i = h[64:84].view(torch.int32).tolist()
    return dict(zip(STATS_FIELDS, d + i))


def config(rho: float = 64.0, tdc_thresh: float = 0.1, block: int = 128, force_prec: int = -1) -> Config:
    return Config(rho, tdc_thresh, block, force_prec)


# ------------------------------------------------------------------------------------------------
# Entry points (same names as the C ABI, minus the prefix)
# ------------------------------------------------------------------------------------------------

def rotate(X: torch.Tensor, Y: torch.Tensor, block: int = 128, stream=None):
    M, K = X.shape
    _ck(lib().sb_rotate(_p(X), _p(Y), M, K, block, _stream(stream)))


def tdc_step(state: torch.Tensor, cfg: Config, stream=None):
    _ck(lib().sb_tdc_step(_p(state), ctypes.byref(cfg), _stream(stream)))


def select_precision(state: torch.Tensor, rule: Rule, cfg: Config, prec: torch.Tensor, stream=None):
    _ck(lib().sb_select_precision(_p(state), ctypes.byref(rule), ctypes.byref(cfg), _p(prec), _stream(stream)))


def prepass(X, X_ref, cfg: Config, mode: int, prec, a4: Fp4Tensor | None, a8: I8Tensor | None, stats, ws: Workspace,
            stream=None):
    M, K = X.shape
    c4 = ctypes.byref(a4.c()) if a4 is not None else None
    c8 = ctypes.byref(a8.c()) if a8 is not None else None
    _ck(lib().sb_prepass(_p(X), _p(X_ref), M, K, ctypes.byref(cfg), mode, _p(prec), c4, c8, _p(stats), ws.ptr,
                         _stream(stream)))


def prepass_chunks(X, chunks, cfg: Config, mode: int, prec, a4: Fp4Tensor | None, a8: I8Tensor | None, stats,
                   ws: Workspace, stream=None):
    """sb_prepass_chunks: the pre-pass from the producer's chunk records (float32 [M, K/128, 4])."""
    M, K = X.shape
    c4 = ctypes.byref(a4.c()) if a4 is not None else None
    c8 = ctypes.byref(a8.c()) if a8 is not None else None
    _ck(lib().sb_prepass_chunks(_p(X), _p(chunks), M, K, ctypes.byref(cfg), mode, _p(prec), c4, c8, _p(stats),
                                ws.ptr, _stream(stream)))


def prepass_static(X, X_ref, cfg: Config, mode: int, prec, a4: Fp4Tensor | None, a8: I8Tensor | None, stats,
                   stream=None):
    """sb_prepass with the library's built-in scratch (no workspace; see include/sixbit.h)."""
    M, K = X.shape
    c4 = ctypes.byref(a4.c()) if a4 is not None else None
    c8 = ctypes.byref(a8.c()) if a8 is not None else None
    _ck(lib().sb_prepass_static(_p(X), _p(X_ref), M, K, ctypes.byref(cfg), mode, _p(prec), c4, c8, _p(stats),
                                _stream(stream)))


def linear(X, a4: Fp4Tensor | None, a8: I8Tensor | None, prec, w: Weight, Y, epilogue: int = EPI_NONE,
           out_dtype: int = OUT_BF16, ws: Workspace | None = None, stream=None):
    M = Y.shape[0]
    c4 = ctypes.byref(a4.c()) if a4 is not None else None
    c8 = ctypes.byref(a8.c()) if a8 is not None else None
    _ck(lib().sb_linear(_p(X), c4, c8, _p(prec), ctypes.byref(w.c()), epilogue, out_dtype, _p(Y), M, ws.ptr,
                        _stream(stream)))


def module_record(y, x, cache, prec, stats, state, ws: Workspace, update_cache: bool = True, stream=None):
    """The difference statistic of y against x and the TDC record of y in one pass (sb_module_record)."""
    M, C = y.shape
    _ck(lib().sb_module_record(_p(y), _p(x), _p(cache), M, C, _p(prec), int(update_cache), _p(stats), _p(state),
                               ws.ptr, _stream(stream)))


def linear_records(X, a4, a8, prec, w: Weight, Y, records, epilogue: int = EPI_NONE, block: int = 128,
                   ws: Workspace = None, stream=None):
    """sb_linear (bf16 output) that also writes Y's chunk records (float32 [M][N/128][4]) for a
    next pre-pass with Hadamard block `block`."""
    M = Y.shape[0]
    c4 = ctypes.byref(a4.c()) if a4 is not None else None
    c8 = ctypes.byref(a8.c()) if a8 is not None else None
    _ck(lib().sb_linear_records(_p(X), c4, c8, _p(prec), ctypes.byref(w.c()), epilogue, _p(Y), M, block,
                                _p(records), ws.ptr, _stream(stream)))


def linear_module_record(X, a4, a8, prec, w: Weight, Y, x, cache, records, stats, state, ws: Workspace,
                         epilogue: int = EPI_NONE, update_cache: bool = True, stream=None):
    """sb_linear (bf16 output) fused with sb_module_record of that output (sb_linear_module_record);
    records: float32 scratch of M * (N / 128) * 8 values."""
    M = Y.shape[0]
    c4 = ctypes.byref(a4.c()) if a4 is not None else None
    c8 = ctypes.byref(a8.c()) if a8 is not None else None
    _ck(lib().sb_linear_module_record(_p(X), c4, c8, _p(prec), ctypes.byref(w.c()), epilogue, _p(Y), M, _p(x),
                                      _p(cache), int(update_cache), _p(records), _p(stats), _p(state), ws.ptr,
                                      _stream(stream)))


def chunk_records(X, records, block: int = 128, stream=None):
    """The chunk records of a bf16 tensor (sb_chunk_records)."""
    M, K = X.shape
    _ck(lib().sb_chunk_records(_p(X), M, K, block, _p(records), _stream(stream)))


def tdc_record(y_new, y_cache, d_src, state, ws: Workspace, update_cache: bool = True, stream=None):
    M, C = y_new.shape
    _ck(lib().sb_tdc_record(_p(y_new), _p(y_cache), M, C, _p(d_src), int(update_cache), _p(state), ws.ptr,
                            _stream(stream)))


def check(ws: Workspace, stream=None):
    _ck(lib().sb_check(ws.ptr, _stream(stream)))


def module_decide(state, cfg: Config, rules, precs, stream=None):
    """sb_module_decide: the TDC check, then precs[i] from rules[i], in one launch."""
    n = len(rules)
    R = (Rule * n)(*rules)
    Pp = (ctypes.c_void_p * n)(*[t.data_ptr() for t in precs])
    _ck(lib().sb_module_decide(_p(state), ctypes.byref(cfg), n, ctypes.cast(R, ctypes.c_void_p),
                               ctypes.cast(Pp, ctypes.c_void_p), _stream(stream)))


# ---- token sharding (include/sixbit.h): partial row work, slot gathering, final reduction ----

GROUP_ROWS = 16
SLOT_BYTES = 48


def alloc_slots(M_total: int, device="cuda") -> torch.Tensor:
    """Zero-filled group-slot array of an M_total-row tensor (int64 words, 16-byte aligned)."""
    n = lib().sb_group_slots_bytes(M_total)
    if n < 0:
        raise SixbitError(SB_ESHAPE, f"M_total must be >= 1 (got {M_total})")
    return torch.zeros(n // 8, dtype=torch.int64, device=device)


def gather_slots(slots: torch.Tensor, group=None) -> torch.Tensor:
    """Combine the shards' slot arrays in place: every rank wrote a disjoint range of its
    zero-filled copy, so an int64 all-reduce SUM reproduces every written word bit for bit."""
    import torch.distributed as dist
    dist.all_reduce(slots, op=dist.ReduceOp.SUM, group=group)
    return slots


def prepass_partial(X, X_ref, row0: int, M_total: int, cfg: Config, mode: int, prec, a8: I8Tensor | None, slots,
                    ws: Workspace, stream=None):
    M, K = X.shape
    c8 = ctypes.byref(a8.c()) if a8 is not None else None
    _ck(lib().sb_prepass_partial(_p(X), _p(X_ref), M, K, row0, M_total, ctypes.byref(cfg), mode, _p(prec), c8,
                                 _p(slots), ws.ptr, _stream(stream)))


def prepass_finish(slots, M_total: int, K: int, has_ref: bool, cfg: Config, mode: int, prec, stats, ws: Workspace,
                   stream=None):
    _ck(lib().sb_prepass_finish(_p(slots), M_total, K, int(has_ref), ctypes.byref(cfg), mode, _p(prec), _p(stats),
                                ws.ptr, _stream(stream)))


def nvfp4_encode(X, cfg: Config, prec, stats, a4: Fp4Tensor, ws: Workspace, stream=None):
    M, K = X.shape
    _ck(lib().sb_nvfp4_encode(_p(X), M, K, ctypes.byref(cfg), _p(prec), _p(stats), ctypes.byref(a4.c()), ws.ptr,
                              _stream(stream)))


def tdc_record_partial(y_new, y_cache, row0: int, M_total: int, state, slots, ws: Workspace,
                       update_cache: bool = True, stream=None):
    M, C = y_new.shape
    _ck(lib().sb_tdc_record_partial(_p(y_new), _p(y_cache), M, C, row0, M_total, int(update_cache), _p(state),
                                    _p(slots), ws.ptr, _stream(stream)))


def tdc_finish(slots, M_total: int, C: int, d_src, state, ws: Workspace, stream=None):
    _ck(lib().sb_tdc_finish(_p(slots), M_total, C, _p(d_src), _p(state), ws.ptr, _stream(stream)))


def tdc_refresh(x, y, delta, state, stream=None):
    """At a computed step keep the module's residual: delta = bf16(y - x) (sb_tdc_refresh)."""
    M, C = x.shape
    _ck(lib().sb_tdc_refresh(_p(x), _p(y), _p(delta), M, C, _p(state), _stream(stream)))


def tdc_reuse(x, delta, y, state, stream=None):
    """At a skipped step produce the output from the kept residual: y = bf16(x + delta)."""
    M, C = x.shape
    _ck(lib().sb_tdc_reuse(_p(x), _p(delta), _p(y), M, C, _p(state), _stream(stream)))


class Fp8Residual:
    """Caller-owned FP8 residual of M token rows of C channels: E4M3 codes and one scale per row."""

    def __init__(self, M: int, C: int, device="cuda"):
        self.codes = torch.zeros((M, C), dtype=torch.uint8, device=device)
        self.scale = torch.zeros(M, dtype=torch.float32, device=device)


def tdc_refresh_fp8(x, y, d: Fp8Residual, state, stream=None):
    M, C = x.shape
    _ck(lib().sb_tdc_refresh_fp8(_p(x), _p(y), _p(d.codes), _p(d.scale), M, C, _p(state), _stream(stream)))


def tdc_reuse_fp8(x, d: Fp8Residual, y, state, stream=None):
    M, C = x.shape
    _ck(lib().sb_tdc_reuse_fp8(_p(x), _p(d.codes), _p(d.scale), _p(y), M, C, _p(state), _stream(stream)))


def wait_flag(flag, value: int, limit_ns: int, ws: Workspace, stream=None):
    """Enqueue a bounded device-side wait until flag[0] == value (see sb_wait_flag)."""
    assert flag.dtype == torch.int32
    _ck(lib().sb_wait_flag(_p(flag), int(value), int(limit_ns), ws.ptr, _stream(stream)))


def drill_gemm_stall(withhold_stage: int, limit_ns: int):
    """Arm the next linear() launch to stall on a withheld stage (see sb_drill_gemm_stall)."""
    _ck(lib().sb_drill_gemm_stall(int(withhold_stage), int(limit_ns)))


# ---- delta tokens (include/sixbit.h: sb_cubes, sb_delta_split, sb_delta_combine) ----

def cubes(text: int, frames: int, height: int, width: int, ct: int = 2, ch: int = 2, cw: int = 2) -> Cubes:
    return Cubes(text, frames, height, width, ct, ch, cw)


def cube_count(c: Cubes, M: int) -> int:
    return int(lib().sb_cube_count(ctypes.byref(c), M))


class CoreTokens:
    """Caller-owned outputs of sb_delta_split for M tokens of K channels."""

    def __init__(self, c: Cubes, M: int, K: int, device="cuda"):
        n = cube_count(c, M)
        if n < 1:
            raise SixbitError(SB_ESHAPE, "the cube layout does not cover the tokens")
        self.n = n
        self.codes = torch.empty((n, K), dtype=torch.uint8, device=device)
        self.scale = torch.empty(n, dtype=torch.float32, device=device)
        self.bf16 = torch.empty((n, K), dtype=torch.bfloat16, device=device)


def delta_split(X, c: Cubes, core: CoreTokens, delta, stream=None):
    M, K = X.shape
    _ck(lib().sb_delta_split(_p(X), M, K, ctypes.byref(c), _p(core.codes), _p(core.scale), _p(core.bf16), _p(delta),
                             _stream(stream)))


def delta_linear(delta, a4, a8, prec, w: "Weight", y_core, c: Cubes, Y, epilogue: int = EPI_NONE,
                 out_dtype: int = OUT_BF16, ws: "Workspace" = None, stream=None):
    """Y = act(linear(delta) + y_core[cube(t)]) with the combine in the GEMM epilogue (sb_delta_linear)."""
    M = Y.shape[0]
    c4 = ctypes.byref(a4.c()) if a4 is not None else None
    c8 = ctypes.byref(a8.c()) if a8 is not None else None
    _ck(lib().sb_delta_linear(_p(delta), c4, c8, _p(prec), ctypes.byref(w.c()), _p(y_core), ctypes.byref(c), epilogue,
                              out_dtype, _p(Y), M, ws.ptr, _stream(stream)))


def delta_combine(y_delta, y_core, c: Cubes, Y, epilogue: int = EPI_NONE, stream=None):
    M, N = Y.shape
    _ck(lib().sb_delta_combine(_p(y_delta), _p(y_core), M, N, ctypes.byref(c), epilogue, _p(Y), _stream(stream)))
