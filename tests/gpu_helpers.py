"""Shared helpers of the GPU parity tests (inputs, conversions, comparisons)."""
import numpy as np
import torch


def u16(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def npy(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().numpy()


def rel_fro(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (den if den > 0 else 1.0))


def bf16_bits_to_f64(h: np.ndarray) -> np.ndarray:
    return (h.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def bf16_ulp_diff(gpu_bits: np.ndarray, ref_f64: np.ndarray) -> np.ndarray:
    """Distance in bf16 units in the last place between GPU bf16 outputs and the RNE-rounded
    FP64 reference (sign-magnitude ordering)."""
    import oracle
    ref_bits = oracle.f32_to_bf16(ref_f64.astype(np.float32))

    def key(b):
        b = b.astype(np.int32)
        return np.where(b & 0x8000, -(b & 0x7FFF), b & 0x7FFF)
    return np.abs(key(gpu_bits) - key(ref_bits))


def sample_rows(M: int, step: int = 64) -> np.ndarray:
    r = list(range(0, M, step))
    if r[-1] != M - 1:
        r.append(M - 1)
    return np.array(r, dtype=np.int64)


def assert_close(got, ref, tol: float = 1e-3):
    """The output tolerance of the quantized and BF16 linear layers, checked two ways:
    relative Frobenius error <= tol over the whole compared block, and elementwise
    |got - ref| <= tol * max|ref| + tol * |ref|, which a localized error (one wrong column group,
    one wrong tile) would break even when it is too small to move the Frobenius norm. The
    elementwise bound holds for every correct kernel here: FP32 accumulation and the FP32
    dequant/bias epilogue err by a few FP32 ulps of the row's magnitude, the SFU tanh of the GELU
    by about 2^-11 of 0.5 |v|, both far below 1e-3 of the block's largest output."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    fro = rel_fro(got, ref)
    assert fro <= tol, f"relative Frobenius error {fro:.3e} > {tol:g}"
    bound = tol * float(np.max(np.abs(ref))) + tol * np.abs(ref)
    err = np.abs(got - ref)
    bad = np.argwhere(err > bound)
    assert bad.size == 0, (f"{len(bad)} elements outside the elementwise bound; first at {tuple(bad[0])}: "
                           f"got {got[tuple(bad[0])]!r}, ref {ref[tuple(bad[0])]!r}")
