"""Failure detection on the GPU without a GPU fault: bounded device-side waits.

sb_wait_flag polls a device-visible int32 until it holds a value and gives up after a deadline of
device time, recording SB_ETIMEOUT in the workspace. The waits here either end by themselves (the
flag is already set, or the host sets it through page-locked memory) or run out on a flag that
nothing sets; no kernel ever waits for another launch. After a timeout the context must still run
the pre-pass bit-exactly. (The bounded waits of the pipelined kernels use the same %globaltimer
deadline.)
"""
import ctypes
import threading
import time

import numpy as np
import pytest
import torch

import oracle
from video_diffusion_mixed_b200 import synth
from gpu_helpers import npy, u16

pytestmark = pytest.mark.gpu


def test_wait_on_a_flag_nothing_sets_times_out_and_is_reported(sbg):
    ws = sbg.Workspace(64, 256)
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.monotonic()
    sbg.wait_flag(flag, 1, 20_000_000, ws)  # 20 ms
    with pytest.raises(sbg.SixbitError) as e:
        sbg.check(ws)
    assert e.value.status == sbg.SB_ETIMEOUT
    assert time.monotonic() - t0 < 5.0
    sbg.check(ws)  # the error word was cleared by the first check


def test_context_stays_usable_after_a_timeout(sbg):
    ws = sbg.Workspace(64, 256)
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    sbg.wait_flag(flag, 7, 5_000_000, ws)
    with pytest.raises(sbg.SixbitError):
        sbg.check(ws)
    X = synth.activations(40, 1024, n_outlier=3, scale=20.0, seed=5, device="cuda")
    Y = torch.empty((40, 1024), dtype=torch.float32, device="cuda")
    sbg.rotate(X, Y, 128)
    torch.cuda.synchronize()
    assert np.array_equal(npy(Y).view(np.uint32), oracle.rotate_rows(u16(X), 128).view(np.uint32))


def test_wait_on_a_set_flag_returns_at_once(sbg):
    ws = sbg.Workspace(64, 256)
    flag = torch.full((1,), 3, dtype=torch.int32, device="cuda")
    t0 = time.monotonic()
    sbg.wait_flag(flag, 3, 2_000_000_000, ws)
    sbg.check(ws)
    assert time.monotonic() - t0 < 1.0


def test_wait_ends_when_the_host_sets_the_flag(sbg):
    from cuda.bindings import runtime as cudart
    ws = sbg.Workspace(64, 256)
    # mapped page-locked host memory and its documented device address
    err, hptr = cudart.cudaHostAlloc(4, cudart.cudaHostAllocMapped)
    assert err == cudart.cudaError_t.cudaSuccess
    try:
        err, dptr = cudart.cudaHostGetDevicePointer(hptr, 0)
        assert err == cudart.cudaError_t.cudaSuccess
        host = (ctypes.c_int32 * 1).from_address(hptr)
        host[0] = 0
        L = sbg.lib()
        stream = torch.cuda.current_stream()
        t0 = time.monotonic()
        st = L.sb_wait_flag(ctypes.c_void_p(dptr), 1, 3_000_000_000, ws.ptr, ctypes.c_void_p(stream.cuda_stream))
        assert st == sbg.SB_OK

        def setter():
            time.sleep(0.05)
            host[0] = 1

        th = threading.Thread(target=setter)
        th.start()
        sbg.check(ws)  # synchronises the stream: returns once the kernel saw the flag
        th.join()
        assert time.monotonic() - t0 < 2.5
    finally:
        torch.cuda.synchronize()
        cudart.cudaFreeHost(hptr)


@pytest.mark.parametrize("M,N,stage", [(512, 512, 2), (4096, 2560, 6)])
@pytest.mark.parametrize("prec", [0, 1, 2])
def test_gemm_stall_drill_times_out_and_the_next_gemm_is_exact(sbg, prec, M, N, stage):
    """The GEMM's pipeline waits give up on a withheld stage: the leader CTA of every pair skips the
    copies of one K-block stage, the MMA issuer's bounded wait for it runs out (20 ms), every other
    role ends by the abort flag or its own limit, and the launch reports SB_ETIMEOUT. The next,
    unarmed launch in the same context gives the same outputs bit for bit as one before the drill.
    (512 x 512: one tile per pair; 4096 x 2560: 160 tiles, so pairs stall with tiles still queued.)"""
    K = 1024
    X = synth.activations(M, K, n_outlier=4, scale=20.0, seed=9, device="cuda")
    W = synth.weight(N, K, seed=9, device="cuda")
    ws = sbg.Workspace(max(M, N), K)
    w = sbg.Weight(W, None, 128, ws)
    a4, a8, st = sbg.Fp4Tensor(M, K), sbg.I8Tensor(M, K), sbg.alloc_stats()
    p = torch.tensor([prec], dtype=torch.int32, device="cuda")
    sbg.prepass(X, None, sbg.config(force_prec=prec), sbg.PREPASS_QUANT, p, a4, a8, st, ws)
    sbg.check(ws)
    out = sbg.OUT_RAW if prec == sbg.INT8 else sbg.OUT_F32
    dt = torch.int32 if prec == sbg.INT8 else torch.float32

    def run():
        Y = torch.full((M, N), 7, dtype=dt, device="cuda")
        sbg.linear(X, a4, a8, p, w, Y, out_dtype=out, ws=ws)
        return Y

    before = run()
    sbg.check(ws)
    t0 = time.monotonic()
    sbg.drill_gemm_stall(stage, 20_000_000)
    run()
    with pytest.raises(sbg.SixbitError) as e:
        sbg.check(ws)
    assert e.value.status == sbg.SB_ETIMEOUT
    assert time.monotonic() - t0 < 5.0
    after = run()
    sbg.check(ws)
    assert torch.equal(before.view(torch.int32), after.view(torch.int32))
