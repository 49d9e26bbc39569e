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
