"""GPU parity of the Temporal Delta Cache and of the decision kernels against the CPU oracle.

delta and every state field are compared bit-exactly; the 30-block trajectory must produce the
oracle's decision log (skip / NVFP4 / INT8 / BF16 per block and step) exactly.
"""
import numpy as np
import pytest
import torch

import oracle
from video_diffusion_mixed_b200 import synth
from gpu_helpers import npy, u16

pytestmark = pytest.mark.gpu


def ostate_dict(s):
    d = s.as_dict()
    return {k: d[k] for k in ("prev_d", "acc", "delta", "have_d", "n_out", "last_skipped", "skip")}


def gstate_dict(sb, st):
    d = sb.decode_state(st)
    return {k: d[k] for k in ("prev_d", "acc", "delta", "have_d", "n_out", "last_skipped", "skip")}


# (70001, 64): more than 4096 groups of 16 rows, so the last CTA folds the group sums in chunks
@pytest.mark.parametrize("M,C", [(1, 8), (33, 1920), (256, 3072), (100, 12288), (70001, 64)])
def test_tdc_record_delta_bitexact(sbg, M, C):
    ws = sbg.Workspace(M, C)
    st = sbg.alloc_state()
    y0 = synth.activations(M, C, seed=1, device="cuda")
    y1 = synth.noisy_copy(y0, 0.05, seed=2)
    cache = torch.zeros_like(y0)
    sbg.tdc_record(y0, cache, None, st, ws)   # first output: no delta, cache <- y0
    sbg.check(ws)
    assert torch.equal(cache, y0)
    s = gstate_dict(sbg, st)
    assert s["n_out"] == 1 and s["delta"] == 0.0 and s["have_d"] == 0
    sbg.tdc_record(y1, cache, None, st, ws)   # second: delta(y1, y0), cache <- y1
    sbg.check(ws)
    ref, s1, s2 = oracle.tdc_delta(u16(y1), u16(y0))
    s = gstate_dict(sbg, st)
    assert s["delta"] == ref, (s["delta"], ref)
    assert s["n_out"] == 2 and s["acc"] == 0.0
    assert torch.equal(cache, y1)


def test_tdc_record_without_cache_update(sbg):
    M, C = 64, 512
    ws = sbg.Workspace(M, C)
    st = sbg.alloc_state()
    y0 = synth.activations(M, C, seed=3, device="cuda")
    y1 = synth.noisy_copy(y0, 0.2, seed=4)
    cache = y0.clone()
    sbg.tdc_record(y0, cache, None, st, ws)
    sbg.tdc_record(y1, cache, None, st, ws, update_cache=False)
    sbg.check(ws)
    assert torch.equal(cache, y0)
    assert sbg.decode_state(st)["delta"] == oracle.tdc_delta(u16(y1), u16(y0))[0]


def test_tdc_zero_cache_gives_inf(sbg):
    ws = sbg.Workspace(16, 64)
    st = sbg.alloc_state()
    z = torch.zeros((16, 64), dtype=torch.bfloat16, device="cuda")
    y = torch.ones((16, 64), dtype=torch.bfloat16, device="cuda")
    cache = z.clone()
    sbg.tdc_record(z, cache, None, st, ws)
    sbg.tdc_record(y, cache, None, st, ws)
    sbg.check(ws)
    assert sbg.decode_state(st)["delta"] == float("inf")


@pytest.mark.parametrize("fused", [False, True], ids=["separate", "module_decide"])
def test_decision_kernels_follow_the_oracle_state_machine(sbg, fused):
    """Drive the device state with dyadic deltas and ds; compare every field after every call
    (the TDC check and the layers' precision choices as separate launches, or as one)."""
    ws = sbg.Workspace(32, 128)
    st = sbg.alloc_state()
    os_ = oracle.State()
    cfg = sbg.config(tdc_thresh=0.125)
    rule = sbg.Rule(1.0, 0.0, 0.1)
    prec = torch.zeros(1, dtype=torch.int32, device="cuda")
    stats = sbg.alloc_stats()
    base = torch.ones((32, 128), dtype=torch.bfloat16, device="cuda")
    cache = torch.zeros_like(base)
    # outputs y_k = 1 + k/32 so that delta between consecutive computed outputs is dyadic
    k_out = 0
    rule2 = sbg.Rule(0.5, 0.0625, 0.0625)
    prec2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    for t in range(24):
        if fused:
            sbg.module_decide(st, cfg, [rule, rule2], [prec, prec2])
        else:
            sbg.tdc_step(st, cfg)
            sbg.select_precision(st, rule, cfg, prec)
            sbg.select_precision(st, rule2, cfg, prec2)
        oracle.tdc_step(os_, 0.125)
        p_ref = oracle.select_precision(os_, 1.0, 0.0, 0.1)
        p2_ref = oracle.select_precision(os_, 0.5, 0.0625, 0.0625)
        torch.cuda.synchronize()
        assert int(prec.item()) == p_ref, t
        assert int(prec2.item()) == p2_ref, t
        assert gstate_dict(sbg, st) == ostate_dict(os_), t
        if p_ref == oracle.SKIP:
            continue
        y = base * (1.0 + k_out / 64.0)
        x = base * (1.0 + 0.0625 * (t % 3))  # module input: d = |y - x| / |x|
        sbg.prepass(y, x, sbg.config(), sbg.PREPASS_STATS, None, None, None, stats, ws)
        st_d = sbg.decode_stats(stats)
        ref_p = oracle.prepass(u16(y), u16(x), 128)
        assert st_d["d"] == ref_p["d"]
        prev = u16(cache)
        sbg.tdc_record(y, cache, stats, st, ws)
        delta = oracle.tdc_delta(u16(y), prev)[0] if os_.n_out >= 1 else None
        oracle.tdc_record(os_, delta, ref_p["d"])
        sbg.check(ws)
        assert gstate_dict(sbg, st) == ostate_dict(os_), t
        k_out += 1


@pytest.mark.parametrize("M,ks", [(256, tuple(range(30))), (17776, (0, 7, 14, 22, 29))],
                         ids=["256tok_30blocks", "17776tok_5blocks"])
def test_trajectory_decisions_bitexact(sbg, M, ks):
    """DiT blocks x 50 steps (hidden 3072): difference-driven NVFP4/INT8, PDR BF16 fallback
    (rho 64), TDC threshold 0.1; all 30 blocks at 256 tokens, and a spread of 5 blocks at the full
    17776 tokens. The decision log and every delta and d must equal the oracle's."""
    blocks, steps, C = 30, 50, 3072
    cfg = sbg.config(rho=64.0, tdc_thresh=0.1)
    rule = sbg.Rule(1.0, 0.0, 0.1)
    ws = sbg.Workspace(M, C)
    a4, a8 = sbg.Fp4Tensor(M, C), sbg.I8Tensor(M, C)
    sx, sy = sbg.alloc_stats(), sbg.alloc_stats()
    prec = torch.zeros(1, dtype=torch.int32, device="cuda")
    log_gpu = np.zeros((len(ks), steps), np.int32)
    log_ref = np.zeros((len(ks), steps), np.int32)
    for kk, k in enumerate(ks):
        traj = synth.Trajectory(M, C, k, blocks=blocks, steps=steps, seed=0, device="cuda")
        st = sbg.alloc_state()
        os_ = oracle.State()
        cache = torch.zeros((M, C), dtype=torch.bfloat16, device="cuda")
        last_y = None
        for t in range(steps):
            x, y = traj.current()
            sbg.tdc_step(st, cfg)
            sbg.select_precision(st, rule, cfg, prec)
            sbg.prepass(x, None, cfg, sbg.PREPASS_QUANT, prec, a4, a8, sx, ws)
            sbg.prepass(y, x, cfg, sbg.PREPASS_STATS, prec, None, None, sy, ws)
            sbg.tdc_record(y, cache, sy, st, ws)
            sbg.check(ws)
            log_gpu[kk, t] = int(prec.item())
            # oracle
            oracle.tdc_step(os_, 0.1)
            p = oracle.select_precision(os_, 1.0, 0.0, 0.1)
            if p != oracle.SKIP:
                rx = oracle.prepass(u16(x), None, 128, want_rot=False)
                p = oracle.apply_pdr(p, rx["ratio"], 64.0)
                ry = oracle.prepass(u16(y), u16(x), 128, want_rot=False)
                yb = u16(y)
                delta = oracle.tdc_delta(yb, last_y)[0] if last_y is not None else None
                oracle.tdc_record(os_, delta, ry["d"])
                last_y = yb
            log_ref[kk, t] = p
            g = gstate_dict(sbg, st)
            assert g == ostate_dict(os_), (k, t, g, ostate_dict(os_))
            if t + 1 < steps:
                traj.advance()
    assert np.array_equal(log_gpu, log_ref)
    # the workload exercises every branch of the decision logic
    assert {0, 1, 2, 3} <= set(np.unique(log_ref).tolist())


def test_trajectory_resumes_from_a_checkpoint(sbg):
    """Checkpoint and resume: the decision state of a module is the 64-byte state record plus its
    cached last output (and, for the reuse path, the kept residual), all caller-owned device
    buffers. Saving them to host memory at step 25 of a 50-step trajectory, restoring them into
    fresh buffers and running steps 25..49 must give the decision log, every state field and the
    cache of the uninterrupted run, bit for bit."""
    M, C, steps, k = 256, 3072, 50, 3  # block 3 carries the outlier channels (PDR fires)
    cfg = sbg.config(rho=64.0, tdc_thresh=0.1)
    rule = sbg.Rule(1.0, 0.0, 0.1)
    ws = sbg.Workspace(M, C)
    a4, a8 = sbg.Fp4Tensor(M, C), sbg.I8Tensor(M, C)
    sx, sy = sbg.alloc_stats(), sbg.alloc_stats()
    prec = torch.zeros(1, dtype=torch.int32, device="cuda")

    def run(traj, st, cache, D, t0, t1, log):
        for t in range(t0, t1):
            x, y = traj.current()
            sbg.tdc_step(st, cfg)
            sbg.select_precision(st, rule, cfg, prec)
            sbg.prepass(x, None, cfg, sbg.PREPASS_QUANT, prec, a4, a8, sx, ws)
            sbg.prepass(y, x, cfg, sbg.PREPASS_STATS, prec, None, None, sy, ws)
            sbg.tdc_record(y, cache, sy, st, ws)
            sbg.tdc_refresh(x, y, D, st)
            sbg.check(ws)
            log.append(int(prec.item()))
            if t + 1 < steps:
                traj.advance()

    # uninterrupted
    traj = synth.Trajectory(M, C, k, steps=steps, seed=0, device="cuda")
    st = sbg.alloc_state()
    cache = torch.zeros((M, C), dtype=torch.bfloat16, device="cuda")
    D = torch.zeros_like(cache)
    full = []
    run(traj, st, cache, D, 0, steps, full)
    # interrupted at step 25: checkpoint to host, fresh buffers, restore, continue
    traj2 = synth.Trajectory(M, C, k, steps=steps, seed=0, device="cuda")
    st2 = sbg.alloc_state()
    cache2 = torch.zeros_like(cache)
    D2 = torch.zeros_like(cache)
    part = []
    run(traj2, st2, cache2, D2, 0, 25, part)
    ckpt = {"state": st2.cpu().clone(), "cache": cache2.cpu().clone(), "D": D2.cpu().clone()}
    del st2, cache2, D2
    st3 = sbg.alloc_state()
    cache3 = torch.zeros_like(cache)
    D3 = torch.zeros_like(cache)
    st3.copy_(ckpt["state"])
    cache3.copy_(ckpt["cache"])
    D3.copy_(ckpt["D"])
    run(traj2, st3, cache3, D3, 25, steps, part)
    assert part == full
    assert sbg.SKIP in full and any(p != sbg.SKIP for p in full)  # skipped and computed steps
    assert torch.equal(st3, st) and torch.equal(cache3, cache) and torch.equal(D3, D)
