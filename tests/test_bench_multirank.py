"""The N > 1 host path of bench.py on CPU, with world-size-2 gloo process groups.

bench.py runs replicas (every rank its own full step on its own batch, no data-path
collective); the only cross-rank step is the timing reduction: the job takes the slowest rank's
device time, and the whole-job throughput counts every rank's batch. The reference arm runs on
rank 0 alone.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        local_ms = 10.0 + 5.0 * rank  # rank 1 is the slower one
        job_ms = bench.max_over_ranks(local_ms, world, dist, "cpu")
        # a second reduction in the same order on every rank (the bench reduces twice)
        job_ms2 = bench.max_over_ranks(2.0 * local_ms, world, dist, "cpu")
        out[rank] = (job_ms, job_ms2)
    finally:
        dist.destroy_process_group()


def test_timing_is_the_max_over_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True,
                           start_method="spawn")
        res = dict(out)
    assert res == {0: (15.0, 30.0), 1: (15.0, 30.0)}


def test_whole_job_throughput_counts_every_replica():
    sys.path.insert(0, ROOT)
    import bench
    one = bench.whole_job_tflops(1, 5.37e12, 2.5)
    assert abs(one - 5.37e12 / 2.5e-3 / 1e12) < 1e-9
    assert abs(bench.whole_job_tflops(4, 5.37e12, 2.5) - 4 * one) < 1e-9
    assert bench.max_over_ranks(3.5, 1, None, "cpu") == 3.5  # one rank: no collective at all


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    bench.run_reference(type("A", (), {"workload": "ffn5b", "cpu_rows": 2, "warmup": 1, "steps": 1})())
    assert capsys.readouterr().out == ""


# ---- the token-sharded step's host sequence (bench.ShardedFfnStep), with a stand-in library ----

class _FakeLib:
    """Records the calls of bench.ShardedFfnStep. Its partial kernels write, into the group slots
    of their own rows only, words derived from the rows' contents; its finish kernels record the
    slot array they are given. Everything else only logs its name."""
    NVFP4, INT8, BF16, SKIP = 0, 1, 2, 3
    PREPASS_QUANT, PREPASS_STATS, EPI_GELU = 0, 1, 1

    def __init__(self):
        self.log, self.finish_inputs = [], []

    def config(self, **kw):
        return kw

    def alloc_slots(self, M_total, device="cpu"):
        import torch
        return torch.zeros(-(-M_total // 16) * 6, dtype=torch.int64)

    @staticmethod
    def _words(t, r0, r1, tag):
        # 6 int64 words per 16-row group from the group's rows (this rank's part of it)
        return [int(t[r0:r1].sum()) * 7 + tag * 1000003 + k for k in range(6)]

    def _partial(self, name, X, row0, slots, tag):
        M = X.shape[0]
        for g in range(row0 // 16, -(-(row0 + M) // 16)):
            r0, r1 = max(g * 16, row0) - row0, min(g * 16 + 16, row0 + M) - row0
            slots[g * 6:(g + 1) * 6] += __import__("torch").tensor(self._words(X, r0, r1, tag))
        self.log.append(name)

    def prepass_partial(self, X, X_ref, row0, M_total, cfg, mode, prec, a8, slots, ws):
        self._partial("prepass_partial", X, row0, slots, 1 + mode + (0 if X_ref is None else 2))

    def tdc_record_partial(self, y_new, y_cache, row0, M_total, state, slots, ws):
        self._partial("tdc_record_partial", y_new, row0, slots, 9)

    def prepass_finish(self, slots, M_total, K, has_ref, cfg, mode, prec, stats, ws):
        self.finish_inputs.append(slots.clone())
        self.log.append("prepass_finish")

    def tdc_finish(self, slots, M_total, C, d_src, state, ws):
        self.finish_inputs.append(slots.clone())
        self.log.append("tdc_finish")

    def __getattr__(self, name):  # module_decide, nvfp4_encode, linear, gather_slots ...
        if name == "gather_slots":
            from video_diffusion_mixed_b200 import sixbit
            return sixbit.gather_slots
        return lambda *a, **k: self.log.append(name)


def _fake_step_state(rank, M):
    import torch
    S = type("S", (), {})()
    S.M, S.K1, S.K2, S.N2 = M, 64, 256, 64
    S.X = torch.arange(M * 4, dtype=torch.int64).reshape(M, 4) + 100000 * (rank + 1)
    S.H = S.X * 3 + 5
    S.Y = S.X * 5 + 11
    for n in ("state", "rule", "p1", "p2", "ax8", "ah8", "ax4", "ah4", "w1", "w2", "sx", "sh", "sy", "cache", "ws"):
        setattr(S, n, None)
    return S


def _shard_rank(rank, world, port, M, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        fake = _FakeLib()
        T = bench.ShardedFfnStep(fake, _fake_step_state(rank, M), rank, world, lambda t: fake.gather_slots(t))
        T.step()
        out[rank] = ([t.tolist() for t in fake.finish_inputs], fake.log)
    finally:
        dist.destroy_process_group()


def test_sharded_step_gives_every_rank_the_same_whole_tensor_slots():
    """Two gloo ranks run bench.ShardedFfnStep's host sequence for one step (NVFP4 and INT8
    passes): every finish call (pre-pass of X, of the hidden tensor, the d statistic, the TDC
    record) receives, on both ranks, the slot array of the whole 2M-row tensor -- each rank's
    words in its own groups, nothing doubled from the previous pass -- and both ranks issue the
    same calls in the same order."""
    world, M = 2, 48
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_shard_rank, args=(world, _free_port(), M, out), nprocs=world, join=True,
                           start_method="spawn")
        res = dict(out)
    (f0, log0), (f1, log1) = res[0], res[1]
    assert log0 == log1 and f0 == f1
    assert log0.count("prepass_finish") == 6 and log0.count("tdc_finish") == 2
    # the expected whole-tensor slots, built directly from both ranks' rows
    fake = _FakeLib()
    exp = []
    for _pass in range(2):
        for attr, tag in (("X", 1), ("H", 1), ("Y", 4), ("Y", 9)):
            slots = fake.alloc_slots(world * M)
            for r in range(world):
                fake._partial("x", getattr(_fake_step_state(r, M), attr), r * M, slots, tag)
            exp.append(slots.tolist())
    assert f0 == exp
