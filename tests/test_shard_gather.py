"""Token sharding on the host: two gloo ranks on CPU gather their slot arrays.

Each rank writes the group slots of its own rows into a zero-filled copy of the whole tensor's
slot array; one int64 all-reduce SUM (sixbit.gather_slots) must give both ranks every rank's words
bit for bit, whatever the words hold (FP64 partial sums, FP32 maxima, flags, NaN or infinity
patterns). The device side of sharding -- shards written by sb_prepass_partial and folded by
sb_prepass_finish -- is covered by tests/test_gpu_shard.py on one GPU.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

SLOT_WORDS = 6  # 48-byte slot = 6 int64 words


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _expected(M_total, seed=7):
    groups = -(-M_total // 16)
    rng = np.random.default_rng(seed)
    words = rng.integers(np.iinfo(np.int64).min, np.iinfo(np.int64).max, size=groups * SLOT_WORDS,
                         dtype=np.int64, endpoint=True)
    # a few slot words holding non-finite FP64 / FP32 patterns must survive too
    special = np.array([np.inf, -np.inf, np.nan], dtype=np.float64).view(np.int64)
    words[:3] = special
    words[3] = np.array([np.float32(np.nan), np.float32(np.inf)], dtype=np.float32).view(np.int64)[0]
    return words


def _rank(rank, world, port, M_total, bounds, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as dist
    from video_diffusion_mixed_b200 import sixbit as sb
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        full = torch.from_numpy(_expected(M_total))
        slots = torch.zeros_like(full)
        r0, r1 = bounds[rank]
        g0, g1 = r0 // 16, -(-r1 // 16)
        slots[g0 * SLOT_WORDS:g1 * SLOT_WORDS] = full[g0 * SLOT_WORDS:g1 * SLOT_WORDS]
        sb.gather_slots(slots)
        out[rank] = bool(torch.equal(slots, full))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("M_total,cut", [(17776, 8896), (50, 32), (16, 16)])
def test_two_ranks_gather_slots_bit_for_bit(M_total, cut):
    world = 2
    bounds = [(0, cut), (cut, M_total)]
    port = _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    procs = [ctx.Process(target=_rank, args=(r, world, port, M_total, bounds, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0] and out[1]
