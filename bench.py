"""Benchmark of the 6Bit-Diffusion hot path on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload ffn5b] [--impl ours|reference]

A step is one pass of the whole hot path over one synthetic CogVideoX-5B FFN module input
(17776 tokens x 3072 channels -> 12288 (GELU) -> 3072), run twice: all layers in NVFP4, then all
layers in INT8 (the precision forced, as the synthetic activations' outlier channels would
otherwise send every layer to the BF16 PDR path). Each pass: TDC check, precision selection,
fused pre-pass + quantization of the layer input, tcgen05 GEMM (+GELU), pre-pass + quantization of
the hidden tensor, tcgen05 GEMM, difference statistic of the module output against its input,
TDC record (delta + cache refresh). The metric is the effective tensor throughput of the step
(4 GEMMs of 2*M*N*K each / step time). Under torchrun every rank runs its own replica on its own
batch (weak scaling, no collective on the data path); time is the max over ranks.

--impl reference times the CPU oracle (the plain C reference) on the machine's host cores on a row
sample of the same step and prints the same line with "impl": "reference".
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "quantized-linear TFLOPS & fused quant GB/s (frac of B200 peak), DiT shapes"

# ncu DRAM traffic per launch (dram__bytes_read.sum + dram__bytes_write.sum, one capture of the
# step's 16 launches at full size, 17776 tokens; ncu flushes the caches before each launch, so
# these are cold-cache figures) of the kernels that can be the dominant one, summarised under
# profiles/, for the ffn5b workload at full size only. An entry is valid only for the sources it
# was measured on (sha over the listed files of csrc/).
_GEMM_SRC = ("gemm.cu", "sb_device.cuh")
_ROWS_SRC = ("prepass.cu", "rows.cuh", "prepass_blk.cuh", "sb_device.cuh", "tmap.h")
TRAFFIC = {
    "gemm_w1_int8": {"bytes": 773.8e6, "files": _GEMM_SRC, "sha": "18b7efe3b2cd2be6"},
    "gemm_w2_int8": {"bytes": 809.3e6, "files": _GEMM_SRC, "sha": "18b7efe3b2cd2be6"},
    "gemm_w1_nvfp4": {"bytes": 516.4e6, "files": _GEMM_SRC, "sha": "18b7efe3b2cd2be6"},
    "gemm_w2_nvfp4": {"bytes": 262.4e6, "files": _GEMM_SRC, "sha": "18b7efe3b2cd2be6"},
    # k_prepass_blk + k_nvfp4_blk (the encode exits at once in the INT8 pass)
    "prepass_h_nvfp4": {"bytes": 970.7e6, "files": _ROWS_SRC, "sha": "e95fb4fcaa331876"},
    "prepass_h_int8": {"bytes": 630.0e6, "files": _ROWS_SRC, "sha": "e95fb4fcaa331876"},
    "prepass_x_nvfp4": {"bytes": 225.6e6, "files": _ROWS_SRC, "sha": "e95fb4fcaa331876"},
    "prepass_x_int8": {"bytes": 127.3e6, "files": _ROWS_SRC, "sha": "e95fb4fcaa331876"},
    "record_nvfp4": {"bytes": 401.2e6, "files": _ROWS_SRC, "sha": "e95fb4fcaa331876"},
    "record_int8": {"bytes": 401.4e6, "files": _ROWS_SRC, "sha": "e95fb4fcaa331876"},
}
TRAFFIC_TOKENS = 17776


def src_sha(files):
    h = hashlib.sha256()
    for name in files:
        with open(os.path.join(ROOT, "video_diffusion_mixed_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "src": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "src": "fallback"}


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index, self.proc, self.lines = index, None, []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons, power = [], None, set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
                power.append(float(f[3]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "power_w_max": max(power) if power else None}


# ------------------------------------------------------------------------------------------------
# Multi-rank bookkeeping (replicas: every rank runs its own full step on its own batch)
# ------------------------------------------------------------------------------------------------

def max_over_ranks(ms, world, dist, device):
    """Device time of the whole job: the slowest rank's. Every rank calls it in the same order."""
    if world > 1:
        import torch
        t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    return ms


def whole_job_tflops(world, flops_per_rank_step, ms_per_step):
    """Throughput of all ranks together: each rank processed its own batch in ms_per_step."""
    return world * flops_per_rank_step / (ms_per_step * 1e-3) / 1e12


# ------------------------------------------------------------------------------------------------
# Our arm
# ------------------------------------------------------------------------------------------------

class FfnStep:
    """All buffers of one FFN module step, allocated once (the library allocates nothing)."""

    def __init__(self, sb, synth, torch, wl, seed, device, tokens=None, records_for=(), fused_record=False):
        self.sb, self.torch = sb, torch
        # precisions whose W1 GEMM also writes the hidden tensor's chunk records, which then stand
        # in for the hidden tensor's statistics pass (FFN-pair fusion)
        self.records_for = tuple(records_for)
        X, layers = synth.workload_inputs(wl, seed=seed, device=device, bias_std=0.0, tokens=tokens)
        self.X = X
        self.M, self.C = X.shape
        (self.N1, self.K1, g1), (self.N2, self.K2, g2) = [(l["N"], l["K"], l["gelu"]) for l in layers]
        self.ws = sb.Workspace(max(self.M, self.N1, self.N2), max(self.K1, self.K2))
        self.w1 = sb.Weight(layers[0]["W"], layers[0]["bias"], 128, self.ws)
        self.w2 = sb.Weight(layers[1]["W"], layers[1]["bias"], 128, self.ws)
        self.ax4, self.ax8 = sb.Fp4Tensor(self.M, self.K1), sb.I8Tensor(self.M, self.K1)
        self.ah4, self.ah8 = sb.Fp4Tensor(self.M, self.K2), sb.I8Tensor(self.M, self.K2)
        self.H = torch.empty((self.M, self.N1), dtype=torch.bfloat16, device=device)
        self.hrec = (torch.empty((self.M, self.N1 // 128, 4), dtype=torch.float32, device=device)
                     if self.records_for else None)
        self.Y = torch.empty((self.M, self.N2), dtype=torch.bfloat16, device=device)
        self.cache = torch.zeros_like(self.Y)
        # the module record computed by the W2 GEMM's epilogue (partial sums per row and 128-column
        # chunk) and folded by one more kernel, instead of a pass over the output
        self.fused_record = fused_record
        self.mrec = (torch.empty(self.M * (self.N2 // 128) * 8, dtype=torch.float32, device=device)
                     if fused_record else None)
        self.spans = KERNEL_SPANS if not fused_record else KERNEL_SPANS[:-1]
        self.state = sb.alloc_state()
        self.sx, self.sh, self.sy = sb.alloc_stats(), sb.alloc_stats(), sb.alloc_stats()
        self.p1 = torch.zeros(1, dtype=torch.int32, device=device)
        self.p2 = torch.zeros(1, dtype=torch.int32, device=device)
        self.rule = sb.Rule(1.0, 0.0, 0.1)
        self.events = None
        torch.cuda.synchronize()

    def gemm_flops(self):
        return 2.0 * self.M * (self.N1 * self.K1 + self.N2 * self.K2)

    def one_pass(self, prec, ev=None, X=None, Y=None):
        sb = self.sb
        X = self.X if X is None else X
        Y = self.Y if Y is None else Y
        cfg = sb.config(rho=64.0, tdc_thresh=-1.0, block=128, force_prec=prec)  # never skip: full work
        sb.module_decide(self.state, cfg, [self.rule, self.rule], [self.p1, self.p2])  # TDC check, both layers
        self._mark(ev, "pre1_0")
        sb.prepass(X, None, cfg, sb.PREPASS_QUANT, self.p1, self.ax4, self.ax8, self.sx, self.ws)
        self._mark(ev, "pre1_1")
        fused = prec in self.records_for
        if fused:
            sb.linear_records(X, self.ax4, self.ax8, self.p1, self.w1, self.H, self.hrec, epilogue=sb.EPI_GELU,
                              block=128, ws=self.ws)
        else:
            sb.linear(X, self.ax4, self.ax8, self.p1, self.w1, self.H, epilogue=sb.EPI_GELU, ws=self.ws)
        self._mark(ev, "gemm1_1")
        self._mark(ev, "pre2_0")
        if fused:
            sb.prepass_chunks(self.H, self.hrec, cfg, sb.PREPASS_QUANT, self.p2, self.ah4, self.ah8, self.sh, self.ws)
        else:
            sb.prepass(self.H, None, cfg, sb.PREPASS_QUANT, self.p2, self.ah4, self.ah8, self.sh, self.ws)
        self._mark(ev, "pre2_1")
        if self.fused_record:  # the W2 GEMM and the module record of its output, one span
            sb.linear_module_record(self.H, self.ah4, self.ah8, self.p2, self.w2, Y, X, self.cache, self.mrec,
                                    self.sy, self.state, self.ws)
            self._mark(ev, "gemm2_1")
        else:
            sb.linear(self.H, self.ah4, self.ah8, self.p2, self.w2, Y, ws=self.ws)
            self._mark(ev, "gemm2_1")
            # the difference statistic of Y against X and the TDC record of Y, one pass over Y
            sb.module_record(Y, X, self.cache, self.p2, self.sy, self.state, self.ws)
        self._mark(ev, "rec_1")

    def _mark(self, ev, name):
        if ev is not None:
            # external: inside a graph capture the record becomes an event node of the graph, so
            # the kernels between two marks are timed as the graph runs them
            e = self.torch.cuda.Event(enable_timing=True, external=True)
            e.record()
            ev.append((name, e))

    def step(self, ev=None, precs=None):
        for prec in precs or (self.sb.NVFP4, self.sb.INT8):
            sub = [] if ev is not None else None
            self.one_pass(prec, sub)
            if ev is not None:
                ev.append((prec, sub))


LAUNCHES_PER_PASS = 8  # decide, prepass(2), gemm, prepass(2), gemm, module record
# with the hidden tensor's chunk records, its pre-pass is 3 launches: fold, INT8 codes, NVFP4 encode


class L2Flush:
    """Empties L2 between timed steps: a 512 MiB memset (larger than the 126 MB L2), then a read
    of a 256 MiB buffer, which writes the memset's dirty lines back and leaves L2 holding clean
    lines. Without the read the first kernel of a step would pay for writing back about 126 MB of
    zeros, a cost no real step has. Both run outside the timed events."""

    def __init__(self, torch, device):
        self.w = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=device)
        self.r = torch.zeros(64 * 1024 * 1024, dtype=torch.float32, device=device)

    def __call__(self):
        self.w.zero_()
        self.r.sum()

    def zero_(self):  # the write alone (where the flush sits inside a timed span)
        self.w.zero_()


class ShardedFfnStep:
    """The FFN step with the token axis split over the ranks (sequence parallelism): each rank
    holds S.M rows of a tensor of world * S.M rows and does the row work of its rows (rotation,
    quantization, GEMMs, cache refresh); the whole-tensor statistics -- the pre-pass of X and of
    the hidden tensor (PDR ratio, NVFP4 tensor amax), the d statistic and the TDC delta -- are
    assembled from every rank's group slots by one int64 all-reduce SUM each (`gather`), after
    which every rank runs the same final reduction and gets the same statistics, decisions and
    module state as one GPU holding all rows. `gather` is sixbit.gather_slots under torchrun and
    the identity on one rank. Every rank issues the same calls in the same order."""

    def __init__(self, sb, S, rank, world, gather):
        self.sb, self.S, self.gather = sb, S, gather
        self.row0, self.Mt = rank * S.M, world * S.M
        dev = S.X.device
        self.slots = [sb.alloc_slots(self.Mt, device=dev) for _ in range(4)]

    def one_pass(self, prec):
        sb, S, g = self.sb, self.S, self.gather
        cfg = sb.config(rho=64.0, tdc_thresh=-1.0, block=128, force_prec=prec)
        for sl in self.slots:
            sl.zero_()  # every rank's copy starts zero-filled; each rank writes only its groups
        sb.module_decide(S.state, cfg, [S.rule, S.rule], [S.p1, S.p2])
        sb.prepass_partial(S.X, None, self.row0, self.Mt, cfg, sb.PREPASS_QUANT, S.p1, S.ax8, self.slots[0], S.ws)
        g(self.slots[0])
        sb.prepass_finish(self.slots[0], self.Mt, S.K1, False, cfg, sb.PREPASS_QUANT, S.p1, S.sx, S.ws)
        sb.nvfp4_encode(S.X, cfg, S.p1, S.sx, S.ax4, S.ws)
        sb.linear(S.X, S.ax4, S.ax8, S.p1, S.w1, S.H, epilogue=sb.EPI_GELU, ws=S.ws)
        sb.prepass_partial(S.H, None, self.row0, self.Mt, cfg, sb.PREPASS_QUANT, S.p2, S.ah8, self.slots[1], S.ws)
        g(self.slots[1])
        sb.prepass_finish(self.slots[1], self.Mt, S.K2, False, cfg, sb.PREPASS_QUANT, S.p2, S.sh, S.ws)
        sb.nvfp4_encode(S.H, cfg, S.p2, S.sh, S.ah4, S.ws)
        sb.linear(S.H, S.ah4, S.ah8, S.p2, S.w2, S.Y, ws=S.ws)
        sb.prepass_partial(S.Y, S.X, self.row0, self.Mt, cfg, sb.PREPASS_STATS, S.p2, None, self.slots[2], S.ws)
        g(self.slots[2])
        sb.prepass_finish(self.slots[2], self.Mt, S.N2, True, cfg, sb.PREPASS_STATS, S.p2, S.sy, S.ws)
        sb.tdc_record_partial(S.Y, S.cache, self.row0, self.Mt, S.state, self.slots[3], S.ws)
        g(self.slots[3])
        sb.tdc_finish(self.slots[3], self.Mt, S.N2, S.sy, S.state, S.ws)

    def step(self):
        for prec in (self.sb.NVFP4, self.sb.INT8):
            self.one_pass(prec)


def run_sharded(args, torch, dist, sb, S, flush, world, rank, device):
    """Times `args.steps` token-sharded steps (eager launches; the four slot gathers per pass are
    NCCL all-reduces under torchrun). Returns ms per step, the slowest rank's."""
    gather = (lambda t: sb.gather_slots(t)) if world > 1 else (lambda t: t)
    T = ShardedFfnStep(sb, S, rank, world, gather)
    for _ in range(args.warmup):
        T.step()
    torch.cuda.synchronize()
    sb.check(S.ws)
    tot = 0.0
    for _ in range(args.steps):
        flush()
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        T.step()
        e1.record()
        torch.cuda.synchronize()
        tot += e0.elapsed_time(e1)
    sb.check(S.ws)
    return max_over_ranks(tot, world, dist, device) / args.steps


KERNEL_SPANS = (("prepass_x", "pre1_0", "pre1_1"), ("gemm_w1", "pre1_1", "gemm1_1"), ("prepass_h", "pre2_0", "pre2_1"),
                ("gemm_w2", "pre2_1", "gemm2_1"), ("record", "gemm2_1", "rec_1"))


def graph_kernel_times(torch, S, flush, reps, precs):
    """Per-kernel device times inside a CUDA graph of the step: the step is captured with timing
    events between its calls (event nodes of the graph), replayed `reps` times after an L2 flush
    each, and every span's median taken. The spans tile the pass, so their sum is the graph's own
    time for the pass, with no host gaps."""
    holder = {}

    def fn():
        ev = []
        S.step(ev, precs)
        holder["ev"] = ev
    g = capture(torch, fn)
    kern = {}
    for _ in range(reps):
        flush()
        g.replay()
        torch.cuda.synchronize()
        for prec, sub in holder["ev"]:
            d = dict(sub)
            for name, a, z in S.spans:
                kern.setdefault(f"{name}_{S.sb.PREC_NAMES[prec]}", []).append(d[a].elapsed_time(d[z]))
    del g
    return {k: statistics.median(v) for k, v in kern.items()}


def capture(torch, fn):
    """A CUDA graph of the launches fn issues on the current stream (one eager call on the
    capture stream first, as graph capture wants). Replaying it runs the same kernels with the same
    arguments, without the per-launch host work."""
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn()
    torch.cuda.current_stream().wait_stream(side)
    with torch.cuda.graph(g, capture_error_mode="thread_local"):
        fn()
    torch.cuda.synchronize()
    return g


class TrajectoryStep:
    """One block-step of the decision-driven trajectory (the 30-block DiT walk at full size): the
    TDC check and both layers' precision from the rule, the pre-pass of the block input (PDR may
    switch a layer to BF16), the FFN's two GEMMs in whatever precision the device flags hold, the
    difference statistic and TDC record of the block's module output, and the residual cache:
    refreshed on a computed step, reused on a skipped one. Every call reads the decisions on the
    device, so one CUDA graph serves every step; a skipped step's kernels exit at once. The
    decisions follow the trajectory's own module output y_t (as in the parity test of the decision
    log); the FFN output is computed on x_t at every computed step."""

    def __init__(self, sb, torch, S):
        self.sb, self.torch, self.S = sb, torch, S
        dev = S.X.device
        # The block input x_t and module output y_t are copied in before every replay; they start
        # as finite data because the graph capture runs the step once eagerly on them first.
        self.Xb = S.X.clone()
        self.Yb = S.X.clone()
        self.cache = torch.zeros_like(S.X)
        self.D = torch.zeros_like(S.X)
        self.Yout = torch.empty_like(S.X)
        self.state = sb.alloc_state()
        self.sx, self.sh, self.sy = sb.alloc_stats(), sb.alloc_stats(), sb.alloc_stats()
        self.p1 = torch.zeros(1, dtype=torch.int32, device=dev)
        self.p2 = torch.zeros(1, dtype=torch.int32, device=dev)
        self.cfg = sb.config(rho=64.0, tdc_thresh=0.1, block=128, force_prec=-1)
        self.rule = sb.Rule(1.0, 0.0, 0.1)
        sb.state_init(self.state)

    def __call__(self):
        sb, S = self.sb, self.S
        sb.module_decide(self.state, self.cfg, [self.rule, self.rule], [self.p1, self.p2])
        sb.prepass(self.Xb, None, self.cfg, sb.PREPASS_QUANT, self.p1, S.ax4, S.ax8, self.sx, S.ws)
        sb.linear(self.Xb, S.ax4, S.ax8, self.p1, S.w1, S.H, epilogue=sb.EPI_GELU, ws=S.ws)
        sb.prepass(S.H, None, self.cfg, sb.PREPASS_QUANT, self.p2, S.ah4, S.ah8, self.sh, S.ws)
        sb.linear(S.H, S.ah4, S.ah8, self.p2, S.w2, S.Y, ws=S.ws)
        sb.module_record(self.Yb, self.Xb, self.cache, self.p2, self.sy, self.state, S.ws)
        sb.tdc_refresh(self.Xb, self.Yb, self.D, self.state)
        sb.tdc_reuse(self.Xb, self.D, self.Yout, self.state)


class DeltaTokensLayer:
    """The CogVideoX-2B attention projection (17776 x 1920 -> 1920) two ways: the plain NVFP4
    linear (pre-pass + NVFP4 GEMM), and with delta tokens (2 x 2 x 2 cubes of the 13 x 30 x 45
    latent grid, 226 text tokens one cube each): the split into FP8 core and bf16 delta tokens,
    the delta tokens' pre-pass, the cores' BF16 GEMM (FP32, no bias), and the delta tokens' NVFP4
    GEMM whose epilogue adds each token's core row and the bias (bf16 output)."""

    def __init__(self, sb, torch, synth, device):
        self.sb, self.torch = sb, torch
        X, layers = synth.workload_inputs("attn2b", seed=7, device=device, bias_std=0.02)
        self.X = X
        self.M, self.K = X.shape
        self.N = layers[0]["N"]
        self.c = sb.cubes(226, 13, 30, 45, 2, 2, 2)
        self.ws = sb.Workspace(self.M, self.K)
        self.w_nb = sb.Weight(layers[0]["W"], None, 128, self.ws)
        self.w_b = sb.Weight(layers[0]["W"], layers[0]["bias"], 128, self.ws)
        self.core = sb.CoreTokens(self.c, self.M, self.K)
        self.delta = torch.empty_like(X)
        self.a4, self.a8, self.st = sb.Fp4Tensor(self.M, self.K), sb.I8Tensor(self.M, self.K), sb.alloc_stats()
        self.p4 = torch.tensor([sb.NVFP4], dtype=torch.int32, device=device)
        self.pb = torch.tensor([sb.BF16], dtype=torch.int32, device=device)
        self.Yc = torch.empty((self.core.n, self.N), dtype=torch.float32, device=device)
        self.Y = torch.empty((self.M, self.N), dtype=torch.bfloat16, device=device)
        self.cfg = sb.config(force_prec=sb.NVFP4)

    def _mark(self, ev, name):
        e = self.torch.cuda.Event(enable_timing=True, external=True)
        e.record()
        ev.append((name, e))

    def plain(self, ev):
        sb = self.sb
        self._mark(ev, "p0")
        sb.prepass(self.X, None, self.cfg, sb.PREPASS_QUANT, self.p4, self.a4, self.a8, self.st, self.ws)
        self._mark(ev, "p1")
        sb.linear(self.X, self.a4, self.a8, self.p4, self.w_b, self.Y, ws=self.ws)
        self._mark(ev, "p2")

    def delta_tokens(self, ev):
        sb = self.sb
        self._mark(ev, "d0")
        sb.delta_split(self.X, self.c, self.core, self.delta)
        self._mark(ev, "d1")
        sb.prepass(self.delta, None, self.cfg, sb.PREPASS_QUANT, self.p4, self.a4, self.a8, self.st, self.ws)
        self._mark(ev, "d2")
        sb.linear(self.core.bf16, None, None, self.pb, self.w_nb, self.Yc, out_dtype=sb.OUT_F32, ws=self.ws)
        self._mark(ev, "d3")
        sb.delta_linear(self.delta, self.a4, self.a8, self.p4, self.w_b, self.Yc, self.c, self.Y, ws=self.ws)
        self._mark(ev, "d4")


def delta_accuracy(torch, sb, synth, L):
    """Output error of the 4-bit linear with and without delta tokens against the BF16 linear (our
    BF16 GEMM, FP32 output), relative Frobenius, on the timed input (independent tokens with outlier
    channels) and on tokens with a video latent's local redundancy (synth.smooth_video_tokens)."""
    out = {}
    f32 = lambda: torch.empty((L.M, L.N), dtype=torch.float32, device=L.X.device)
    Yref, Yp, Yd = f32(), f32(), f32()
    inputs = {"independent_tokens": L.X,
              "smooth_video_tokens": synth.smooth_video_tokens(226, 13, 30, 45, L.K, seed=8, device=L.X.device)}
    for name, X in inputs.items():
        sb.linear(X, None, None, L.pb, L.w_b, Yref, out_dtype=sb.OUT_F32, ws=L.ws)
        sb.prepass(X, None, L.cfg, sb.PREPASS_QUANT, L.p4, L.a4, L.a8, L.st, L.ws)
        sb.linear(X, L.a4, L.a8, L.p4, L.w_b, Yp, out_dtype=sb.OUT_F32, ws=L.ws)
        sb.delta_split(X, L.c, L.core, L.delta)
        sb.prepass(L.delta, None, L.cfg, sb.PREPASS_QUANT, L.p4, L.a4, L.a8, L.st, L.ws)
        sb.linear(L.core.bf16, None, None, L.pb, L.w_nb, L.Yc, out_dtype=sb.OUT_F32, ws=L.ws)
        sb.delta_linear(L.delta, L.a4, L.a8, L.p4, L.w_b, L.Yc, L.c, Yd, out_dtype=sb.OUT_F32, ws=L.ws)
        sb.check(L.ws)
        nref = float(torch.linalg.vector_norm(Yref.double()))
        out[name] = {"rel_err_nvfp4": round(float(torch.linalg.vector_norm((Yp - Yref).double())) / nref, 5),
                     "rel_err_delta_tokens": round(float(torch.linalg.vector_norm((Yd - Yref).double())) / nref, 5)}
    return out


def run_delta_tokens(torch, sb, synth, flush, device, reps=10):
    L = DeltaTokensLayer(sb, torch, synth, device)
    spans = {"plain_prepass": ("p0", "p1"), "plain_gemm_nvfp4": ("p1", "p2"), "split": ("d0", "d1"),
             "delta_prepass": ("d1", "d2"), "core_gemm_bf16": ("d2", "d3"), "delta_gemm_nvfp4_core_added": ("d3", "d4")}
    holder = {}

    def fn():
        ev = []
        L.plain(ev)
        L.delta_tokens(ev)
        holder["ev"] = ev
    g = capture(torch, fn)
    times = {}
    for _ in range(reps):
        flush()
        g.replay()
        torch.cuda.synchronize()
        d = dict(holder["ev"])
        for k, (a, z) in spans.items():
            times.setdefault(k, []).append(d[a].elapsed_time(d[z]))
    sb.check(L.ws)
    del g
    ms = {k: round(statistics.median(v), 4) for k, v in times.items()}
    plain = ms["plain_prepass"] + ms["plain_gemm_nvfp4"]
    dq = sum(v for k, v in ms.items() if not k.startswith("plain"))
    flops = 2.0 * L.M * L.N * L.K
    return {"what": "CogVideoX-2B attention projection (17776 x 1920 -> 1920): the plain NVFP4 linear against the "
                    "delta-token linear (2x2x2 cubes of the 13x30x45 latent grid + 226 text tokens: FP8 cores, "
                    "4-bit deltas), one graph of both, L2 flushed before each replay",
            "cubes": L.core.n, "ms": ms, "ms_plain": round(plain, 4), "ms_delta_tokens": round(dq, 4),
            "tflops_plain": round(flops / (plain * 1e-3) / 1e12, 1),
            "tflops_delta_tokens": round(flops / (dq * 1e-3) / 1e12, 1),
            "accuracy_vs_bf16": delta_accuracy(torch, sb, synth, L)}


def run_residual_cache(torch, sb, S, flush, reps=10):
    """The Temporal Delta Cache's residual on the module's block (17776 x 3072 at full size): the
    refresh of a computed step and the reuse of a skipped one, with the residual in bf16 and in
    FP8 (E4M3 codes + one FP32 scale per token). Each call is timed alone after an L2 flush."""
    M, C = S.X.shape
    x = S.X
    y = S.X.clone()
    y.add_(0.125)
    out = torch.empty_like(x)
    d16 = torch.empty_like(x)
    d8 = sb.Fp8Residual(M, C)
    st_c, st_s = sb.alloc_state(), sb.alloc_state()
    sb.state_init(st_c)
    sb.state_init(st_s)
    st_s.view(torch.int32)[9] = 1  # sb_module_state.skip (bytes 36..39): the reuse calls run
    calls = {"refresh_bf16": lambda: sb.tdc_refresh(x, y, d16, st_c), "reuse_bf16": lambda: sb.tdc_reuse(x, d16, out, st_s),
             "refresh_fp8": lambda: sb.tdc_refresh_fp8(x, y, d8, st_c), "reuse_fp8": lambda: sb.tdc_reuse_fp8(x, d8, out, st_s)}
    nbytes = {"refresh_bf16": 6 * M * C, "reuse_bf16": 6 * M * C, "refresh_fp8": 5 * M * C + 4 * M, "reuse_fp8": 5 * M * C + 4 * M}
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    res = {}
    for k, fn in calls.items():
        fn()
        ts = []
        for _ in range(reps):
            flush()
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        ms = statistics.median(ts)
        res[k] = {"ms": round(ms, 4), "achieved_gbs": round(nbytes[k] / (ms * 1e-3) / 1e9, 1)}
    return {"what": f"TDC residual cache on the block input ({M} x {C}): refresh (computed step) and reuse (skipped "
                    "step), residual in bf16 or FP8 (E4M3 + FP32 scale per token); algorithmic bytes: bf16 6 B/el, "
                    "FP8 5 B/el + 4 B/token; one call per L2 flush", **res}


def run_trajectory(torch, sb, synth, S, flush, blocks, steps=50):
    """Times the decision-driven path: `blocks` of the 30-block trajectory, `steps` steps each, at
    the module's full token count. Inputs are drawn outside the timed events; each block-step is
    one graph replay after an L2 flush."""
    T = TrajectoryStep(sb, torch, S)
    g = capture(torch, T)
    sb.check(S.ws)
    names = {sb.NVFP4: "nvfp4", sb.INT8: "int8", sb.BF16: "bf16", sb.SKIP: "skip"}
    counts = {f"w{i}_{n}": 0 for i in (1, 2) for n in names.values()}
    by_kind, total, flops = {}, 0.0, 0.0
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for k in blocks:
        traj = synth.Trajectory(S.M, S.K1, k, blocks=30, steps=steps, seed=0, device=S.X.device)
        sb.state_init(T.state)
        T.cache.zero_()
        for t in range(steps):
            x, y = traj.current()
            T.Xb.copy_(x)
            T.Yb.copy_(y)
            flush()
            e0.record()
            g.replay()
            e1.record()
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1)
            p1, p2 = int(T.p1.item()), int(T.p2.item())
            counts[f"w1_{names[p1]}"] += 1
            counts[f"w2_{names[p2]}"] += 1
            key = names[p1] if p1 == p2 else f"{names[p1]}+{names[p2]}"
            by_kind.setdefault(key, []).append(ms)
            total += ms
            flops += (0.0 if p1 == sb.SKIP else 2.0 * S.M * S.N1 * S.K1) + \
                     (0.0 if p2 == sb.SKIP else 2.0 * S.M * S.N2 * S.K2)
            if t + 1 < steps:
                traj.advance()
    sb.check(S.ws)
    del g
    n = len(blocks) * steps
    return {"what": "decision-driven FFN block-steps of the 30-block trajectory (hidden 3072, FFN 12288, "
                    f"{S.M} tokens, rho 64, rule 1*d+0 > 0.1 -> INT8, TDC threshold 0.1): TDC check + rule, "
                    "pre-passes, GEMMs of the chosen kind, difference and TDC record, residual-cache "
                    "refresh / reuse; one graph replay per block-step, L2 flushed before each",
            "blocks": list(blocks), "steps": steps, "block_steps": n, "ms_total": round(total, 3),
            "ms_per_block_step": round(total / n, 4), "gemm_tflops_effective": round(flops / (total * 1e-3) / 1e12, 1),
            "decisions": counts,
            "ms_per_block_step_by_decision": {k: round(statistics.mean(v), 4) for k, v in sorted(by_kind.items())},
            "block_steps_by_decision": {k: len(v) for k, v in sorted(by_kind.items())}}


def run_e2e(torch, sb, S, flush, steps, barrier, with_outputs):
    """The end-to-end leg (see run_ours). Returns (ms for `steps` steps, H2D bytes per step, D2H
    bytes per step)."""
    comp = torch.cuda.current_stream()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    Xh = torch.empty(S.X.shape, dtype=S.X.dtype, pin_memory=True)
    Xh.copy_(S.X.cpu())
    Xd = [S.X, S.X.clone()]  # finite from the start: capturing a pass runs it once eagerly
    Yd = [S.Y, torch.empty_like(S.Y)]
    # per pass: the output tensor (with_outputs) or the statistics records and module state
    recs = [S.sx, S.sh, S.sy, S.state]
    Rh = [[torch.empty(r.shape, dtype=r.dtype, pin_memory=True) for r in recs] for _ in range(2)]
    Yh = [torch.empty(S.Y.shape, dtype=S.Y.dtype, pin_memory=True) for _ in range(2)] if with_outputs else None
    ev = lambda: torch.cuda.Event(enable_timing=False)
    x_free = [None, None]      # compute finished with Xd[b]
    y_free = [None, None]      # download finished with pass p's results
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # one graph per (pass, input buffer); pass p always writes Yd[p]
    g_pass = {(p, b): capture(torch, lambda prec=prec, b=b, p=p: S.one_pass(prec, X=Xd[b], Y=Yd[p]))
              for p, prec in enumerate((sb.NVFP4, sb.INT8)) for b in range(2)}
    sb.check(S.ws)
    torch.cuda.synchronize()
    barrier()
    for i in range(steps):
        b = i % 2
        with torch.cuda.stream(up):
            if i == 0:
                t0.record()
            if x_free[b] is not None:
                up.wait_event(x_free[b])
            Xd[b].copy_(Xh, non_blocking=True)
            x_ready = ev()
            x_ready.record()
        comp.wait_event(x_ready)
        flush.zero_()
        for p, prec in enumerate((sb.NVFP4, sb.INT8)):
            if y_free[p] is not None:
                comp.wait_event(y_free[p])
            g_pass[(p, b)].replay()
            y_ready = ev()
            y_ready.record()
            with torch.cuda.stream(down):
                down.wait_event(y_ready)
                if with_outputs:
                    Yh[p].copy_(Yd[p], non_blocking=True)
                for r, h in zip(recs, Rh[p]):
                    h.copy_(r, non_blocking=True)
                y_free[p] = ev()
                y_free[p].record()
        x_free[b] = ev()
        x_free[b].record()
    with torch.cuda.stream(down):
        down.wait_event(x_free[(steps - 1) % 2])
        t1.record()
    torch.cuda.synchronize()
    barrier()
    del g_pass
    h2d = S.X.numel() * S.X.element_size()
    d2h = 2 * sum(r.numel() * r.element_size() for r in recs)
    if with_outputs:
        d2h += 2 * S.Y.numel() * S.Y.element_size()
    return t0.elapsed_time(t1), h2d, d2h


def run_ours(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    device = f"cuda:{local}"
    torch.cuda.set_device(local)
    from video_diffusion_mixed_b200 import build as b
    b.build()
    from video_diffusion_mixed_b200 import sixbit as sb
    from video_diffusion_mixed_b200 import synth

    records_for = {"none": (), "nvfp4": (sb.NVFP4,), "both": (sb.NVFP4, sb.INT8)}[args.ffn_records]
    S = FfnStep(sb, synth, torch, args.workload, seed=rank, device=device, tokens=args.tokens,
                records_for=records_for, fused_record=(args.module_record == "fused"))
    flush = L2Flush(torch, device)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        S.step()
    sb.check(S.ws)
    barrier()

    # ---- timed: K steps, each one replay of the step's CUDA graph; an L2 flush before each step,
    # excluded by per-step events
    g_step = capture(torch, S.step)
    sb.check(S.ws)
    clk = ClockSampler(local)
    clk.start()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier()
    t_wall0 = time.perf_counter()
    for i in range(args.steps):
        flush()
        starts[i].record()
        g_step.replay()
        ends[i].record()
    barrier()
    t_wall = time.perf_counter() - t_wall0
    clocks = clk.stop()
    sb.check(S.ws)
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = max_over_ranks(sum(step_ms), world, dist, device)
    ms_per_step = total_ms / args.steps
    flops = 2 * S.gemm_flops()  # both precision passes
    value = whole_job_tflops(world, flops, ms_per_step)

    # ---- per-kernel breakdown: a graph of the same step with timing events between its calls
    reps = max(5, min(args.steps, 20))
    kern_ms = graph_kernel_times(torch, S, flush, reps, None)
    # ---- the BF16 fallback (the Purified Delta Refresh path) forced on the same module, reported
    # beside the headline step (not part of it)
    bf16_ms = graph_kernel_times(torch, S, flush, reps, (sb.BF16,))
    sb.check(S.ws)
    # ---- what the quantized passes cost in accuracy: the module output of each pass against the
    # BF16 pass on the same input (relative Frobenius; bf16 outputs)
    outs = {}
    for prec in (sb.BF16, sb.NVFP4, sb.INT8):
        S.one_pass(prec)
        outs[prec] = S.Y.double()
    sb.check(S.ws)
    ref_norm = float(torch.linalg.vector_norm(outs[sb.BF16]))
    accuracy = {sb.PREC_NAMES[p]: round(float(torch.linalg.vector_norm(outs[p] - outs[sb.BF16])) / ref_norm, 5)
                for p in (sb.NVFP4, sb.INT8)}
    # the same passes with weights and activations rotated by smaller or larger Hadamard blocks
    by_block = {"nvfp4": {}, "int8": {}}
    for B in (16, 64, 128, 256):
        w1 = sb.Weight(S.w1.W, S.w1.bias, B, S.ws)
        w2 = sb.Weight(S.w2.W, S.w2.bias, B, S.ws)
        for prec in (sb.NVFP4, sb.INT8):
            cfg = sb.config(rho=64.0, tdc_thresh=-1.0, block=B, force_prec=prec)  # no PDR switch
            S.p1.fill_(prec)
            S.p2.fill_(prec)
            sb.prepass(S.X, None, cfg, sb.PREPASS_QUANT, S.p1, S.ax4, S.ax8, S.sx, S.ws)
            sb.linear(S.X, S.ax4, S.ax8, S.p1, w1, S.H, epilogue=sb.EPI_GELU, ws=S.ws)
            sb.prepass(S.H, None, cfg, sb.PREPASS_QUANT, S.p2, S.ah4, S.ah8, S.sh, S.ws)
            sb.linear(S.H, S.ah4, S.ah8, S.p2, w2, S.Y, ws=S.ws)
            sb.check(S.ws)
            by_block[sb.PREC_NAMES[prec]][B] = round(
                float(torch.linalg.vector_norm(S.Y.double() - outs[sb.BF16])) / ref_norm, 5)
        del w1, w2
    accuracy["by_hadamard_block"] = by_block
    del outs

    # ---- the token-sharded step (the tensor's rows split over the ranks; statistics gathered)
    sharded = None
    if args.shard == "tokens":
        sms = run_sharded(args, torch, dist, sb, S, flush, world, rank, device)
        sharded = {"what": f"token-sharded step: {world} ranks x {S.M} rows of one {world * S.M}-row tensor per "
                           "layer; row work local, whole-tensor statistics from one int64 all-reduce SUM of group "
                           "slots each (4 per pass); eager launches",
                   "ms_per_step": round(sms, 4), "value": round(whole_job_tflops(world, 2 * S.gemm_flops(), sms), 2),
                   "unit": "TFLOPS", "scaling": "weak"}

    # ---- delta tokens on the attention projection, beside the plain NVFP4 linear
    delta_tok = run_delta_tokens(torch, sb, synth, flush, device) if not args.no_delta_tokens else None

    # ---- the residual cache of the reuse path, bf16 and FP8
    resid = run_residual_cache(torch, sb, S, flush)

    # ---- the decision-driven path (rule, restart, PDR and skips live) on the trajectory
    traj = run_trajectory(torch, sb, synth, S, flush, args.traj_blocks) if args.traj_blocks else None

    # ---- end to end through the public API with host buffers: every step uploads its X from
    # pinned host memory and reads back, per pass, the step's result: the module's statistics
    # records and decision state (what the host sees of a module step; its output tensor feeds the
    # next module on the device). A second leg also downloads both passes' output tensors (218 MB
    # a step at full size, bound by the host link). A deployment pipelines the transfers: the
    # upload of step i + 1 (copy stream U) and each pass's download (copy stream D) overlap the
    # compute of the neighbouring passes on the compute stream, through double-buffered device
    # inputs (and outputs) ordered by events. The timed span runs from the first upload to the last
    # download; the L2 flush stays inside it on the compute stream.
    e2e_ms, h2d, d2h = run_e2e(torch, sb, S, flush, args.steps, barrier, with_outputs=False)
    e2e_ms = max_over_ranks(e2e_ms, world, dist, device)
    e2e_value = whole_job_tflops(world, flops, e2e_ms / args.steps)
    e2eo_ms, _, d2ho = run_e2e(torch, sb, S, flush, args.steps, barrier, with_outputs=True)
    e2eo_ms = max_over_ranks(e2eo_ms, world, dist, device)
    e2eo_value = whole_job_tflops(world, flops, e2eo_ms / args.steps)

    # ---- roofline of the dominant kernel and of the fused pre-pass
    pk = peaks()
    ratio = {"nvfp4": 4.0, "int8": 2.0, "bf16": 1.0}  # nominal dense ratio to bf16 (9 / 4.5 / 2.25 PFLOP/s)
    # The burst bf16 figure applies while the SM clock stays near its maximum during the timed
    # region; the sustained (power-capped) one otherwise.
    burst = bool(clocks.get("sm_mhz") and clocks.get("sm_max_mhz") and clocks["sm_mhz"] >= 0.95 * clocks["sm_max_mhz"])
    tensor_peak = pk["bf16_tflops"] if burst else pk["bf16_tflops_sustained"]
    M, K1, N1, K2, N2 = S.M, S.K1, S.N1, S.K2, S.N2
    gemm_flops = {"gemm_w1": 2.0 * M * N1 * K1, "gemm_w2": 2.0 * M * N2 * K2}
    def roof_rows(kms):
        out = []
        for k, ms in kms.items():
            base, tag = k.rsplit("_", 1)
            if base in gemm_flops:
                ach = gemm_flops[base] / (ms * 1e-3) / 1e12
                peak = tensor_peak * ratio[tag]
                out.append({"kernel": k, "bound": "tensor", "ms": ms, "achieved": ach, "peak": peak,
                            "unit": "TFLOP/s", "frac": ach / peak})
            else:
                Kx = {"prepass_x": K1, "prepass_h": K2, "record": N2}[base]
                el = M * Kx
                if base in ("prepass_x", "prepass_h"):
                    # algorithmic bytes: read bf16 X, write the quantized form of the chosen precision
                    # (nothing under BF16: the pre-pass then only gathers the statistics)
                    byt = el * 2 + {"int8": el * 1 + M * 4, "nvfp4": el * (0.5 + 1 / 16) + 4, "bf16": 0}[tag]
                else:
                    byt = el * 8  # record: read y, x and the cache, refresh the cache
                ach = byt / (ms * 1e-3) / 1e9
                out.append({"kernel": k, "bound": "hbm", "ms": ms, "achieved": ach, "peak": pk["hbm_gbs"],
                            "unit": "GB/s", "frac": ach / pk["hbm_gbs"]})
        return out

    rows = roof_rows(kern_ms)
    rows_bf16 = roof_rows(bf16_ms)
    dom = max(rows, key=lambda r: r["ms"])

    def traffic_of(kernel):  # measured DRAM bytes per launch, while the sources are the measured ones
        tr = TRAFFIC.get(kernel)
        ok = tr is not None and args.workload == "ffn5b" and M == TRAFFIC_TOKENS and src_sha(tr["files"]) == tr["sha"]
        return int(tr["bytes"]) if ok else None

    traffic = traffic_of(dom["kernel"])
    roofline = {"bound": dom["bound"], "achieved": round(dom["achieved"], 1), "peak": round(dom["peak"], 1),
                "unit": dom["unit"], "frac": round(dom["frac"], 4), "traffic": traffic, "kernel": dom["kernel"],
                "peak_src": f"{pk['src']} bf16 {'burst' if burst else 'sustained'} x nominal dtype ratio"
                if dom["bound"] == "tensor"
                else f"{pk['src']} HBM copy"}
    pre = [r for r in rows if r["kernel"].startswith("prepass")]
    launches_per_step = 2 * LAUNCHES_PER_PASS + len(S.records_for)
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOPS", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "nvfp4+int8 (fp32 accumulate), bf16 activations", "data": "synthetic",
        "config": {"workload": f"{args.workload}: CogVideoX-5B FFN, X [{M} x {K1}] bf16 (0.5% outlier channels x50) "
                               f"-> W1 [{N1} x {K1}] (GELU) -> W2 [{N2} x {K2}]; NVFP4 pass + INT8 pass per step",
                   "tokens": M, "hidden": K1, "ffn": N1, "hadamard_block": 128, "parallelism": f"replicas x{world}",
                   "l2": "flushed before every step (512 MiB memset, then a 256 MiB read that leaves L2 clean; "
                         "outside the per-step events)",
                   "ffn_records": args.ffn_records,
                   "module_record": args.module_record,
                   "launch": f"each step replays one CUDA graph of its {launches_per_step} kernels"},
        "roofline": roofline,
        "roofline_prepass": {r["kernel"]: {"achieved_gbs": round(r["achieved"], 1), "frac": round(r["frac"], 4),
                                           "ms": round(r["ms"], 4), "traffic": traffic_of(r["kernel"])} for r in pre},
        "kernels": {r["kernel"]: {"ms": round(r["ms"], 4), "achieved": round(r["achieved"], 1), "unit": r["unit"],
                                  "frac": round(r["frac"], 4), "traffic": traffic_of(r["kernel"])} for r in rows},
        "kernels_timing": "event nodes inside a CUDA graph of the step (median of the replays, L2 flushed "
                          "before each); the spans tile the step",
        "trajectory": traj,
        "sharded": sharded,
        "delta_tokens": delta_tok,
        "residual_cache": resid,
        "accuracy_vs_bf16": {"what": "relative Frobenius error of the module output of each pass against the "
                                     "BF16 pass on the same input (block Hadamard B = 128, bf16 outputs)", **accuracy},
        "bf16_pass": {"what": "the same module with every layer forced to the BF16 fallback (the Purified Delta "
                              "Refresh path), timed like the kernels above; not part of the headline step",
                      "ms": round(sum(bf16_ms.values()), 4),
                      "kernels": {r["kernel"]: {"ms": round(r["ms"], 4), "achieved": round(r["achieved"], 1),
                                                "unit": r["unit"], "frac": round(r["frac"], 4)} for r in rows_bf16}},
        "e2e": {"value": round(e2e_value, 2), "unit": "TFLOPS", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "result": "per pass the statistics records (pre-pass of X, of the hidden tensor, d of the output) and "
                          "the module state"},
        "e2e_with_outputs": {"value": round(e2eo_value, 2), "unit": "TFLOPS", "h2d_bytes_per_step": h2d,
                             "d2h_bytes_per_step": d2ho, "result": "also both passes' output tensors"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
        "wall_s_timed": round(t_wall, 3),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args, S.X, S.w1.W, S.w2.W)
    del g_step  # the graphs hold no collectives; released before the process group anyway
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------------------------
# The oracle on host cores (cpu_baseline leg and the reference arm)
# ------------------------------------------------------------------------------------------------

_WP = {}


def oracle_weights(W1_u16, W2_u16, B=128):
    """Offline weight preparation by the oracle (rotation, NVFP4 and INT8 copies), cached."""
    import oracle
    key = (W1_u16.ctypes.data, W2_u16.ctypes.data, B)
    if key not in _WP:
        _WP[key] = (oracle.prepare_weight(W1_u16, B), oracle.prepare_weight(W2_u16, B))
    return _WP[key]


def oracle_sample_step(X_u16, W1_u16, W2_u16, rows, B=128):
    """The oracle's version of one step restricted to `rows` tokens: pre-pass + quantization of
    the sampled X rows, W1 GEMM (+GELU) in NVFP4 and in INT8, bf16 rounding of the hidden rows,
    their pre-pass + quantization, W2 GEMM. Weight preparation is offline (not timed).
    Returns the GEMM FLOPs it performed and the seconds it took."""
    import numpy as np
    import oracle
    xs = np.ascontiguousarray(X_u16[rows])
    n = len(rows)
    flops = 0.0
    wp1, wp2 = oracle_weights(W1_u16, W2_u16, B)
    t0 = time.perf_counter()
    st = oracle.prepass(xs, None, B)
    q8, s8 = oracle.quant_int8(st["y"], st["row_amax"])
    c4, sf, _, sg = oracle.quant_nvfp4(st["y"], st["amax_rot"])
    for prec in ("nvfp4", "int8"):
        if prec == "nvfp4":
            h = oracle.gemm_nvfp4(c4, sf, sg, wp1["c4"], wp1["sf4"], wp1["sg4"], None, W1_u16.shape[1], B, gelu=True)
        else:
            h = oracle.gemm_int8(q8, s8, wp1["q8"], wp1["s8"], None, B, gelu=True)
        hb = oracle.f32_to_bf16(h.astype(np.float32))
        sh = oracle.prepass(hb, None, B)
        if prec == "nvfp4":
            c, f, _, g = oracle.quant_nvfp4(sh["y"], sh["amax_rot"])
            oracle.gemm_nvfp4(c, f, g, wp2["c4"], wp2["sf4"], wp2["sg4"], None, W2_u16.shape[1], B)
        else:
            q, s = oracle.quant_int8(sh["y"], sh["row_amax"])
            oracle.gemm_int8(q, s, wp2["q8"], wp2["s8"], None, B)
        flops += 2.0 * n * (W1_u16.shape[0] * W1_u16.shape[1] + W2_u16.shape[0] * W2_u16.shape[1])
    return flops, time.perf_counter() - t0


def _u16(t):
    import numpy as np
    import torch
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def cpu_baseline(args, X, W1, W2):
    import numpy as np
    M = X.shape[0]
    rows = np.linspace(0, M - 1, args.cpu_baseline_rows).round().astype(np.int64)
    flops, secs = oracle_sample_step(_u16(X), _u16(W1), _u16(W2), rows)
    return {"value": round(flops / secs / 1e12, 6), "unit": "TFLOPS", "cores": os.cpu_count(), "kind": "oracle",
            "sample": f"{len(rows)} of {M} tokens (evenly spaced), both precision passes of the step; "
                      f"{secs:.1f} s; weight preparation untimed"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    import numpy as np
    import torch
    from video_diffusion_mixed_b200 import synth
    import oracle
    oracle.build()
    X, layers = synth.workload_inputs(args.workload, seed=0, device="cpu", bias_std=0.0)
    Xu, W1u, W2u = _u16(X), _u16(layers[0]["W"]), _u16(layers[1]["W"])
    M = X.shape[0]
    rows = np.linspace(0, M - 1, args.cpu_rows).round().astype(np.int64)
    for _ in range(args.warmup if args.warmup < 1 else 1):
        oracle_sample_step(Xu, W1u, W2u, rows[:2])
    tot_f, tot_s = 0.0, 0.0
    for _ in range(args.steps):
        f, s = oracle_sample_step(Xu, W1u, W2u, rows)
        tot_f += f
        tot_s += s
    value = tot_f / tot_s / 1e12
    full_flops = 2 * 2.0 * M * (layers[0]["N"] * layers[0]["K"] + layers[1]["N"] * layers[1]["K"])
    line = {
        "metric": METRIC, "impl": "reference", "value": round(value, 6), "unit": "TFLOPS", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(full_flops / (value * 1e12) * 1e3, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle)",
        "data": "synthetic",
        "config": {"workload": f"{args.workload}: CogVideoX-5B FFN (same as our arm), row sample",
                   "tokens": M, "parallelism": "host cores (OpenMP)"},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOPS", "cores": os.cpu_count(), "kind": "oracle",
                         "sample": f"{len(rows)} of {M} tokens per step, both precision passes"},
        "e2e": {"value": round(value, 6), "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="ffn5b", choices=["ffn5b", "ffn2b"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-rows", type=int, default=32, help="tokens per step of the reference arm's sample")
    ap.add_argument("--cpu-baseline-rows", type=int, default=1024,
                    help="tokens in the cpu_baseline sample of our arm (about 10 s on 16 cores)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-delta-tokens", action="store_true", help="skip the delta-token layer timing")
    ap.add_argument("--module-record", default="separate", choices=["fused", "separate"],
                    help="the module record in the W2 GEMM's epilogue + a fold kernel, or its own pass")
    ap.add_argument("--ffn-records", default="none", choices=["none", "nvfp4", "both"],
                    help="passes whose W1 GEMM writes the hidden tensor's chunk records for its pre-pass")
    ap.add_argument("--shard", default="none", choices=["none", "tokens"],
                    help="also time the token-sharded step (under torchrun: the rows of every tensor split "
                         "over the ranks, statistics gathered with NCCL)")
    ap.add_argument("--traj-blocks", type=lambda v: [int(x) for x in v.split(",") if x != ""], default=[0, 7, 14, 29],
                    help="blocks of the 30-block trajectory timed on the decision-driven path ('' to skip)")
    ap.add_argument("--tokens", type=int, default=None,
                    help="override the token count (small profiling case; the bench line is then not the metric)")
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "ours":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
