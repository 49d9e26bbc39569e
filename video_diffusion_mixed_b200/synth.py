"""Seeded synthetic inputs with the shapes and value distributions of DiT linear layers.

This module only draws random numbers (torch.Generator, fixed seeds) and lays them out; it holds
none of the method's arithmetic. Tests feed the same bytes to the CUDA path and to the CPU
oracle; ``bench.py`` draws its timed inputs here.

Workloads (CogVideoX-shaped; the models, weights and prompt suites themselves are not used):
  tiny      X [256 x 256] ~N(0,1), 4 fixed channels x20; W [256 x 256] ~N(0, 0.02)
  attn2b    X [17776 x 1920] ~N(0,1), 1% channels replaced by 30 * Student-t(3); W [1920 x 1920]
  ffn2b     X [17776 x 1920] -> W1 [7680 x 1920] (GELU) -> W2 [1920 x 7680]
  ffn5b     X [17776 x 3072], 0.5% channels x50; W1 [12288 x 3072], W2 [3072 x 12288]
  traj5b    30 blocks x 50 steps, hidden 3072, random walk x_t = x_{t-1} + sigma_t N(0,1)
Weights are stored [N_out x K_in] (row = output channel), activations [tokens x channels].
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch

TOKENS = 17776  # 49 frames of CogVideoX latent tokens (13 x 60 x 90 / 4 + 226 text tokens)


def sub_seed(seed: int, tensor_id: int, block: int = 0, step: int = 0) -> int:
    return (seed * 1000003 + tensor_id * 4099 + block * 131 + step) & 0x7FFFFFFFFFFFFFFF


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def outlier_channels(K: int, n: int, seed: int, device="cpu") -> torch.Tensor:
    """n distinct channel indices drawn by randperm (recorded by callers)."""
    g = _gen("cpu", seed)
    return torch.randperm(K, generator=g)[:n].to(device)


def student_t3(shape, g, device) -> torch.Tensor:
    """Student-t with 3 degrees of freedom: z / sqrt(chi2_3 / 3), built from normals only."""
    z = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    c = torch.randn((3,) + tuple(shape), generator=g, device=device, dtype=torch.float32)
    chi2 = (c * c).sum(0)
    return z / torch.sqrt(chi2 / 3.0)


def activations(M: int, K: int, *, n_outlier: int = 0, scale: float = 1.0, student: bool = False,
                seed: int = 0, tensor_id: int = 0, device="cpu", channels=None) -> torch.Tensor:
    """X [M x K] bf16 ~ N(0,1); outlier channels multiplied by ``scale`` (or replaced by
    scale * Student-t(3) values when ``student``)."""
    g = _gen(device, sub_seed(seed, tensor_id))
    x = torch.randn((M, K), generator=g, device=device, dtype=torch.float32)
    if n_outlier > 0 or channels is not None:
        ch = channels if channels is not None else outlier_channels(K, n_outlier, sub_seed(seed, tensor_id, 1), device)
        ch = ch.to(device)
        if student:
            x[:, ch] = scale * student_t3((M, ch.numel()), g, device)
        else:
            x[:, ch] = x[:, ch] * scale
    return x.to(torch.bfloat16)


def weight(N: int, K: int, *, std: float = 0.02, seed: int = 0, tensor_id: int = 100, device="cpu") -> torch.Tensor:
    g = _gen(device, sub_seed(seed, tensor_id))
    return (torch.randn((N, K), generator=g, device=device, dtype=torch.float32) * std).to(torch.bfloat16)


def bias(N: int, *, std: float = 0.02, seed: int = 0, tensor_id: int = 200, device="cpu") -> torch.Tensor:
    if std == 0.0:
        return torch.zeros(N, device=device, dtype=torch.bfloat16)
    g = _gen(device, sub_seed(seed, tensor_id))
    return (torch.randn((N,), generator=g, device=device, dtype=torch.float32) * std).to(torch.bfloat16)


def noisy_copy(x: torch.Tensor, rel: float, *, seed: int = 0, tensor_id: int = 300) -> torch.Tensor:
    """x + rel * rms(x) * N(0,1) (a synthetic "module output" whose difference to x is ~rel)."""
    g = _gen(x.device, sub_seed(seed, tensor_id))
    xf = x.float()
    rms = torch.sqrt(torch.mean(xf * xf))
    return (xf + rel * rms * torch.randn(x.shape, generator=g, device=x.device, dtype=torch.float32)).to(torch.bfloat16)


@dataclass
class Workload:
    name: str
    M: int
    K: int
    n_outlier: int
    scale: float
    student: bool
    layers: tuple  # ((N, K, gelu), ...) applied in sequence


WORKLOADS = {
    "tiny": Workload("tiny", 256, 256, 4, 20.0, False, ((256, 256, False),)),
    "attn2b": Workload("attn2b", TOKENS, 1920, 19, 30.0, True, ((1920, 1920, False),)),
    "ffn2b": Workload("ffn2b", TOKENS, 1920, 19, 30.0, True, ((7680, 1920, True), (1920, 7680, False))),
    "ffn5b": Workload("ffn5b", TOKENS, 3072, 15, 50.0, False, ((12288, 3072, True), (3072, 12288, False))),
}


def smooth_video_tokens(text: int, F: int, H: int, W: int, K: int, *, noise: float = 0.1, waves: int = 4,
                        seed: int = 0, tensor_id: int = 500, device="cpu") -> torch.Tensor:
    """Tokens with the local redundancy of a video latent, bf16 [text + F H W, K]: `text` tokens
    N(0, 1), then the F x H x W grid in (f, h, w) order, each channel a sum of `waves` sinusoids of
    low frequency (up to one period along each axis, random phase), scaled to unit variance, plus
    N(0, noise^2): neighbouring grid tokens differ by a small fraction of their magnitude."""
    g = _gen(device, sub_seed(seed, tensor_id))
    n = F * H * W
    f = torch.arange(F, device=device, dtype=torch.float32).repeat_interleave(H * W) / F
    h = torch.arange(H, device=device, dtype=torch.float32).repeat_interleave(W).repeat(F) / H
    w = torch.arange(W, device=device, dtype=torch.float32).repeat(F * H) / W
    coords = torch.stack([f, h, w], dim=1)  # [n, 3]
    field = torch.zeros((n, K), device=device, dtype=torch.float32)
    for _ in range(waves):
        freq = torch.rand((3, K), generator=g, device=device)  # up to one period along each axis
        phase = torch.rand((1, K), generator=g, device=device) * (2 * math.pi)
        field += torch.cos(2 * math.pi * (coords @ freq) + phase)
    field *= math.sqrt(2.0 / waves)
    field += noise * torch.randn((n, K), generator=g, device=device)
    txt = torch.randn((text, K), generator=g, device=device)
    return torch.cat([txt, field], dim=0).to(torch.bfloat16)


def workload_inputs(name: str, *, seed: int = 0, device="cpu", tokens: int | None = None, bias_std: float = 0.0):
    """Activations, weights and biases of one named workload."""
    w = WORKLOADS[name]
    M = tokens or w.M
    x = activations(M, w.K, n_outlier=w.n_outlier, scale=w.scale, student=w.student, seed=seed,
                    tensor_id=0, device=device)
    layers = []
    for i, (N, K, gelu) in enumerate(w.layers):
        layers.append({"W": weight(N, K, seed=seed, tensor_id=100 + i, device=device),
                       "bias": bias(N, std=bias_std, seed=seed, tensor_id=200 + i, device=device),
                       "N": N, "K": K, "gelu": gelu})
    return x, layers


# ------------------------------------------------------------------------------------------------
# 30-block trajectory: x_t = x_{t-1} + sigma_t N(0,1); y_t = x_t + r_t, r_t its own walk
# ------------------------------------------------------------------------------------------------

def sigma_schedule(steps: int = 50, hi: float = 0.3, lo: float = 0.01) -> list:
    """sigma_t for t = 1..steps-1, geometric from hi to lo (sigma_0 unused)."""
    n = steps - 1
    return [0.0] + [hi * (lo / hi) ** ((t - 1) / (n - 1)) for t in range(1, steps)]


def block_alpha(k: int, blocks: int = 30) -> float:
    return 0.02 * 25.0 ** (k / (blocks - 1))


class Trajectory:
    """Streams (x_t, y_t) for one block over the steps, seeded per (block, step)."""

    def __init__(self, M: int, C: int, block: int, *, blocks: int = 30, steps: int = 50, seed: int = 0,
                 device="cpu", outlier_every: int = 3, n_outlier: int | None = None, scale: float = 50.0):
        self.M, self.C, self.k, self.steps, self.seed, self.device = M, C, block, steps, seed, device
        self.sig = sigma_schedule(steps)
        self.alpha = block_alpha(block, blocks)
        n_out = n_outlier if n_outlier is not None else max(1, int(round(0.005 * C)))
        with_out = (block % outlier_every == 0)
        g = _gen(device, sub_seed(seed, 400, block, 0))
        x = torch.randn((M, C), generator=g, device=device, dtype=torch.float32)
        if with_out:
            ch = outlier_channels(C, n_out, sub_seed(seed, 401, block, 0), device)
            x[:, ch] *= scale
        self.x = x
        self.r = self.alpha * torch.randn((M, C), generator=g, device=device, dtype=torch.float32)
        self.t = 0

    def current(self):
        """bf16 (x_t, y_t) of the current step."""
        return self.x.to(torch.bfloat16), (self.x + self.r).to(torch.bfloat16)

    def advance(self):
        self.t += 1
        s = self.sig[self.t]
        g = _gen(self.device, sub_seed(self.seed, 402, self.k, self.t))
        self.x = self.x + s * torch.randn(self.x.shape, generator=g, device=self.device, dtype=torch.float32)
        self.r = self.r + self.alpha * s * torch.randn(self.x.shape, generator=g, device=self.device, dtype=torch.float32)


def rms(t: torch.Tensor) -> float:
    f = t.float()
    return math.sqrt(float(torch.mean(f * f)))
