"""Seeded synthetic inputs for the W6A6 / W6A8 linear layers.

This module draws random FP16 matrices and names the benchmark shapes; it
holds none of the quantization or GEMM arithmetic, so that the CUDA path and
the CPU oracle can both be fed from it without sharing any of the method.

Distributions (FlexQ evaluates on LLaMA-family linear layers, arXiv abstract;
no weights or activations are available here, so seeded synthetic stand-ins
of the same shapes are used):

* weights  W[N, K] ~ N(0, std) with std 0.02 (0.015 for the 70B shapes);
* activations X[M, K] ~ N(0, 1), with a fixed random set of ceil(frac * K)
  channels (the same for every row) multiplied by ``outlier_scale`` before
  the FP16 cast: 1% x20, or 0.5% x50 for the 70B shapes.

Draws use torch's CPU generator so that every consumer sees identical bits
for a given seed (weights may also be drawn on a CUDA device, see weights).
"""

import math

import torch

# ---------------------------------------------------------------- shapes ---
# (name, N, K) for one transformer block's linear layers.
LLAMA2_7B_LAYERS = [
    ("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
    ("gate", 11008, 4096), ("up", 11008, 4096), ("down", 4096, 11008),
]
LLAMA2_7B_M = [1, 16, 256, 2048]
# One LLaMA-2-7B transformer block with the input site of each layer (as
# LLAMA2_70B_BLOCK below).
LLAMA2_7B_BLOCK = [
    ("q", 4096, 4096, "attn_in"), ("k", 4096, 4096, "attn_in"), ("v", 4096, 4096, "attn_in"),
    ("o", 4096, 4096, "attn_out"),
    ("gate", 11008, 4096, "mlp_in"), ("up", 11008, 4096, "mlp_in"),
    ("down", 4096, 11008, "mlp_act"),
]

LLAMA2_13B_LAYERS = [("qkvo", 5120, 5120), ("gate_up", 13824, 5120),
                     ("down", 5120, 13824)]
LLAMA2_13B_M = [1, 64, 4096]

# (name, N, K, activation bits)
LLAMA2_70B_LAYERS = [("q_o", 8192, 8192, 6), ("gate_up", 28672, 8192, 6),
                     ("down", 8192, 28672, 8)]
# One LLaMA-2-70B transformer block, layer by layer: (name, N, K, input site).
# k and v are 1024 wide (8 key/value heads of 128 under grouped-query
# attention); layers with the same site read the same activations.
LLAMA2_70B_BLOCK = [
    ("q", 8192, 8192, "attn_in"), ("k", 1024, 8192, "attn_in"), ("v", 1024, 8192, "attn_in"),
    ("o", 8192, 8192, "attn_out"),
    ("gate", 28672, 8192, "mlp_in"), ("up", 28672, 8192, "mlp_in"),
    ("down", 8192, 28672, "mlp_act"),
]
LLAMA2_70B_M = [1, 16, 512, 8192]

SWEEP_NK = 8192
SWEEP_GS = [32, 64, 128, 256]
SWEEP_M = [1, 8, 32, 128, 1024, 4096, 16384]


def _gen(seed):
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def weights(N, K, std=0.02, seed=0, device="cpu"):
    """FP16 [N, K] drawn from N(0, std).  With a CUDA device the draw uses that
    device's generator (fast for the largest layers; its bits differ from the
    CPU draw of the same seed, so use it only where no oracle comparison
    follows)."""
    dev = torch.device(device)
    if dev.type == "cuda":
        g = torch.Generator(device=dev)
        g.manual_seed(int(seed))
        w = torch.randn(N, K, generator=g, dtype=torch.float32, device=dev)
        w.mul_(std)
        return w.to(torch.float16)
    w = torch.randn(N, K, generator=_gen(seed), dtype=torch.float32) * std
    return w.to(torch.float16)


def outlier_channels(K, frac, seed):
    """The sorted indices of ceil(frac*K) outlier channels (empty if frac=0)."""
    n = int(math.ceil(frac * K)) if frac > 0 else 0
    if n == 0:
        return torch.empty(0, dtype=torch.long)
    return torch.sort(torch.randperm(K, generator=_gen(seed))[:n]).values


def activations(M, K, outlier_frac=0.01, outlier_scale=20.0, seed=1):
    """FP16 [M, K] ~ N(0, 1) with a fixed set of scaled outlier channels."""
    x = torch.randn(M, K, generator=_gen(seed), dtype=torch.float32)
    ch = outlier_channels(K, outlier_frac, seed + 1)
    if ch.numel():
        x[:, ch] *= outlier_scale
    return x.to(torch.float16)


def uniform_fp16(shape, lo, hi, seed):
    """FP16 values uniform in [lo, hi) (edge-case tests)."""
    u = torch.rand(*shape, generator=_gen(seed), dtype=torch.float32)
    return (lo + (hi - lo) * u).to(torch.float16)


def random_codes(shape, lo, hi, seed):
    """int8 codes uniform in [lo, hi] (GEMM tests that bypass quantization)."""
    return torch.randint(lo, hi + 1, shape, generator=_gen(seed),
                         dtype=torch.int16).to(torch.int8)


def random_scales(shape, lo, hi, seed):
    """Positive FP16 scales uniform in [lo, hi)."""
    return uniform_fp16(shape, lo, hi, seed)


def layer_seed(*parts):
    """A stable seed for a named (config, shape) pair."""
    h = 0
    for p in parts:
        for ch in str(p):
            h = (h * 131 + ord(ch)) % 1_000_003
        h = (h * 131 + 7) % 1_000_003
    return h
