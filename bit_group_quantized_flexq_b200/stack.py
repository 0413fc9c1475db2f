"""A stack of group-quantized linear layers with per-layer activation bits.

FlexQ keeps 8-bit activations in the layers whose activations are sensitive
to quantization and runs the rest at 6 bits, with 6-bit weights everywhere
(FlexQ paper, arXiv abstract; drgamma blog, "Fine-Grained Quantization and
Layer Sensitivity").  Which layers get 8 bits comes from a configuration
here: the sensitivity analysis that picks them needs calibration data.

Layers that read the same activations (a "site": q, k and v all read the
attention input) and use the same bit width share one quantization.  In
layer order: a layer whose site is already quantized at its width runs
flexq.gemm on those codes; otherwise, where the library quantizes inside the
GEMM (flexq.linear_launches == 1), flexq.linear; otherwise the site is
quantized once (flexq.quantize_act) for this and later layers.  Every output
is bit-identical to flexq.linear on that layer alone.

Configuration (a dict, or a JSON file holding one):

    {"group_size": 128,
     "act_bits": {"q": 6, "k": 6, "v": 6, "o": 6, "gate": 6, "up": 6, "down": 8}}

Every layer of the stack must be named, with 6 or 8 bits.
"""

import json
import os

import torch

from bit_group_quantized_flexq_b200 import flexq, inputs

# the configuration the 70B benchmark shapes use: 8-bit activations for the
# MLP down projection (the layer whose input carries the largest outliers)
LLAMA2_70B_MIXED = {
    "group_size": 128,
    "act_bits": {"q": 6, "k": 6, "v": 6, "o": 6, "gate": 6, "up": 6, "down": 8},
}


def parse_config(cfg, layers):
    """(group size, {layer name: activation bits}) from a config dict or the
    path of a JSON file; raises ValueError on anything missing or invalid."""
    if isinstance(cfg, (str, os.PathLike)):
        with open(cfg) as f:
            cfg = json.load(f)
    if not isinstance(cfg, dict):
        raise ValueError("config must be a dict or a JSON file holding one")
    gs = cfg.get("group_size", 128)
    if gs not in (32, 64, 128, 256):
        raise ValueError(f"group_size {gs!r} not in (32, 64, 128, 256)")
    bits = cfg.get("act_bits")
    if not isinstance(bits, dict):
        raise ValueError("config needs an 'act_bits' mapping of layer name to 6 or 8")
    names = [l[0] for l in layers]
    unknown = sorted(set(bits) - set(names))
    missing = [n for n in names if n not in bits]
    if unknown or missing:
        raise ValueError(f"act_bits: unknown layers {unknown}, missing layers {missing}")
    for n in names:
        if bits[n] not in (6, 8):
            raise ValueError(f"act_bits[{n!r}] = {bits[n]!r}, not 6 or 8")
    for name, N, K, _ in layers:
        if flexq.weight_packed_bytes(N, K, gs) == 0:
            raise ValueError(f"layer {name}: {N}x{K} not supported with group size {gs}")
    return gs, {n: int(bits[n]) for n in names}


class LayerStack:
    """Packed weights of a stack of linear layers and the per-layer bits.

    layers:  [(name, N, K, site)], e.g. inputs.LLAMA2_70B_BLOCK;
    config:  see the module docstring;
    weights: {name: FP16 [N, K] tensor} (any device), or None for seeded
             synthetic weights drawn on `device` (N(0, std)).
    """

    def __init__(self, layers, config, device="cuda", weights=None, std=0.015, seed=0):
        self.layers = list(layers)
        self.gs, self.bits = parse_config(config, self.layers)
        self.device = torch.device(device)
        self.site_k = {}
        for name, N, K, site in self.layers:
            if self.site_k.setdefault(site, K) != K:
                raise ValueError(f"site {site!r} read with K = {self.site_k[site]} and {K}")
        self.packed = {}
        for name, N, K, _ in self.layers:
            if weights is not None:
                w = weights[name].to(self.device)
            else:
                w = inputs.weights(N, K, std=std, seed=inputs.layer_seed("stack", seed, name),
                                   device=self.device)
            self.packed[name] = flexq.quantize_weight(w, self.gs)
            del w

    def sites(self):
        """{site: K}: the activations the stack reads."""
        return dict(self.site_k)

    def packed_bytes(self):
        return sum(wp.numel() + ws.numel() * 2 for wp, ws in self.packed.values())

    def launches(self, M):
        """Kernel launches of one forward at batch M."""
        n, quantized = 0, set()
        for name, N, K, site in self.layers:
            key = (site, self.bits[name])
            if key in quantized or flexq.linear_launches(M, N, K, self.gs) == 1:
                n += 1
            else:
                n += 2
                quantized.add(key)
        return n

    def forward(self, acts, out=None):
        """acts: {site: FP16 [M, K]} on the stack's device.  Returns
        {layer name: FP16 [M, N]} (written into `out` when given)."""
        M = None
        for site, K in self.site_k.items():
            x = acts[site]
            if x.dim() != 2 or x.shape[1] != K:
                raise ValueError(f"activations of site {site!r} must be [M, {K}]")
            if M is None:
                M = x.shape[0]
            elif x.shape[0] != M:
                raise ValueError("every site must hold the same number of tokens")
        out = {} if out is None else out
        codes = {}
        for name, N, K, site in self.layers:
            wp, ws = self.packed[name]
            bits = self.bits[name]
            y = out.get(name)
            key = (site, bits)
            if key not in codes and flexq.linear_launches(M, N, K, self.gs) == 1:
                out[name] = flexq.linear(acts[site], wp, ws, N, self.gs, bits, out=y)
                continue
            if key not in codes:
                codes[key] = flexq.quantize_act(acts[site], self.gs, bits)
            xq, xs = codes[key]
            out[name] = flexq.gemm(xq, xs, wp, ws, N, self.gs, bits, out=y)
        return out
