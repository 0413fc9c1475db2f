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

With group_sites=True (the default) the layers of one site and width run as
one grouped call (flexq.linear_group): one quantization and one kernel
launch for, e.g., q, k and v, each layer keeping its own packed weights and
output.

With fuse_sites=True the layers of one site and width are instead merged into
one GEMM (the fused q/k/v and gate/up projections of inference engines):
their FP16 weights are stacked along N and quantized as one matrix (the
quantization is per row, so every layer keeps its codes and scales), and
each layer's output is its column slice of the merged output.  One launch
then carries several layers' set-up and split-K tail; each output equals
flexq.linear on the stacked weights, and differs from the layer run alone
only in the FP32 summation order of a different K split.

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

    layers:     [(name, N, K, site)], e.g. inputs.LLAMA2_70B_BLOCK;
    config:     see the module docstring;
    weights:    {name: FP16 [N, K] tensor} (any device), or None for seeded
                synthetic weights drawn on `device` (N(0, std));
    fuse_sites: merge the layers of one site and width into one GEMM;
    group_sites: run the layers of one site and width as one grouped call
                 (ignored with fuse_sites).
    """

    def __init__(self, layers, config, device="cuda", weights=None, std=0.015, seed=0,
                 fuse_sites=False, group_sites=True):
        self.layers = list(layers)
        self.gs, self.bits = parse_config(config, self.layers)
        self.device = torch.device(device)
        self.fuse_sites = fuse_sites
        self.group_sites = group_sites and not fuse_sites
        self.site_k = {}
        for name, N, K, site in self.layers:
            if self.site_k.setdefault(site, K) != K:
                raise ValueError(f"site {site!r} read with K = {self.site_k[site]} and {K}")

        def weight(name, N, K):
            if weights is not None:
                return weights[name].to(self.device)
            return inputs.weights(N, K, std=std, seed=inputs.layer_seed("stack", seed, name),
                                  device=self.device)

        # units of work in layer order: one layer, or (fuse_sites) all layers
        # of a (site, bits) pair, stacked along N at the first one's place
        self.units = []                    # (key, site, bits, K, [(name, N, offset)], N_total)
        by_key = {}
        for name, N, K, site in self.layers:
            key = (site, self.bits[name]) if fuse_sites else name
            if key not in by_key:
                by_key[key] = len(self.units)
                self.units.append([key, site, self.bits[name], K, [], 0])
            u = self.units[by_key[key]]
            u[4].append((name, N, u[5]))
            u[5] += N
        self.packed = {}                   # unit key -> (packed weights, scales)
        for key, site, bits, K, members, n_total in self.units:
            if len(members) == 1:
                w = weight(members[0][0], members[0][1], K)
            else:
                w = torch.cat([weight(name, N, K) for name, N, _ in members], dim=0)
            self.packed[key] = flexq.quantize_weight(w, self.gs)
            del w
        # grouped calls: the units of one (site, bits), in order of first use
        self.groups = []
        by_q = {}
        for i, (key, site, bits, K, members, n_total) in enumerate(self.units):
            q = (site, bits)
            if self.group_sites and q in by_q:
                self.groups[by_q[q]].append(i)
            else:
                by_q[q] = len(self.groups)
                self.groups.append([i])
        self._ybuf = {}

    def sites(self):
        """{site: K}: the activations the stack reads."""
        return dict(self.site_k)

    def packed_bytes(self):
        return sum(wp.numel() + ws.numel() * 2 for wp, ws in self.packed.values())

    def layer_weights(self, name):
        """(packed weights, scales, N) that produce layer `name`: its own, or
        its merged unit's (fuse_sites; the layer is a column slice of it)."""
        for key, site, bits, K, members, n_total in self.units:
            if any(m[0] == name for m in members):
                wp, ws = self.packed[key]
                return wp, ws, n_total
        raise KeyError(name)

    def launches(self, M):
        """Kernel launches of one forward at batch M."""
        if self.group_sites:
            n = 0
            for g in self.groups:
                K = self.units[g[0]][3]
                n += flexq.group_plan(M, K, self.gs, [self.units[i][5] for i in g])[3]
            return n
        n, quantized = 0, set()
        for key, site, bits, K, members, n_total in self.units:
            q = (site, bits)
            if q in quantized or flexq.linear_launches(M, n_total, K, self.gs) == 1:
                n += 1
            else:
                n += 2
                quantized.add(q)
        return n

    def forward(self, acts, out=None):
        """acts: {site: FP16 [M, K]} on the stack's device.  Returns
        {layer name: FP16 [M, N]}: written into `out` for layers run alone
        when given; merged layers (fuse_sites) are column views of a buffer
        the stack keeps per batch size."""
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
        if self.group_sites:
            for g in self.groups:
                key, site, bits, K, members, n_total = self.units[g[0]]
                weights = [self.packed[self.units[i][0]] + (self.units[i][5],) for i in g]
                outs = [out.get(self.units[i][4][0][0]) for i in g]
                ys = flexq.linear_group(acts[site], weights, self.gs, bits, outs=outs)
                for i, y in zip(g, ys):
                    out[self.units[i][4][0][0]] = y
            return out
        codes = {}
        for key, site, bits, K, members, n_total in self.units:
            wp, ws = self.packed[key]
            if len(members) == 1:
                y = out.get(members[0][0])
            else:                          # merged unit: one buffer per batch size
                y = self._ybuf.get((key, M))
                if y is None:
                    y = torch.empty(M, n_total, dtype=torch.float16, device=self.device)
                    self._ybuf[(key, M)] = y
            q = (site, bits)
            if q not in codes and flexq.linear_launches(M, n_total, K, self.gs) == 1:
                y = flexq.linear(acts[site], wp, ws, n_total, self.gs, bits, out=y)
            else:
                if q not in codes:
                    codes[q] = flexq.quantize_act(acts[site], self.gs, bits)
                xq, xs = codes[q]
                y = flexq.gemm(xq, xs, wp, ws, n_total, self.gs, bits, out=y)
            if len(members) == 1:
                out[members[0][0]] = y
            else:
                for name, N, off in members:
                    out[name] = y[:, off:off + N]
        return out
