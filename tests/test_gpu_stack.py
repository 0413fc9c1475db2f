"""The mixed W6A6 / W6A8 layer stack on the GPU: run layer by layer, every
layer's output is bit-identical to flexq.linear on that layer alone (the
stack only shares the quantization of a site between layers of the same bit
width); run with grouped calls, to flexq.linear_group on the site's layers;
always within the GEMM tolerance of the oracle's linear layer."""

import pytest
import torch

from bit_group_quantized_flexq_b200 import flexq, inputs, stack
from oracle import flexq_oracle as orc
from tests.gpu_util import assert_within, np16

pytestmark = pytest.mark.gpu

TOL = 1e-3

# the 70B block with every width divided by 8 (same structure, quick oracle)
SMALL = [(n, N // 8, K // 8, site) for (n, N, K, site) in inputs.LLAMA2_70B_BLOCK]
MIXED = {"group_size": 128,
         "act_bits": {"q": 6, "k": 8, "v": 6, "o": 8, "gate": 6, "up": 6, "down": 8}}


def _acts(layers, M, seed):
    sites = {}
    for name, N, K, site in layers:
        sites.setdefault(site, K)
    return {site: inputs.activations(M, K, outlier_frac=0.005, outlier_scale=50.0,
                                     seed=inputs.layer_seed("stack-x", seed, site))
            for site, K in sites.items()}


@pytest.mark.parametrize("M", [1, 5, 40])
def test_small_block_matches_single_layers_and_the_oracle(M):
    w = {name: inputs.weights(N, K, std=0.015, seed=inputs.layer_seed("stack-w", name))
         for name, N, K, _ in SMALL}
    st = stack.LayerStack(SMALL, MIXED, weights=w, group_sites=False)
    acts = _acts(SMALL, M, seed=M)
    dacts = {k: v.cuda() for k, v in acts.items()}
    out = st.forward(dacts)
    for name, N, K, site in SMALL:
        wp, ws, _ = st.layer_weights(name)
        bits = MIXED["act_bits"][name]
        alone = flexq.linear(dacts[site], wp, ws, N, 128, bits)
        assert torch.equal(out[name], alone), name
        ref = orc.linear_layer(acts[site].numpy(), w[name].numpy(), 128, bits)
        assert_within(np16(out[name]), ref["y64"], TOL)


@pytest.mark.parametrize("M", [1, 16])
def test_70b_block_matches_single_layers(M):
    st = stack.LayerStack(inputs.LLAMA2_70B_BLOCK, stack.LLAMA2_70B_MIXED, group_sites=False)
    acts = {k: v.cuda() for k, v in _acts(inputs.LLAMA2_70B_BLOCK, M, seed=70).items()}
    out = st.forward(acts)
    for name, N, K, site in inputs.LLAMA2_70B_BLOCK:
        wp, ws, _ = st.layer_weights(name)
        alone = flexq.linear(acts[site], wp, ws, N, 128, st.bits[name])
        assert torch.equal(out[name], alone), name
    assert flexq.device_status()[0] == flexq.FLEXQ_OK


def test_launch_count_shares_site_quantization():
    st = stack.LayerStack(SMALL, MIXED, group_sites=False)
    assert st.launches(1) == 7                       # quantization inside each GEMM
    # M = 40: attn_in has 6-bit q, v and 8-bit k (2 quantizations + 3 GEMMs),
    # attn_out 2, mlp_in 1 + 2, mlp_act 2
    assert st.launches(40) == 5 + 2 + 3 + 2
    # the 70B block at M = 1: q, k, v and o (8, 4, 4 and 8 stages per CTA)
    # quantize inside their GEMMs; gate (32 stages) and down (28) quantize
    # first; up reuses gate's codes
    big = stack.LayerStack(inputs.LLAMA2_70B_BLOCK, stack.LLAMA2_70B_MIXED, group_sites=False)
    assert big.launches(1) == 1 + 1 + 1 + 1 + 2 + 1 + 2
    # at M = 4 only k and v (4 stages) still do
    assert big.launches(4) == 2 + 1 + 1 + 2 + 2 + 1 + 2


def test_forward_rejects_mismatched_sites():
    st = stack.LayerStack(SMALL, MIXED)
    acts = {k: v.cuda() for k, v in _acts(SMALL, 4, seed=1).items()}
    acts["mlp_act"] = acts["mlp_act"][:3]
    with pytest.raises(ValueError, match="same number of tokens"):
        st.forward(acts)
    acts["mlp_act"] = torch.zeros(4, 100, dtype=torch.float16, device="cuda")
    with pytest.raises(ValueError, match="must be"):
        st.forward(acts)


@pytest.mark.parametrize("M", [1, 4, 40])
def test_fused_sites_match_the_stacked_layer_and_the_oracle(M):
    w = {name: inputs.weights(N, K, std=0.015, seed=inputs.layer_seed("stack-w", name))
         for name, N, K, _ in SMALL}
    cfg = {"group_size": 128,
           "act_bits": {"q": 6, "k": 6, "v": 8, "o": 8, "gate": 6, "up": 6, "down": 8}}
    st = stack.LayerStack(SMALL, cfg, weights=w, fuse_sites=True)
    # q and k merge (v has other bits); gate and up merge
    assert [len(u[4]) for u in st.units] == [2, 1, 1, 2, 1]
    acts = _acts(SMALL, M, seed=M + 7)
    dacts = {k: v.cuda() for k, v in acts.items()}
    out = st.forward(dacts)
    for name, N, K, site in SMALL:
        bits = cfg["act_bits"][name]
        wp, ws, n_total = st.layer_weights(name)
        merged = flexq.linear(dacts[site], wp, ws, n_total, 128, bits)
        off = [m for u in st.units for m in u[4] if m[0] == name][0][2]
        assert torch.equal(out[name], merged[:, off:off + N]), name
        ref = orc.linear_layer(acts[site].numpy(), w[name].numpy(), 128, bits)
        assert_within(np16(out[name]), ref["y64"], TOL)


def test_fused_70b_block_launches():
    st = stack.LayerStack(inputs.LLAMA2_70B_BLOCK, stack.LLAMA2_70B_MIXED, fuse_sites=True)
    assert [len(u[4]) for u in st.units] == [3, 1, 2, 1]      # qkv, o, gate+up, down
    assert st.launches(16) == 4 * 2
    acts = {k: v.cuda() for k, v in _acts(inputs.LLAMA2_70B_BLOCK, 16, seed=71).items()}
    out = st.forward(acts)
    assert out["k"].shape == (16, 1024) and out["up"].shape == (16, 28672)
    assert flexq.device_status()[0] == flexq.FLEXQ_OK


@pytest.mark.parametrize("M", [1, 5, 40])
def test_grouped_small_block_matches_grouped_calls_and_the_oracle(M):
    w = {name: inputs.weights(N, K, std=0.015, seed=inputs.layer_seed("stack-w", name))
         for name, N, K, _ in SMALL}
    st = stack.LayerStack(SMALL, MIXED, weights=w)            # grouped by default
    # attn_in: q, v (6 bits) grouped, k (8 bits) alone; mlp_in: gate + up
    assert sorted(len(g) for g in st.groups) == [1, 1, 1, 2, 2]
    acts = _acts(SMALL, M, seed=M + 3)
    dacts = {k: v.cuda() for k, v in acts.items()}
    out = st.forward(dacts)
    for g in st.groups:
        names = [st.units[i][4][0][0] for i in g]
        site, bits = st.units[g[0]][1], st.units[g[0]][2]
        ys = flexq.linear_group(dacts[site], [st.layer_weights(n) for n in names], 128, bits)
        for n, y in zip(names, ys):
            assert torch.equal(out[n], y), n
    for name, N, K, site in SMALL:
        ref = orc.linear_layer(acts[site].numpy(), w[name].numpy(), 128, MIXED["act_bits"][name])
        assert_within(np16(out[name]), ref["y64"], TOL)


def test_grouped_70b_block_launches_and_runs():
    st = stack.LayerStack(inputs.LLAMA2_70B_BLOCK, stack.LLAMA2_70B_MIXED)
    # q/k/v (11 stages per CTA) and gate/up (32) grouped: quantizer + one
    # grouped launch each; o (8 stages) quantizes inside its GEMM; down (28)
    # quantizer + GEMM
    assert st.launches(1) == 2 + 1 + 2 + 2
    assert st.launches(16) == 2 + 2 + 2 + 2
    acts = {k: v.cuda() for k, v in _acts(inputs.LLAMA2_70B_BLOCK, 16, seed=72).items()}
    out = st.forward(acts)
    assert out["k"].shape == (16, 1024) and out["up"].shape == (16, 28672)
    assert flexq.device_status()[0] == flexq.FLEXQ_OK
