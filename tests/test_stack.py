"""The layer-stack configuration (host only): every layer named with 6 or 8
activation bits, a supported group size, shapes the library packs."""

import json

import pytest

from bit_group_quantized_flexq_b200 import inputs, stack

BLOCK = inputs.LLAMA2_70B_BLOCK


def test_the_default_mixed_config_is_valid():
    gs, bits = stack.parse_config(stack.LLAMA2_70B_MIXED, BLOCK)
    assert gs == 128
    assert [bits[n] for n, *_ in BLOCK] == [6, 6, 6, 6, 6, 6, 8]


def test_config_from_a_json_file(tmp_path):
    cfg = {"group_size": 64, "act_bits": {n: 8 for n, *_ in BLOCK}}
    p = tmp_path / "stack.json"
    p.write_text(json.dumps(cfg))
    gs, bits = stack.parse_config(str(p), BLOCK)
    assert gs == 64 and set(bits.values()) == {8}


@pytest.mark.parametrize("cfg, msg", [
    ({"act_bits": {n: 6 for n, *_ in BLOCK if n != "down"}}, "missing"),
    ({"act_bits": dict({n: 6 for n, *_ in BLOCK}, lm_head=6)}, "unknown"),
    ({"act_bits": dict({n: 6 for n, *_ in BLOCK}, o=4)}, "not 6 or 8"),
    ({"group_size": 96, "act_bits": {n: 6 for n, *_ in BLOCK}}, "group_size"),
    ({"group_size": 128}, "act_bits"),
    ([6, 6, 8], "dict"),
])
def test_invalid_configs_are_rejected(cfg, msg):
    with pytest.raises(ValueError, match=msg):
        stack.parse_config(cfg, BLOCK)


def test_unsupported_layer_shapes_are_rejected():
    layers = [("odd", 200, 8192, "x")]                 # N not a multiple of 128
    with pytest.raises(ValueError, match="not supported"):
        stack.parse_config({"act_bits": {"odd": 6}}, layers)


def test_block_sites_share_their_width():
    ks = {}
    for name, N, K, site in BLOCK:
        assert ks.setdefault(site, K) == K
    assert ks == {"attn_in": 8192, "attn_out": 8192, "mlp_in": 8192, "mlp_act": 28672}
