"""flexq_debug_export_canonical: the packed weights of either device layout
turned back into the canonical 6-bit form (four codes in three bytes,
row-major).  Compared byte for byte with the oracle's canonical packing of
the oracle's codes, for quantized weights and for every 6-bit code value
(including -32, which the quantizer never produces) placed by the oracle's
own device-form packers."""

import numpy as np
import pytest
import torch

from bit_group_quantized_flexq_b200 import flexq, inputs
from oracle import flexq_oracle as orc
from tests.gpu_util import np16

pytestmark = pytest.mark.gpu
LAYOUTS = [flexq.LAYOUT_BYTE_ALIGNED, flexq.LAYOUT_4_2]


@pytest.mark.parametrize("layout", LAYOUTS)
@pytest.mark.parametrize("N,K,gs", [(128, 256, 32), (384, 1024, 128), (1024, 4096, 64)])
def test_export_of_quantized_weights_equals_the_oracle(N, K, gs, layout):
    w = inputs.weights(N, K, std=0.02, seed=inputs.layer_seed("canon", N, K, gs))
    wp, _ = flexq.quantize_weight(w.cuda(), gs, layout=layout)
    canon = flexq.export_canonical(wp, N, K, layout)
    qw, _ = orc.quantize_weight(w.numpy(), gs)
    assert np.array_equal(np16(canon), orc.pack_canonical(qw))


@pytest.mark.parametrize("layout", LAYOUTS)
def test_export_of_every_code_value(layout):
    N, K = 256, 512
    rng = np.random.default_rng(20261202)
    codes = rng.integers(-32, 32, size=(N, K)).astype(np.int8)
    codes[0, :64] = np.arange(-32, 32)                      # each value at a known place
    codes[1] = -32
    codes[2] = 31
    pack = orc.pack_device_form if layout == flexq.LAYOUT_BYTE_ALIGNED else orc.pack_device_form42
    dev = torch.from_numpy(np.ascontiguousarray(pack(codes)).reshape(-1)).cuda()
    canon = flexq.export_canonical(dev, N, K, layout)
    want = orc.pack_canonical(codes)
    assert np.array_equal(np16(canon), want)
    assert np.array_equal(orc.unpack_canonical(np16(canon), K), codes)


def test_both_layouts_export_the_same_bytes():
    N, K, gs = 512, 2048, 128
    w = inputs.weights(N, K, std=0.02, seed=inputs.layer_seed("canon-ab", N, K))
    a, _ = flexq.quantize_weight(w.cuda(), gs, layout=flexq.LAYOUT_BYTE_ALIGNED)
    b, _ = flexq.quantize_weight(w.cuda(), gs, layout=flexq.LAYOUT_4_2)
    assert not torch.equal(a, b)                            # different device forms
    assert torch.equal(flexq.export_canonical(a, N, K, flexq.LAYOUT_BYTE_ALIGNED),
                       flexq.export_canonical(b, N, K, flexq.LAYOUT_4_2))
