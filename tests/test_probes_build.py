"""The hardware-rate probes compile for sm_100a (they run only on a GPU, by
`python -m bit_group_quantized_flexq_b200.probes.run`)."""

import os
import subprocess

import pytest

from bit_group_quantized_flexq_b200 import build as flexq_build
from bit_group_quantized_flexq_b200.probes import run as probes

HERE = os.path.dirname(os.path.abspath(probes.__file__))


@pytest.mark.parametrize("name", probes.PROBES)
def test_probe_compiles(name, tmp_path):
    out = tmp_path / name
    r = subprocess.run([flexq_build.nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a",
                        "-O3", "-std=c++17", "-o", str(out), os.path.join(HERE, name + ".cu")],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr[-2000:]
    assert out.exists()
