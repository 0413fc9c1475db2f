"""Build every probe in this directory for sm_100a (into _build/probes/ at the
repository root) and run it, printing its lines under a header.  Each probe
runs one CTA per SM for a few milliseconds; every wait in them is bounded."""

import os
import subprocess
import sys

from bit_group_quantized_flexq_b200 import build as flexq_build

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
PROBES = ["mma_rate", "bulk_copy_rate", "tmem_rate", "tmem_vs_mma", "fp_pipe_rate"]


def main(names):
    out_dir = os.path.join(ROOT, "_build", "probes")
    os.makedirs(out_dir, exist_ok=True)
    rc = 0
    for name in names:
        exe = os.path.join(out_dir, name)
        cmd = [flexq_build.nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3",
               "-std=c++17", "-o", exe, os.path.join(HERE, name + ".cu")]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode:
            print(f"== {name}: build failed\n{r.stderr[-2000:]}", flush=True)
            rc = 1
            continue
        print(f"== {name}", flush=True)
        r = subprocess.run([exe], capture_output=True, text=True, timeout=300)
        print(r.stdout, end="", flush=True)
        if r.returncode:
            print(f"   exit {r.returncode}: {r.stderr[-500:]}", flush=True)
            rc = 1
    return rc


if __name__ == "__main__":
    sys.exit(main(sys.argv[1:] or PROBES))
