"""Shared helpers for the GPU parity tests (test infrastructure)."""

import numpy as np
import torch

from oracle import flexq_oracle as orc


def np16(t):
    return t.detach().cpu().numpy()


def bits16(a):
    return np.asarray(a, dtype=np.float16).view(np.uint16)


def oracle_weight_device_form(w16, gs):
    """Oracle codes, scales and device-form bytes for an FP16 weight [N, K]."""
    qw, sw = orc.quantize_weight(w16, gs)
    N, K = w16.shape
    dev = orc.pack_device_form(qw)
    return qw, sw, dev


def upload_codes_as_weights(qw):
    """Pack arbitrary 6-bit codes [N, K] (oracle packing) into a device buffer."""
    N, K = qw.shape
    dev = orc.pack_device_form(qw)
    return torch.from_numpy(dev.copy()).cuda()


def assert_within(y_gpu, y64, tol=1e-3):
    err = orc.rel_err_vs_max(np.asarray(y_gpu, dtype=np.float64), y64)
    assert err <= tol, f"max|dY|/max|Y| = {err:.3e} > {tol}"
    return err
