"""Test helpers: moving generator output to the device and comparing with the oracle."""
from __future__ import annotations

import numpy as np

TOL = {"f32": 1e-5, "bf16": 2e-3}  # max|x - x_ref| <= TOL * max|x_ref|


def to_device(x: dict, device="cuda"):
    import torch

    out = {}
    for k, v in x.items():
        if v is None:
            out[k] = None
        elif v.dtype == np.uint16:
            out[k] = torch.from_numpy(v.view(np.int16)).view(torch.bfloat16).to(device)
        else:
            out[k] = torch.from_numpy(v).to(device)
    return out


def rel_err(got, ref) -> float:
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    scale = float(np.max(np.abs(ref))) if ref.size else 0.0
    err = float(np.max(np.abs(got - ref))) if ref.size else 0.0
    if scale == 0.0:
        return err
    return err / scale


def run_gpu(xd, softplus=True, **kw):
    from selective_state_space_ss_b200 import ss_scan_fwd

    return ss_scan_fwd(xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], D=xd["D"], z=xd["z"],
                       delta_bias=xd["delta_bias"], softplus=softplus, **kw)
