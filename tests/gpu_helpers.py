"""Helpers for the GPU parity tests: moving seeded numpy inputs to the device
and comparing results with the oracle."""

import numpy as np
import torch

from workloads import bf16_to_f64

# spec tolerance for bf16 attention outputs against the fp64 oracle
MAX_ABS = 2e-2
MEAN_ABS = 2e-3


def dev(x):
    """numpy -> cuda tensor (uint16 bf16 bits become torch.bfloat16)."""
    if x.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def host_f64(t):
    """cuda tensor -> float64 numpy (bf16 widened exactly)."""
    if t.dtype == torch.bfloat16:
        return bf16_to_f64(t.view(torch.int16).cpu().numpy().view(np.uint16))
    return t.cpu().numpy().astype(np.float64)


def assert_close_attention(got, want, what=""):
    err = np.abs(got - want)
    assert np.all(np.isfinite(got)), what + ": non-finite output"
    assert err.max() <= MAX_ABS, "%s: max abs err %.3g" % (what, err.max())
    assert err.mean() <= MEAN_ABS, "%s: mean abs err %.3g" % (what, err.mean())


def status(t):
    torch.cuda.synchronize()
    return int(t.item())
