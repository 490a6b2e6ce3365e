"""Shared helpers for the GPU tests (device transfer, error norms)."""
import numpy as np
import torch

TOL = 1e-5  # normwise relative tolerance on fp32 outputs


def dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def host(t):
    return t.detach().cpu().numpy()


def bits16(t):
    """binary16 tensor -> uint16 bit patterns (numpy)."""
    return host(t.contiguous().view(torch.int16)).view(np.uint16)


def rowwise_err(got, want):
    """max_j |got - want| / max_j |want| per row (normwise relative error)."""
    got = np.asarray(got, np.float64).reshape(got.shape[0], -1)
    want = np.asarray(want, np.float64).reshape(want.shape[0], -1)
    den = np.maximum(np.abs(want).max(axis=1), 1e-300)
    return np.abs(got - want).max(axis=1) / den


def status():
    from invariant_numerics_b200 import invnum
    return invnum.inv_get_device_status()
