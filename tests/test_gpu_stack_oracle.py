"""Divergence of the 32-layer stack from the float64 oracle at the size of the
chunked-prefill workload (vocab 32000, an 8192-token random prompt), by the two
reduced oracle runs of bench.stack_divergence: teacher-forced per layer at 64
sampled positions, and free-running over a 512-token prefix plus 16 greedily
decoded tokens.

The divergences are reported (printed, and recorded by bench.py in its JSON
line).  The bounds below only catch breakage: a layer's own error stays within
a few INT16 quanta of the oracle (2e-4 normwise: the GPU's fp32 K/V and the
oracle's float64 K/V can round to neighbouring codes, one code being
max|x|/32767 of a row), and the accumulated distance after 32 layers stays far
below the size of the hidden states.
"""
import json

import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def inv():
    from invariant_numerics_b200 import invnum
    assert invnum.inv_get_device_status() == invnum.INV_OK
    return invnum


def test_stack_divergence_32_layers_8192_prompt(inv):
    import bench
    r = bench.stack_divergence(inv, torch, torch.device("cuda"))
    print(json.dumps(r))
    tf, fr = r["teacher_forced"], r["free_running"]
    assert len(tf["per_layer_max_normwise"]) == 32 and len(fr["per_layer_max_normwise"]) == 32
    assert tf["positions"] == 64
    assert tf["max"] <= 2e-4, tf
    assert fr["max"] <= 1e-2, fr
