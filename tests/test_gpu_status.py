"""Failure path on the GPU without a fault: a bounded wait that runs out.

bd_debug_wait_timeout launches a kernel whose barrier nothing ever arrives
on; its wait gives up after a few polls, records BD_ERR_TIMEOUT and returns.
The context must stay usable afterwards.
"""

import pytest
import torch

from block_diffusion_lm_bd_b200 import api

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    assert api.get_device_status() == 0
    api.debug_wait_timeout(2000)  # 2 ms
    assert api.get_device_status() == 4  # BD_ERR_TIMEOUT
    assert api.get_device_status() == 0  # cleared
    x = torch.randn(4, 1000, device="cuda")
    res = api.unmask(x, torch.ones(4, dtype=torch.uint8, device="cuda"), 0.9)
    assert res["tokens"].cpu().tolist() == x.argmax(1).cpu().tolist()
    assert api.get_device_status() == 0


def test_launch_counter_counts_library_kernels():
    n0 = api.launch_count()
    x = torch.randn(4, 1000, device="cuda")
    api.unmask(x, torch.ones(4, dtype=torch.uint8, device="cuda"), 0.9)
    assert api.launch_count() - n0 == 2
