"""Failure detection without a GPU fault: a kernel waiting on a flag that
nothing sets gives up after its limit and the host reads NVFP4_ERR_TIMEOUT;
the context stays usable afterwards."""
import pytest

import nvfp4_w4a4_quantized_05_b200 as nv
from gpu_util import device

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_recovers():
    import torch
    flag = torch.zeros(4, dtype=torch.int32, device=device())
    assert nv.nvfp4_get_last_device_error() == 0
    assert nv.nvfp4_probe_bounded_wait(flag.data_ptr(), 1_000_000) == 0      # 1 ms
    assert nv.nvfp4_get_last_device_error() == 5                              # timed out
    assert nv.nvfp4_get_last_device_error() == 0                              # cleared
    flag.fill_(1)
    assert nv.nvfp4_probe_bounded_wait(flag.data_ptr(), 1_000_000) == 0
    assert nv.nvfp4_get_last_device_error() == 0
    x = torch.ones(1024, device=device())
    assert float(x.sum()) == 1024.0                                          # context still usable


def test_wait_limit_setter_round_trips():
    old = nv.nvfp4_set_wait_limit_ns(123456)
    assert nv.nvfp4_set_wait_limit_ns(old) == 123456
