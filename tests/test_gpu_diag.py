"""Failure detection without a GPU fault: a kernel waiting on a flag that
nothing sets gives up after its limit and the host reads NVFP4_ERR_TIMEOUT;
the context stays usable afterwards."""
import numpy as np
import pytest

import oracle as O
import workloads as W
import nvfp4_w4a4_quantized_05_b200 as nv
from gpu_util import bf16_to_device, device

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


def test_cached_workspace_reset_after_a_reported_timeout():
    """What a timed-out grid barrier leaves behind, made on the host: one
    CTA's generation word in the binding's cached quantizer workspace is
    moved ahead of the others (the next call's CTAs would then never agree
    and would wait in vain), and the device error word is set by the
    bounded-wait probe.  check_device_error reports the timeout and
    re-initialises the cached workspaces, so the next quantization is the
    oracle's bit for bit, with no timeout."""
    import torch
    xb = W.gaussian_bf16((300, 1024), 0, 77, 1.0, outlier_frac=0.01)
    x = bf16_to_device(xb)
    nv.quantize_act(x)
    torch.cuda.synchronize()
    nv.check_device_error()
    stream = torch.cuda.current_stream().cuda_stream
    key = (device().index if device().index is not None else torch.cuda.current_device(), nv.OP_QUANTIZE_ACT, 0,
           stream)
    ws = nv._ws_cache[key]
    words = ws.view(torch.int64)
    words[0] += 7 << 32                                   # CTA 0's generation, 7 ahead
    flag = torch.zeros(4, dtype=torch.int32, device=device())
    assert nv.nvfp4_probe_bounded_wait(flag.data_ptr(), 1_000_000) == 0
    with pytest.raises(nv.Nvfp4Error) as e:
        nv.check_device_error()
    assert e.value.status == 5
    assert int(ws.to(torch.int64).sum()) == 0            # re-initialised
    q = nv.quantize_act(x)
    torch.cuda.synchronize()
    nv.check_device_error()
    oc, osf, og = O.quantize_1d(xb)
    assert np.array_equal(q.codes.cpu().numpy(), oc) and np.array_equal(q.scales.cpu().numpy(), osf)
    assert q.global_scale.item() == float(np.float32(og))
