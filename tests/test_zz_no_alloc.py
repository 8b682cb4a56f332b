"""The allocation-free quantizer entry point.

nvfp4_quantize_act_static serves callers that cannot allocate device memory
where they quantize (a plugin whose host engine owns all device memory, a
latency-critical path that may not call cudaMalloc): it keeps its scratch in
a fixed array inside the library instead of taking a workspace.  Called
through the C ABI, two calls in a row, it must give the same codes, scale
bytes and global scales as nvfp4_quantize_act with a workspace (bit-exact,
the tolerance of every quantizer test), for one tensor and for row groups,
and reject more groups than its fixed scratch holds.

Kept in a file that sorts last, so a run that stops at the first failure has
already run every other test."""
import numpy as np
import pytest

import workloads as W
import nvfp4_w4a4_quantized_05_b200 as nv
from gpu_util import bf16_to_device, device

pytestmark = pytest.mark.gpu


def _buffers(rows, k, groups):
    import torch
    dev = device()
    sbytes = nv.nvfp4_scale_bytes(rows, k) if groups == 0 else nv.nvfp4_grouped_scale_bytes(rows, groups, k)
    return (torch.empty((rows, k // 2), dtype=torch.uint8, device=dev),
            torch.empty(sbytes, dtype=torch.uint8, device=dev),
            torch.empty(max(1, groups), dtype=torch.float32, device=dev))


def _run_both(x, off, groups):
    import torch
    rows, k = x.shape
    stream = torch.cuda.current_stream().cuda_stream
    offp = 0 if off is None else off.data_ptr()
    ws = torch.zeros(nv.nvfp4_workspace_bytes(nv.OP_QUANTIZE_ACT, rows, 0, k, groups), dtype=torch.uint8,
                     device=device())
    ref = _buffers(rows, k, groups)
    st = nv.nvfp4_quantize_act(x.data_ptr(), rows, k, x.stride(0), offp, groups, ref[0].data_ptr(),
                               ref[1].data_ptr(), ref[2].data_ptr(), ws.data_ptr(), stream)
    assert st == 0
    outs = []
    for _ in range(2):                       # two calls in a row share the fixed scratch
        got = _buffers(rows, k, groups)
        for t in got:
            t.fill_(0xA5 if t.dtype == torch.uint8 else 7.0)
        st = nv.nvfp4_quantize_act_static(x.data_ptr(), rows, k, x.stride(0), offp, groups, got[0].data_ptr(),
                                          got[1].data_ptr(), got[2].data_ptr(), stream)
        assert st == 0
        outs.append(got)
    torch.cuda.synchronize()
    nv.check_device_error()
    # bytes of the scale buffer that the quantizer writes: every group's block,
    # padded to 128 rows (the buffer itself is sized by an upper bound)
    if off is None:
        written = ref[1].numel()
    else:
        sizes = (off[1:] - off[:-1]).cpu().numpy()
        written = int(sum((int(s) + 127) // 128 * 128 for s in sizes)) * ((k // 16 + 3) // 4 * 4)
    for got in outs:
        assert torch.equal(got[0], ref[0])
        assert torch.equal(got[1][:written], ref[1][:written])
        assert torch.equal(got[2].view(torch.int32), ref[2].view(torch.int32))


def test_static_scratch_matches_workspace_entry_point_one_tensor():
    xb = W.gaussian_bf16((300, 4096), 0, 900, 1.0, outlier_frac=0.01)
    _run_both(bf16_to_device(xb), None, 0)


def test_static_scratch_matches_workspace_entry_point_groups():
    import torch
    sizes = [0, 5, 128, 130, 0, 1, 257, 64]
    off = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    xb = W.gaussian_bf16((int(off[-1]), 2048), 0, 901, 1.0, outlier_frac=0.01)
    _run_both(bf16_to_device(xb), torch.from_numpy(off).to(device()), len(sizes))


@pytest.mark.parametrize("k", [48, 80])
def test_static_scratch_two_kernel_path(k):
    """k % 64 != 0 takes the two-kernel path, whose scratch words (the CTA
    counter, the per-group amaxes and the groups' first scale rows) sit
    elsewhere in the array than the one-launch path's: one tensor and row
    groups, two calls in a row each."""
    import torch
    xb = W.gaussian_bf16((333, k), 0, 902 + k, 1.0, outlier_frac=0.01)
    _run_both(bf16_to_device(xb), None, 0)
    sizes = [7, 0, 200, 129, 1]
    off = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    xg = W.gaussian_bf16((int(off[-1]), k), 0, 903 + k, 1.0, outlier_frac=0.01)
    _run_both(bf16_to_device(xg), torch.from_numpy(off).to(device()), len(sizes))


@pytest.mark.parametrize("k", [128, 80])
def test_static_scratch_at_its_group_limit(k):
    """Exactly 1024 row groups, the most the fixed array holds (sizes 0..9,
    runs of empty groups), on the one-launch (k = 128) and the two-kernel
    (k = 80) path."""
    import torch
    rng = np.random.default_rng(k)
    sizes = rng.integers(0, 10, 1024)
    sizes[100:140] = 0
    off = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    xb = W.gaussian_bf16((int(off[-1]), k), 0, 904 + k, 1.0, outlier_frac=0.01)
    _run_both(bf16_to_device(xb), torch.from_numpy(off).to(device()), 1024)


def test_static_scratch_rejects_more_groups_than_it_holds():
    import torch
    groups = 1025
    off = torch.zeros(groups + 1, dtype=torch.int32, device=device())
    x = bf16_to_device(np.zeros((16, 64), np.uint16))
    got = _buffers(16, 64, groups)
    st = nv.nvfp4_quantize_act_static(x.data_ptr(), 16, 64, 64, off.data_ptr(), groups, got[0].data_ptr(),
                                      got[1].data_ptr(), got[2].data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == 2                           # NVFP4_ERR_UNSUPPORTED_SHAPE
