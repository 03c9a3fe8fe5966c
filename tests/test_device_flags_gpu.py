"""Device-side failure reports through the workspace header, made on the host.

No kernel is made to fail here: after a good call, the test writes a flag
into word 1 of the workspace header (where the kernels record failures) and
checks that rb_gemv_check / rb_gemm_check report RB_ERR_DEVICE, and that the
next call clears the header again. The grouped matvec's own descriptor check
is driven for real: the device copy of the descriptors is changed after the
launch was planned on the host copy, and the kernel refuses to run.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import residual_binary_weight_b200 as rb
from residual_binary_weight_b200 import _lib
from gpu_util import to_dev_planes

pytestmark = pytest.mark.gpu


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _case(M=300, K=1024, T=3, seed=5):
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((M, K)) * 0.02).astype(np.float16)
    ref_p, ref_a, _ = oracle.pack(W, 2, 0)
    planes = to_dev_planes(ref_p)
    alpha = torch.from_numpy(ref_a.astype(np.float32)).cuda()
    x = torch.from_numpy(rng.standard_normal((T, K)).astype(np.float16)).cuda()
    return planes, alpha, x


def test_gemv_check_reports_a_flag_in_the_workspace():
    lib = _lib.load()
    planes, alpha, x = _case()
    ws = torch.zeros(rb.gemv_workspace_bytes(300, 1024, 2, 0, 3), dtype=torch.uint8, device="cuda")
    rb.gemv(planes, alpha, x, workspace=ws)
    assert lib.rb_gemv_check(_p(ws), _stream()) == 0
    ws.view(torch.int32)[1] = 1                      # what a kernel's atomicOr would leave
    rc = lib.rb_gemv_check(_p(ws), _stream())
    assert _lib.STATUS_NAMES[rc] == "RB_ERR_DEVICE"
    assert b"flag 0x1" in lib.rb_last_error()
    rb.gemv(planes, alpha, x, workspace=ws)            # the next call clears the header
    assert lib.rb_gemv_check(_p(ws), _stream()) == 0


@pytest.mark.parametrize("T", [3, 130])
def test_gemm_check_reports_a_flag_in_the_workspace(T):
    lib = _lib.load()
    planes, alpha, x = _case(T=T)
    need = rb.gemm_workspace_bytes(300, 1024, 2, 0, T)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    rb.gemm(planes, alpha, x, workspace=ws)
    assert lib.rb_gemm_check(_p(ws), _stream()) == 0
    ws.view(torch.int32)[1] = 4
    rc = lib.rb_gemm_check(_p(ws), _stream())
    assert _lib.STATUS_NAMES[rc] == "RB_ERR_DEVICE"
    assert b"operand expansion" in lib.rb_last_error()
    rb.gemm(planes, alpha, x, workspace=ws)
    assert lib.rb_gemm_check(_p(ws), _stream()) == 0


def test_grouped_refuses_device_descriptors_that_differ_from_the_host_copy():
    """The launch is planned (and its workspace sized) from the host
    descriptors; a device copy that gives another plan is caught by the
    kernel before it reads any plane or writes any output."""
    planes, alpha, x = _case(T=1)
    y = torch.full((1, 300), float("nan"), dtype=torch.float16, device="cuda")
    g = rb.GroupedGemv([(planes, alpha, x, y)], n_paths=2, group=0, T=1)
    g.run()
    g.check_device_flag()
    assert torch.isfinite(y).all()
    # M of descriptor 0 in the device copy: 300 -> 30000 rows (more units)
    desc = g.dev_descs.view(torch.int64)
    assert int(desc[4]) == 300
    desc[4] = 30000
    y.fill_(float("nan"))
    g.run()
    with pytest.raises(rb.RbError, match="descriptors differ"):
        g.check_device_flag()
    assert torch.isnan(y).all()
    desc[4] = 300
    g.run()
    g.check_device_flag()
    assert torch.isfinite(y).all()
