"""rb_gemv_noalloc: the matvec for callers that cannot allocate device memory.

Its scratch lives in a static device array instead of a caller workspace.
Through the C ABI it must give the same outputs as rb_gemv (within the
output tolerance used for every matvec test, 1e-3 * sum_k sum_j
|alpha_k x_j|), on two calls in a row (the shared array keeps the last
call's contents, so the second call checks that the counters are cleared).
This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import residual_binary_weight_b200 as rb
from residual_binary_weight_b200 import _lib

pytestmark = pytest.mark.gpu


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def test_noalloc_matches_workspace_entry_point():
    lib = _lib.load()
    rng = np.random.default_rng(2024)
    M, K, T = 700, 4096, 2          # few rows: the plan splits K, so the scratch is used
    W = (rng.standard_normal((M, K)) * 0.02).astype(np.float16)
    x = rng.standard_normal((T, K)).astype(np.float16)
    planes_h, alpha_h, _ = oracle.pack(W, 2, 0)
    a32 = alpha_h.astype(np.float32)
    y_ref, den = oracle.matvec(planes_h, a32.astype(np.float64), x.astype(np.float64))

    L = rb.layout(M, K, 2, 0, "sliced")
    assert lib.rb_gemv_workspace_bytes(L, T) > 256, "this case must use K-split scratch"
    from gpu_util import to_dev_planes
    planes = to_dev_planes(planes_h, order="sliced")
    alpha = torch.from_numpy(a32).cuda()
    xd = torch.from_numpy(x).cuda()
    y_ws = rb.gemv(planes, alpha, xd, group=0, y_dtype=torch.float32)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        y_na = torch.full((T, M), float("nan"), dtype=torch.float32, device="cuda")
        rc = lib.rb_gemv_noalloc(_ptr(planes), _ptr(alpha), _lib.RB_F32, L, _ptr(xd), K, T,
                                 _ptr(y_na), _lib.RB_F32, M, stream)
        assert rc == 0, lib.rb_last_error()
        torch.cuda.synchronize()
        got, want = y_na.cpu().numpy(), y_ws.cpu().numpy()
        assert np.all(np.isfinite(got)), call
        nbad, worst = oracle.compare_outputs(got, want.astype(np.float64), den)
        assert nbad == 0, (call, worst)
        nbad, worst = oracle.compare_outputs(got, y_ref, den)
        assert nbad == 0, (call, worst)
        # no kernel-side failure recorded in the static scratch
        assert lib.rb_gemv_check(None, stream) == 0, lib.rb_last_error()


def _shape_beyond_scratch(lib):
    """A layout whose K-split scratch is larger than the static 1 MiB array."""
    for n_paths in (1, 2, 4):
        for M in (1024, 2048, 3072, 4096, 6144, 8192, 12288, 16384):
            for T in (64, 32, 16):
                L = rb.layout(M, 8192, n_paths, 0, "sliced")
                if lib.rb_gemv_workspace_bytes(L, T) > (1 << 20):
                    return L, M, T
    return None


def test_noalloc_refuses_shapes_beyond_its_scratch():
    lib = _lib.load()
    found = _shape_beyond_scratch(lib)
    assert found is not None
    L, M, T = found
    p = ctypes.c_void_p(1 << 40)
    rc = lib.rb_gemv_noalloc(p, p, _lib.RB_F32, L, p, 8192, T, p, _lib.RB_F16, M, None)
    assert _lib.STATUS_NAMES[rc] == "RB_ERR_UNSUPPORTED"
    assert b"static array" in lib.rb_last_error()
