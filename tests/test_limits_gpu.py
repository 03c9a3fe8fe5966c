"""The largest sizes the entry points accept, against the oracle.

* K = 65536, the largest row one per-row scale covers: rb_pack takes its
  one-CTA-per-row kernel (K > 32768), the matvec splits K into chunks, and
  rb_gemm runs both its decode and its prefill kernels over 128 K-stages.
* T = 64, the largest batch rb_gemv and the decode rb_gemm take, and T = 65,
  the first the prefill kernel takes.
* M = 1: one row (a tile of 128 with 127 rows past M).
"""
import numpy as np
import pytest
import torch

import oracle
import residual_binary_weight_b200 as rb
from gpu_util import check_pack, to_dev_planes

pytestmark = pytest.mark.gpu


def _out(Y, ref_p, ref_a, X):
    y_ref, den = oracle.matvec(ref_p, ref_a.astype(np.float32).astype(np.float64), X.astype(np.float64))
    nbad, worst = oracle.compare_outputs(Y.float().cpu().numpy(), y_ref, den)
    assert nbad == 0, worst


def test_pack_and_evaluate_at_the_longest_row():
    rng = np.random.default_rng(65536)
    M, K = 130, 65536
    W = (rng.standard_normal((M, K)) * 0.02).astype(np.float16)
    rep, nbad_a, _, _ = check_pack(W, 2, 0, alpha_f16=False, order="sliced")
    assert rep.ok and nbad_a == 0, (rep, nbad_a)
    ref_p, ref_a, _ = oracle.pack(W, 2, 0)
    planes, alpha = to_dev_planes(ref_p, order="sliced"), torch.from_numpy(ref_a.astype(np.float32)).cuda()
    for T in (1, 3, 130):
        X = rng.standard_normal((T, K)).astype(np.float16)
        Xd = torch.from_numpy(X).cuda()
        _out(rb.gemm(planes, alpha, Xd, check_device=True), ref_p, ref_a, X)
        if T <= 64:
            _out(rb.gemv(planes, alpha, Xd, check_device=True), ref_p, ref_a, X)


@pytest.mark.parametrize("T", [64, 65])
def test_largest_decode_batch_and_first_prefill_block(T):
    rng = np.random.default_rng(T)
    M, K = 300, 2048
    W = (rng.standard_normal((M, K)) * 0.02).astype(np.float16)
    ref_p, ref_a, _ = oracle.pack(W, 2, 0)
    planes, alpha = to_dev_planes(ref_p), torch.from_numpy(ref_a.astype(np.float32)).cuda()
    X = rng.standard_normal((T, K)).astype(np.float16)
    Xd = torch.from_numpy(X).cuda()
    _out(rb.gemm(planes, alpha, Xd, check_device=True), ref_p, ref_a, X)
    if T <= 64:
        _out(rb.gemv(planes, alpha, Xd, check_device=True), ref_p, ref_a, X)


@pytest.mark.parametrize("group", [0, 128])
def test_single_row(group):
    rng = np.random.default_rng(1 + group)
    W = (rng.standard_normal((1, 1024)) * 0.02).astype(np.float16)
    rep, nbad_a, _, nbad16 = check_pack(W, 2, group, alpha_f16=True)
    assert rep.ok and nbad_a == 0 and nbad16 == 0, (rep, nbad_a, nbad16)
    ref_p, ref_a, _ = oracle.pack(W, 2, group)
    a16 = oracle.alpha_to_f16(ref_a)
    planes, alpha = to_dev_planes(ref_p), torch.from_numpy(a16).cuda()
    for T in (1, 16, 100):
        X = rng.standard_normal((T, 1024)).astype(np.float16)
        Xd = torch.from_numpy(X).cuda()
        y_ref, den = oracle.matvec(ref_p, a16.astype(np.float64), X.astype(np.float64))
        Y = rb.gemm(planes, alpha, Xd, group=group, check_device=True)
        assert oracle.compare_outputs(Y.float().cpu().numpy(), y_ref, den)[0] == 0
        if T <= 64:
            y = rb.gemv(planes, alpha, Xd, group=group, check_device=True)
            assert oracle.compare_outputs(y.float().cpu().numpy(), y_ref, den)[0] == 0
