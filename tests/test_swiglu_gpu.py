"""The gated MLP block on the GPU against the fp64 oracle: rb_gemv_swiglu
(h = silu(G x) * (U x) in one launch) and the chain y = D h (mlp_gemv).

Kernel parity on the oracle's planes and scales. The bounds are derived
from the arithmetic, from oracle quantities only:
  * g and u are fp32 sums whose error is below EPS_SUM of their tolerance
    scales Dg, Du (the matvec's fp32 rounding bound, with margin);
  * |silu'| <= 1.1 everywhere, so
        |h_gpu - h| <= (|silu(g)| + 1.1 dg) du + 1.1 |u| dg
    with dg = EPS_SUM Dg, du = EPS_SUM Du; the fp32 gate itself adds at most
    1e-6 |h|, and rounding h to fp16 on both sides at most 2^-10 |h|;
  * the down projection then adds its own 1e-3 Dd (the matvec bound) and
    sum_k sum_j alpha^D_kij |tol_h j| for the difference of its inputs.
"""
import numpy as np
import pytest
import torch

import oracle
import residual_binary_weight_b200 as rb
import synth
from gpu_util import to_dev_planes

pytestmark = pytest.mark.gpu

EPS_SUM = 1e-5


def h_tolerance(g, u, dg_scale, du_scale, rounded=True):
    dg, du = EPS_SUM * dg_scale, EPS_SUM * du_scale
    silu = oracle.silu_gate(g, 1.0)
    h = silu * u
    tol = (np.abs(silu) + 1.1 * dg) * du + 1.1 * np.abs(u) * dg + 1e-6 * np.abs(h) + 1e-30
    if rounded:
        tol += 2.0 ** -10 * np.abs(h)
    return tol


def _pair(rng, M, K, n, group, wdt=np.float16):
    Wg = (rng.standard_normal((M, K)) * 0.02).astype(wdt)
    Wu = (rng.standard_normal((M, K)) * 0.02).astype(wdt)
    pg, ag, _ = oracle.pack(Wg, n, group)
    pu, au, _ = oracle.pack(Wu, n, group)
    return np.concatenate([pg, pu]), np.concatenate([ag, au])


def _scales_dev(a, f16):
    return torch.from_numpy(oracle.alpha_to_f16(a) if f16 else a.astype(np.float32)).cuda()


def _stored(a, f16):
    return (oracle.alpha_to_f16(a) if f16 else a.astype(np.float32)).astype(np.float64)


def _check_h(h_gpu, planes, alpha_stored, x, rounded=True):
    h, g, u, dg, du = oracle.swiglu_matvec(planes, alpha_stored, x.astype(np.float64))
    ref = h.astype(np.float16).astype(np.float64) if rounded else h
    tol = h_tolerance(g, u, dg, du, rounded)
    err = np.abs(h_gpu.astype(np.float64) - ref)
    assert np.isfinite(h_gpu).all()
    assert (err <= tol).all(), float((err / tol).max())
    return h, tol


@pytest.mark.parametrize("order", ["rows", "sliced"])
@pytest.mark.parametrize("n,group,f16", [(1, 0, False), (2, 0, False), (2, 0, True), (4, 0, False),
                                         (2, 128, True), (4, 128, True)])
@pytest.mark.parametrize("M,K,T", [(300, 1024, 1), (300, 6144, 3), (130, 8192, 2)])
def test_swiglu_matches_oracle(n, group, f16, order, M, K, T):
    rng = np.random.default_rng(M + K + 7 * n + group + T)
    planes, alpha = _pair(rng, M, K, n, group)
    x = rng.standard_normal((T, K)).astype(np.float16)
    if K == 6144:
        x[:, rng.choice(K, 30, replace=False)] *= 20   # outlier channels
    h = rb.gemv_swiglu(to_dev_planes(planes, order=order), _scales_dev(alpha, f16), torch.from_numpy(x).cuda(),
                       group=group, check_device=True)
    _check_h(h.float().cpu().numpy(), planes, _stored(alpha, f16), x)


def test_swiglu_fp32_output_and_pitches():
    rng = np.random.default_rng(11)
    M, K, T = 333, 2048, 3
    planes, alpha = _pair(rng, M, K, 2, 0)
    x = rng.standard_normal((T, K)).astype(np.float16)
    xt = torch.zeros((T, K + 64), dtype=torch.float16)
    xt[:, :K] = torch.from_numpy(x)
    hbig = torch.full((T, M + 5), float("nan"), dtype=torch.float32, device="cuda")
    rb.gemv_swiglu(to_dev_planes(planes, order="sliced"), _scales_dev(alpha, False), xt.cuda()[:, :K],
                   h=hbig[:, :M], check_device=True)
    hh = hbig.cpu().numpy()
    assert np.isnan(hh[:, M:]).all(), "wrote past the row"
    _check_h(hh[:, :M], planes, _stored(alpha, False), x, rounded=False)


def test_swiglu_refuses_odd_and_too_many_paths():
    rng = np.random.default_rng(12)
    planes, alpha = _pair(rng, 128, 512, 1, 0)
    x = torch.from_numpy(rng.standard_normal((1, 512)).astype(np.float16)).cuda()
    with pytest.raises(ValueError):
        rb.gemv_swiglu(to_dev_planes(planes[:1]), _scales_dev(alpha[:1], False), x)
    big = np.concatenate([planes] * 5)            # 10 paths = 5 per matrix
    with pytest.raises(rb.RbError, match="RB_ERR_UNSUPPORTED"):
        rb.gemv_swiglu(to_dev_planes(big), _scales_dev(np.concatenate([alpha] * 5), False), x)


def _check_y(y_gpu, d_planes, d_alpha, h_or16, tol_h, group):
    y, dd = oracle.matvec(d_planes, d_alpha, h_or16)
    N, Md, G = d_alpha.shape[0], d_alpha.shape[1], d_alpha.shape[2]
    Kd = h_or16.shape[1]
    # sum_k sum_j alpha_kij tol_j, grouped by the scale groups of the columns
    tsum = tol_h.reshape(tol_h.shape[0], G, Kd // G).sum(2)            # [T, groups]
    prop = np.einsum("kmg,tg->tm", np.abs(d_alpha), tsum)
    bound = 1e-3 * dd * (1 + 1e-3) + prop
    err = np.abs(y_gpu.astype(np.float64) - y)
    assert (err <= bound).all(), float((err / bound).max())


@pytest.mark.parametrize("group,f16", [(0, False), (128, True)])
def test_mlp_chain_matches_oracle(group, f16):
    """y = D (silu(G x) * (U x)) through mlp_gemv: two launches, h in fp16."""
    rng = np.random.default_rng(21 + group)
    M, K, Md, T = 384, 2048, 256, 2
    planes, alpha = _pair(rng, M, K, 2, group)
    Wd = (rng.standard_normal((Md, M)) * 0.02).astype(np.float16)
    dp, da, _ = oracle.pack(Wd, 2, group)
    x = rng.standard_normal((T, K)).astype(np.float16)
    y, h = rb.mlp_gemv(to_dev_planes(planes, order="sliced"), _scales_dev(alpha, f16),
                       to_dev_planes(dp, order="sliced"), _scales_dev(da, f16), torch.from_numpy(x).cuda(),
                       group=group, check_device=True)
    h_exact, tol = _check_h(h.float().cpu().numpy(), planes, _stored(alpha, f16), x)
    _check_y(y.float().cpu().numpy(), dp, _stored(da, f16), h_exact.astype(np.float16).astype(np.float64), tol,
             group)


def test_mlp_llama2_7b_full_size():
    """The 7B MLP block at full size, T = 1: gate and up 11008 x 4096, down
    4096 x 11008, weights drawn on the device and packed by the oracle (all
    rows), every h and y element checked."""
    wl = synth.WORKLOADS["llama2_7b_decode"]
    W = {m: synth.device_weight(wl, 0, m, "cuda").cpu().numpy() for m in ("gate", "up", "down")}
    pg, ag, _ = oracle.pack(W["gate"], 2, 0)
    pu, au, _ = oracle.pack(W["up"], 2, 0)
    dp, da, _ = oracle.pack(W["down"], 2, 0)
    planes, alpha = np.concatenate([pg, pu]), np.concatenate([ag, au])
    x = synth.device_activations(wl, 0, "gate", 1, "cuda")
    xh = x.cpu().numpy()
    y, h = rb.mlp_gemv(to_dev_planes(planes, order="sliced"), _scales_dev(alpha, False),
                       to_dev_planes(dp, order="sliced"), _scales_dev(da, False), x, check_device=True)
    h_exact, tol = _check_h(h.float().cpu().numpy(), planes, _stored(alpha, False), xh)
    _check_y(y.float().cpu().numpy(), dp, _stored(da, False), h_exact.astype(np.float16).astype(np.float64), tol, 0)
