"""The dual-scale binary block on the GPU against the fp64 oracle (RaBiT
section 4.1: per-channel output scales h_k and input scales g_k,
W^_k = diag(h_k) B_k diag(g_k); section 4.2: paths derived in turn).

rb_pack_fixed: sign planes bit-exact except near-zero residuals (|R| at most
1e-6 of the entry's scale h_k[i] g_k[j]), counted against the 1e-6 bound.
rb_dual_gemv: kernel parity on the oracle's planes, |dy| <= 1e-3 * D with
D = sum_k sum_j |h_k x_k| (x_k the fp16 input the binary core sees).
"""
import numpy as np
import pytest
import torch

import oracle
import residual_binary_weight_b200 as rb
import synth
from gpu_util import planes_np, to_dev_planes

pytestmark = pytest.mark.gpu


def _scales(rng, N, M, K, with_g):
    h = (rng.uniform(0.5, 1.5, (N, M)) * 0.02 * 0.5 ** np.arange(N)[:, None]).astype(np.float32)
    g = rng.uniform(0.5, 1.5, (N, K)).astype(np.float32) if with_g else None
    return h, g


def _entry_scale(h, g, K):
    s = h.astype(np.float64)[:, :, None] * np.ones((1, 1, K))
    if g is not None:
        s = s * g.astype(np.float64)[:, None, :]
    return s


@pytest.mark.parametrize("order", ["rows", "sliced"])
@pytest.mark.parametrize("with_g", [True, False])
@pytest.mark.parametrize("N,M,K,wdt", [(1, 37, 640, np.float16), (2, 300, 4096, np.float16),
                                       (4, 129, 1152, np.float32), (3, 64, 128, np.float32)])
def test_pack_fixed_matches_oracle(N, M, K, wdt, with_g, order):
    rng = np.random.default_rng(N * 1000 + M + K)
    W = (rng.standard_normal((M, K)) * 0.02).astype(wdt)
    W[0, :7] = 0.0
    h, g = _scales(rng, N, M, K, with_g)
    planes = rb.pack_fixed(torch.from_numpy(W).cuda(), torch.from_numpy(h).cuda(),
                           torch.from_numpy(g).cuda() if g is not None else None, order=order)
    torch.cuda.synchronize()
    ref, rabs = oracle.pack_fixed(W, h, g, want_rabs=True)
    rep = oracle.compare_planes(planes_np(planes, K), ref, rabs, _entry_scale(h, g, K))
    assert rep.ok, rep
    if order == "sliced" and K % 512:
        q = planes.cpu().numpy().view(np.uint32)
        assert np.all(q[:, -1, :, (K // 32) % 16:] == 0)


def test_pack_fixed_full_size():
    """A Llama-2-7B-shaped gate matrix (11008 x 4096, config-2 distribution)
    with 2 paths, learned-scale stand-ins h (mean |W| per row, then half of
    it) and g (uniform 0.5..1.5), every row against the oracle."""
    wl = synth.WORKLOADS["llama2_7b_decode"]
    W = synth.device_weight(wl, 0, "gate", "cuda")
    rng = np.random.default_rng(77)
    m1 = W.float().abs().mean(1).cpu().numpy()
    h = np.stack([m1, 0.5 * m1]).astype(np.float32)
    g = rng.uniform(0.5, 1.5, (2, W.shape[1])).astype(np.float32)
    planes = rb.pack_fixed(W, torch.from_numpy(h).cuda(), torch.from_numpy(g).cuda(), order="sliced")
    torch.cuda.synchronize()
    Wh = W.cpu().numpy()
    P = planes_np(planes, W.shape[1])
    flipped = bad = 0
    for r0 in range(0, W.shape[0], 2048):
        r1 = min(W.shape[0], r0 + 2048)
        ref, rabs = oracle.pack_fixed(Wh[r0:r1], h[:, r0:r1], g, want_rabs=True)
        rep = oracle.compare_planes(P[:, r0:r1], ref, rabs, _entry_scale(h[:, r0:r1], g, W.shape[1]))
        flipped += rep.flipped
        bad += rep.bad
    total = oracle.compare.PlaneReport(W.shape[0] * W.shape[1], flipped, bad)
    print(f"{flipped} allowed flips in {total.entries} entries")
    assert total.ok, total


@pytest.mark.parametrize("order", ["rows", "sliced"])
@pytest.mark.parametrize("with_g", [True, False])
@pytest.mark.parametrize("N,M,K,T", [(2, 300, 4096, 1), (1, 33, 640, 3), (4, 129, 1152, 16), (2, 1000, 28672, 2),
                                     (3, 514, 384, 64)])
def test_dual_gemv_matches_oracle(N, M, K, T, with_g, order):
    rng = np.random.default_rng(N * 7 + M + K + T)
    W = (rng.standard_normal((M, K)) * 0.02).astype(np.float16)
    h, g = _scales(rng, N, M, K, with_g)
    ref, _ = oracle.pack_fixed(W, h, g)
    x = rng.standard_normal((T, K)).astype(np.float16)
    x[:, ::53] *= 20
    y_ref, den = oracle.dual_matvec(ref, h, oracle.dual_inputs(g, x, N))
    for y_dtype, ldx_pad, ldy_pad in ((torch.float16, 0, 0), (torch.float32, 8, 3)):
        xt = torch.zeros((T, K + ldx_pad), dtype=torch.float16)
        xt[:, :K] = torch.from_numpy(x)
        xd = xt.cuda()[:, :K]
        yd = torch.full((T, M + ldy_pad), float("nan"), dtype=y_dtype, device="cuda")
        rb.dual_gemv(to_dev_planes(ref, order=order), torch.from_numpy(h).cuda(),
                     torch.from_numpy(g).cuda() if g is not None else None, xd, y=yd[:, :M], check_device=True)
        yh = yd.float().cpu().numpy()
        if ldy_pad:
            assert np.all(np.isnan(yh[:, M:])), "wrote past the row"
        nbad, worst = oracle.compare_outputs(yh[:, :M], y_ref, den)
        assert nbad == 0, (y_dtype, worst)


def test_dual_gemv_with_mean_abs_scales_is_the_analytical_layer():
    """g = None and h = the analytical scales: the dual block is the layer
    rb_gemv evaluates (same planes, same scales); both within tolerance of
    the oracle."""
    wl = synth.WORKLOADS["llama2_7b_decode"]
    W = synth.host_rows(wl, 0, "q", range(256))
    x = synth.host_activations(wl, 0, "q", 2)
    ref, alpha, _ = oracle.pack(W, 2, 0)
    h = alpha[:, :, 0].astype(np.float32)
    pf, _ = oracle.pack_fixed(W, h)
    y_ref, den = oracle.dual_matvec(pf, h, oracle.dual_inputs(None, x, 2))
    planes = to_dev_planes(pf, order="sliced")
    yd = rb.dual_gemv(planes, torch.from_numpy(h).cuda(), None, torch.from_numpy(x).cuda(), y_dtype=torch.float32,
                      check_device=True)
    yg = rb.gemv(planes, torch.from_numpy(h[:, :, None].copy()).cuda(), torch.from_numpy(x).cuda(),
                 y_dtype=torch.float32)
    for y in (yd, yg):
        nbad, worst = oracle.compare_outputs(y.cpu().numpy(), y_ref, den)
        assert nbad == 0, worst
