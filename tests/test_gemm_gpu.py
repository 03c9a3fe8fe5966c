"""rb_gemm (tcgen05 prefill kernel) on the GPU against the fp64 oracle.

As for the matvec, the oracle packs the weight and both sides evaluate the
same planes and stored scales on the same X; outputs must be within
1e-3 * sum_k sum_j |alpha_k x_j| per element.
"""
import numpy as np
import pytest
import torch

import oracle
import residual_binary_weight_b200 as rb
import synth
from gpu_util import planes_np, to_dev_planes

pytestmark = pytest.mark.gpu


def _run(W, X, n_paths, group, alpha_f16, order="rows", y_dtype=torch.float16, ldx_pad=0, ldy_pad=0):
    ref_p, ref_a, _ = oracle.pack(W, n_paths, group)
    stored = oracle.alpha_to_f16(ref_a) if alpha_f16 else ref_a.astype(np.float32)
    y_ref, den = oracle.matvec(ref_p, stored.astype(np.float64), X.astype(np.float64))
    T, K = X.shape
    M = W.shape[0]
    xt = torch.zeros((T, K + ldx_pad), dtype=torch.float16)
    xt[:, :K] = torch.from_numpy(X)
    Xd = xt.cuda()[:, :K]
    Yd = torch.full((T, M + ldy_pad), float("nan"), dtype=y_dtype, device="cuda")
    rb.gemm(to_dev_planes(ref_p, order=order), torch.from_numpy(stored).cuda(), Xd, group=group, Y=Yd[:, :M],
            check_device=True)
    Yh = Yd.float().cpu().numpy()
    if ldy_pad:
        assert np.all(np.isnan(Yh[:, M:])), "wrote past the row"
    return oracle.compare_outputs(Yh[:, :M], y_ref, den)


def _ok(res, what):
    nbad, worst = res
    assert nbad == 0, (what, worst)


@pytest.mark.parametrize("order", ["rows", "sliced"])
def test_small_two_paths(order):
    rng = np.random.default_rng(1)
    W = (rng.standard_normal((256, 512)) * 0.02).astype(np.float16)
    X = rng.standard_normal((300, 512)).astype(np.float16)          # one full and one partial token tile
    _ok(_run(W, X, 2, 0, False, order), order)


@pytest.mark.parametrize("M,K,T", [(1, 128, 1), (130, 128, 7), (200, 384, 257), (129, 640, 64)])
def test_ragged_shapes(M, K, T):
    rng = np.random.default_rng(M + K + T)
    W = (rng.standard_normal((M, K)) * 0.02).astype(np.float32)
    X = rng.standard_normal((T, K)).astype(np.float16)
    _ok(_run(W, X, 2, 0, False), (M, K, T))
    _ok(_run(W, X, 2, 0, False, "sliced"), (M, K, T, "sliced"))


@pytest.mark.parametrize("T", [130, 16])
@pytest.mark.parametrize("n_paths", [1, 2, 3, 4])
@pytest.mark.parametrize("group,alpha_f16", [(0, False), (0, True), (128, True)])
def test_paths_and_scales(n_paths, group, alpha_f16, T):
    rng = np.random.default_rng(10 * n_paths + group + T)
    W = (rng.standard_t(4, (260, 1024)) * 0.014).astype(np.float16)
    X = rng.standard_normal((T, 1024)).astype(np.float16)
    _ok(_run(W, X, n_paths, group, alpha_f16), (n_paths, group, alpha_f16, T))


@pytest.mark.parametrize("T", [16, 130])
def test_fp32_group_scales_are_refused(T):
    """With one scale per 128 columns the scales become fp16 operand values;
    fp32 scales would be rounded, so the call refuses them instead."""
    rng = np.random.default_rng(3)
    W = (rng.standard_normal((128, 256)) * 0.02).astype(np.float16)
    ref_p, ref_a, _ = oracle.pack(W, 2, 128)
    X = torch.from_numpy(rng.standard_normal((T, 256)).astype(np.float16)).cuda()
    with pytest.raises(rb.RbError, match="RB_ERR_UNSUPPORTED"):
        rb.gemm(to_dev_planes(ref_p), torch.from_numpy(ref_a.astype(np.float32)).cuda(), X, group=128)


def test_dtypes_and_pitches():
    rng = np.random.default_rng(5)
    W = (rng.standard_normal((160, 768)) * 0.02).astype(np.float16)
    X = rng.standard_normal((96, 768)).astype(np.float16)
    _ok(_run(W, X, 2, 0, False, y_dtype=torch.float32, ldx_pad=8, ldy_pad=3), "f32 out, pitches")
    _ok(_run(W, X, 4, 128, True, "sliced", ldx_pad=16, ldy_pad=1), "g128 pitches")
    # 300 tokens: 240-wide token tiles (A in shared memory), partial last tile
    X3 = rng.standard_normal((300, 768)).astype(np.float16)
    _ok(_run(W, X3, 2, 0, False, "sliced", ldx_pad=8, ldy_pad=5), "240-wide tiles, pitches")


def test_qbb_batch16():
    wl = synth.WORKLOADS["qbb_g128"]
    W = synth.host_rows(wl, 0, "down", range(256))
    X = synth.host_activations(wl, 0, "down", 16)
    _ok(_run(W, X, 4, 128, True, "sliced"), "qbb down T=16")


@pytest.mark.parametrize("matrix", ["up", "down"])
def test_prefill_full_size_sampled(matrix):
    """The 2048-token prefill block through a full 14336-wide projection.
    The weight is drawn on the device and packed by the GPU; 64 sampled rows
    are replaced by the oracle's planes and scales, and their outputs for 48
    sampled tokens are checked against the oracle."""
    wl = synth.WORKLOADS["prefill"]
    spec = {m.name: m for m in wl.matrices}[matrix]
    W = synth.device_weight(wl, 0, matrix, "cuda")
    planes, alpha, _ = rb.pack(W, 2, 0, order="sliced")
    rng = np.random.default_rng(9)
    rows = np.sort(rng.choice(spec.M, 64, replace=False))
    idx = torch.from_numpy(rows).cuda()
    Wr = W.index_select(0, idx).cpu().numpy()
    del W
    ref_p, ref_a, rabs = oracle.pack(Wr, 2, 0, want_rabs=True)
    rep = oracle.compare_planes(planes_np(planes[:, :, idx], spec.K), ref_p, rabs, ref_a)
    print(f"{matrix}: {rep.flipped} allowed flips in {rep.entries} sampled entries")
    assert rep.ok, rep
    planes[:, :, idx] = to_dev_planes(ref_p, order="sliced")
    a32 = ref_a.astype(np.float32)
    alpha[:, idx] = torch.from_numpy(a32).cuda()
    X = synth.device_activations(wl, 0, matrix, 2048, "cuda")
    Y = rb.gemm(planes, alpha, X, check_device=True)
    toks = np.sort(rng.choice(2048, 48, replace=False))
    Xs = X[torch.from_numpy(toks).cuda()].cpu().numpy().astype(np.float64)
    y_ref, den = oracle.matvec(ref_p, a32.astype(np.float64), Xs)
    got = Y[torch.from_numpy(toks).cuda()][:, idx].float().cpu().numpy()
    nbad, worst = oracle.compare_outputs(got, y_ref, den)
    assert nbad == 0, worst


@pytest.mark.parametrize("T", [1, 5, 16, 17, 33, 64, 100, 129, 241, 300, 481])
@pytest.mark.parametrize("n_paths,group", [(2, 0), (4, 0), (4, 128), (3, 128)])
def test_token_tile_widths(T, n_paths, group):
    """Every token-tile width (16..256, and 240 when it saves a wave) the
    launcher picks from T, with partial last token tiles."""
    rng = np.random.default_rng(T * 7 + n_paths)
    W = (rng.standard_normal((160, 512)) * 0.02).astype(np.float16)
    X = rng.standard_normal((T, 512)).astype(np.float16)
    _ok(_run(W, X, n_paths, group, group == 128, "sliced"), (T, n_paths, group))


@pytest.mark.parametrize("T", [1, 4, 16, 64])
@pytest.mark.parametrize("matrix", ["attn", "up", "down"])
def test_llama3_full_size_sampled(matrix, T):
    """The Llama-3-70B-shaped projections at batches 1, 4, 16 and 64 on the
    tensor-core path (the decode-batch kernel: stream-K over all SMs, partial
    tiles reduced through the workspace): weight drawn and packed on the device, 32 sampled rows replaced by
    the oracle's planes and scales, all tokens of those rows checked."""
    wl = synth.WORKLOADS["llama3_70b_decode"]
    spec = {m.name: m for m in wl.matrices}[matrix]
    W = synth.device_weight(wl, 0, matrix, "cuda")
    planes, alpha, _ = rb.pack(W, 2, 0, order="sliced")
    rng = np.random.default_rng(3 * T + spec.K)
    rows = np.sort(rng.choice(spec.M, 32, replace=False))
    idx = torch.from_numpy(rows).cuda()
    Wr = W.index_select(0, idx).cpu().numpy()
    del W
    ref_p, ref_a, _ = oracle.pack(Wr, 2, 0)
    planes[:, :, idx] = to_dev_planes(ref_p, order="sliced")
    a32 = ref_a.astype(np.float32)
    alpha[:, idx] = torch.from_numpy(a32).cuda()
    X = synth.device_activations(wl, 0, matrix, T, "cuda")
    Y = rb.gemm(planes, alpha, X, check_device=True)
    y_ref, den = oracle.matvec(ref_p, a32.astype(np.float64), X.cpu().numpy().astype(np.float64))
    got = Y[:, idx].float().cpu().numpy()
    nbad, worst = oracle.compare_outputs(got, y_ref, den)
    assert nbad == 0, worst


# --------------------------------------------------------------- reconstruct-once
def _run_rec(W, X, alpha_f16, order="rows", y_dtype=torch.float16, ldx_pad=0, ldy_pad=0):
    """Kernel parity of rb_gemm_reconstruct: the oracle reconstructs
    RN_fp16(sum_k alpha_k B_k) from its own planes and stored scales and
    multiplies in fp64 (BLAS); |dY| <= 1e-3 * |X| |W^|^T. Also returns the
    error against the unrounded layer relative to its own tolerance scale."""
    ref_p, ref_a, _ = oracle.pack(W, 2, 0)
    stored = oracle.alpha_to_f16(ref_a) if alpha_f16 else ref_a.astype(np.float32)
    Wr = oracle.reconstruct_f16(ref_p, stored.astype(np.float64))
    y_ref, den = oracle.dense_matvec(Wr, X.astype(np.float64))
    y_exact, den_exact = oracle.matvec(ref_p, stored.astype(np.float64), X.astype(np.float64))
    T, K = X.shape
    M = W.shape[0]
    xt = torch.zeros((T, K + ldx_pad), dtype=torch.float16)
    xt[:, :K] = torch.from_numpy(X)
    Xd = xt.cuda()[:, :K]
    Yd = torch.full((T, M + ldy_pad), float("nan"), dtype=y_dtype, device="cuda")
    rb.gemm(to_dev_planes(ref_p, order=order), torch.from_numpy(stored).cuda(), Xd, Y=Yd[:, :M], check_device=True,
            reconstruct=True)
    Yh = Yd.float().cpu().numpy()
    if ldy_pad:
        assert np.all(np.isnan(Yh[:, M:])), "wrote past the row"
    nbad, worst = oracle.compare_outputs(Yh[:, :M], y_ref, den)
    _, worst_exact = oracle.compare_outputs(Yh[:, :M], y_exact, den_exact)
    return nbad, worst, worst_exact


@pytest.mark.parametrize("T", [1, 16, 100, 130, 241, 300])
@pytest.mark.parametrize("alpha_f16,order", [(False, "rows"), (True, "sliced")])
def test_reconstruct_matches_oracle(T, alpha_f16, order):
    rng = np.random.default_rng(T + 3)
    W = (rng.standard_normal((260, 1024)) * 0.02).astype(np.float16)
    X = rng.standard_normal((T, 1024)).astype(np.float16)
    nbad, worst, worst_exact = _run_rec(W, X, alpha_f16, order)
    assert nbad == 0, worst
    # against the unrounded layer: within the fp16 rounding of the weights and output
    assert worst_exact < 2.0 ** -10, worst_exact


def test_reconstruct_pitches_and_fp32_output():
    rng = np.random.default_rng(8)
    W = (rng.standard_normal((333, 640)) * 0.02).astype(np.float32)
    X = rng.standard_normal((257, 640)).astype(np.float16)
    nbad, worst, _ = _run_rec(W, X, False, "sliced", torch.float32, ldx_pad=8, ldy_pad=3)
    assert nbad == 0, worst


def test_reconstruct_refuses_other_layouts():
    rng = np.random.default_rng(9)
    W = (rng.standard_normal((128, 256)) * 0.02).astype(np.float16)
    X = torch.from_numpy(rng.standard_normal((130, 256)).astype(np.float16)).cuda()
    for n_paths, group in ((3, 0), (2, 128)):
        p, a, _ = oracle.pack(W, n_paths, group)
        with pytest.raises(rb.RbError, match="RB_ERR_UNSUPPORTED"):
            rb.gemm(to_dev_planes(p), torch.from_numpy(oracle.alpha_to_f16(a)).cuda(), X, group=group,
                    reconstruct=True)


@pytest.mark.parametrize("matrix", ["up", "down"])
def test_reconstruct_prefill_full_size_sampled(matrix):
    """The 2048-token prefill block through a full 14336-wide projection with
    the reconstructed operand: 64 sampled rows get the oracle's planes and
    scales, and their outputs for 48 sampled tokens are checked against the
    oracle's reconstruction."""
    wl = synth.WORKLOADS["prefill"]
    spec = {m.name: m for m in wl.matrices}[matrix]
    W = synth.device_weight(wl, 0, matrix, "cuda")
    planes, alpha, _ = rb.pack(W, 2, 0, order="sliced")
    rng = np.random.default_rng(19)
    rows = np.sort(rng.choice(spec.M, 64, replace=False))
    idx = torch.from_numpy(rows).cuda()
    Wr = W.index_select(0, idx).cpu().numpy()
    del W
    ref_p, ref_a, _ = oracle.pack(Wr, 2, 0)
    planes[:, :, idx] = to_dev_planes(ref_p, order="sliced")
    a32 = ref_a.astype(np.float32)
    alpha[:, idx] = torch.from_numpy(a32).cuda()
    X = synth.device_activations(wl, 0, matrix, 2048, "cuda")
    Y = rb.gemm(planes, alpha, X, check_device=True, reconstruct=True)
    toks = np.sort(rng.choice(2048, 48, replace=False))
    Xs = X[torch.from_numpy(toks).cuda()].cpu().numpy().astype(np.float64)
    y_ref, den = oracle.dense_matvec(oracle.reconstruct_f16(ref_p, a32.astype(np.float64)), Xs)
    got = Y[torch.from_numpy(toks).cuda()][:, idx].float().cpu().numpy()
    nbad, worst = oracle.compare_outputs(got, y_ref, den)
    assert nbad == 0, worst
