"""rb_pack on the GPU against the fp64 oracle (planes, fp32 and fp16 scales)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import check_pack, planes_np

pytestmark = pytest.mark.gpu


def _ok(res, what):
    rep, nbad_a, worst_a, nbad16 = res
    assert rep.bad == 0 and rep.ok, (what, rep)
    assert nbad_a == 0, (what, worst_a)
    assert nbad16 == 0, what


@pytest.mark.parametrize("order", ["rows", "sliced"])
def test_layer256_full(order):
    wl = synth.WORKLOADS["layer256"]
    W = synth.host_weight(wl, 0, "w")
    assert W.dtype == np.float32
    _ok(check_pack(W, 2, 0, order=order), "layer256")


@pytest.mark.parametrize("order", ["rows", "sliced"])
@pytest.mark.parametrize("matrix,rows", [("q", 256), ("gate", 192), ("down", 160)])
def test_llama2_shapes_row_scales(matrix, rows, order):
    wl = synth.WORKLOADS["llama2_7b_decode"]
    spec = {m.name: m for m in wl.matrices}[matrix]
    W = synth.host_rows(wl, 3, matrix, range(rows))
    assert W.shape == (rows, spec.K)
    _ok(check_pack(W, 2, 0, order=order), matrix)


@pytest.mark.parametrize("order", ["rows", "sliced"])
@pytest.mark.parametrize("matrix,rows", [("up", 192), ("down", 96)])
def test_qbb_g128_four_paths(matrix, rows, order):
    wl = synth.WORKLOADS["qbb_g128"]
    W = synth.host_rows(wl, 0, matrix, range(rows))
    _ok(check_pack(W, 4, 128, order=order), matrix)


@pytest.mark.parametrize("matrix,rows", [("attn", 48), ("down", 24)])
def test_llama3_shapes(matrix, rows):
    wl = synth.WORKLOADS["llama3_70b_decode"]
    W = synth.host_rows(wl, 0, matrix, range(rows))
    _ok(check_pack(W, 2, 0), matrix)


@pytest.mark.parametrize("n_paths", [1, 3, 8])
@pytest.mark.parametrize("group", [0, 128])
def test_path_counts(n_paths, group):
    rng = np.random.default_rng(100 + n_paths)
    W = (rng.standard_normal((37, 640)) * 0.02).astype(np.float16)
    _ok(check_pack(W, n_paths, group), (n_paths, group))


@pytest.mark.parametrize("order", ["rows", "sliced"])
@pytest.mark.parametrize("K", [128, 384, 1152, 33280])
@pytest.mark.parametrize("group", [0, 128])
def test_ragged_and_minimum_shapes(K, group, order):
    """Small and ragged K, and K = 33280 (> 32768), which takes the
    one-CTA-per-row kernel instead of the word-per-thread one."""
    rng = np.random.default_rng(K)
    W = (rng.standard_normal((3, K)) * 0.05).astype(np.float32)
    _ok(check_pack(W, 2, group, order=order), (K, group))
    W1 = W[:1]
    _ok(check_pack(W1, 2, group, order=order), (1, K, group))


def test_row_pitch_and_fp32_groups():
    rng = np.random.default_rng(5)
    W = (rng.standard_normal((20, 512)) * 0.02).astype(np.float32)
    _ok(check_pack(W, 2, 128, ldw_pad=4), "fp32 g128 padded")
    W16 = W.astype(np.float16)
    _ok(check_pack(W16, 2, 0, ldw_pad=8), "fp16 row padded")
    # several rows per CTA in the word-per-thread kernel, with a row pitch
    Wl = (rng.standard_normal((37, 4096)) * 0.02).astype(np.float32)
    _ok(check_pack(Wl.astype(np.float16), 2, 0, ldw_pad=24, order="sliced"), "fp16 4096 padded")
    _ok(check_pack(Wl, 3, 0, ldw_pad=4), "fp32 4096 padded")


def test_zeros_negative_zeros_and_ties():
    W = np.zeros((4, 256), dtype=np.float32)
    W[1] = -0.0
    W[2, ::2] = 1.0
    W[2, 1::2] = -1.0          # R_1 = 0 exactly: every later plane is all +1
    W[3, :128] = np.linspace(-1, 1, 128)
    for group in (0, 128):
        planes, alpha, _ = __import__("residual_binary_weight_b200").pack(torch.from_numpy(W).cuda(), 3, group)
        p = planes_np(planes)
        ref_p, ref_a, rabs = oracle.pack(W, 3, group, want_rabs=True)
        assert np.array_equal(p[:, :3], ref_p[:, :3]), group
        assert np.all(p[:, 0] == 0xFFFFFFFF) and np.all(p[:, 1] == 0xFFFFFFFF)
        assert np.all(alpha.cpu().numpy()[:, :2] == 0.0)
        rep = oracle.compare_planes(p, ref_p, rabs, ref_a)
        assert rep.ok, rep


def test_full_size_sampled_rows():
    """Full 28672 x 8192 matrix drawn on the device, packed in one launch;
    64 sampled rows checked against the oracle on the host."""
    wl = synth.WORKLOADS["llama3_70b_decode"]
    W = synth.device_weight(wl, 0, "up", "cuda")
    import residual_binary_weight_b200 as rb
    planes, alpha, _ = rb.pack(W, 2, 0)
    torch.cuda.synchronize()
    rows = np.sort(np.random.default_rng(1).choice(W.shape[0], 64, replace=False))
    idx = torch.from_numpy(rows).cuda()
    Wr = W.index_select(0, idx).cpu().numpy()
    ref_p, ref_a, rabs = oracle.pack(Wr, 2, 0, want_rabs=True)
    got_p = planes_np(planes[:, idx])
    got_a = alpha[:, idx].cpu().numpy()
    rep = oracle.compare_planes(got_p, ref_p, rabs, ref_a)
    print(f"{rep.flipped} allowed flips in {rep.entries} sampled entries")
    assert rep.ok, rep
    assert oracle.compare_scales(got_a, ref_a)[0] == 0


@pytest.mark.parametrize("matrix", ["up", "down"])
def test_qbb_full_size_all_rows(matrix):
    """Both QBB matrices (11008 x 4096 and 4096 x 11008; 4 paths, one scale per
    128 columns, fp16 copies) drawn and packed at full size on the device in
    one launch, and every row checked against the oracle, in blocks of rows.
    The g128 kernel walks the groups in a grid-stride loop of at most
    8 CTAs x 8 warps x 8 groups per SM and pass (75,776 groups on 148 SMs);
    these matrices have 352,256 groups, so every pass is checked. The flip
    bound is applied to the whole matrix."""
    import residual_binary_weight_b200 as rb
    wl = synth.WORKLOADS["qbb_g128"]
    spec = {m.name: m for m in wl.matrices}[matrix]
    W = synth.device_weight(wl, 0, matrix, "cuda")
    planes, alpha, a16 = rb.pack(W, 4, 128, alpha_f16=True, order="sliced")
    torch.cuda.synchronize()
    M, K = spec.M, spec.K
    groups = M * (K // 128)
    per_pass = torch.cuda.get_device_properties(0).multi_processor_count * 8 * 8 * 8
    assert groups > 4 * per_pass
    Wh = W.cpu().numpy()
    del W
    P = planes_np(planes, K)
    A = alpha.cpu().numpy()
    A16 = a16.cpu().numpy()
    flipped = bad = 0
    step = 512
    for r0 in range(0, M, step):
        r1 = min(M, r0 + step)
        ref_p, ref_a, rabs = oracle.pack(Wh[r0:r1], 4, 128, want_rabs=True)
        rep = oracle.compare_planes(P[:, r0:r1], ref_p, rabs, ref_a)
        flipped += rep.flipped
        bad += rep.bad
        assert oracle.compare_scales(A[:, r0:r1], ref_a)[0] == 0, r0
        assert oracle.compare_scales_f16(A16[:, r0:r1], ref_a) == 0, r0
    total = oracle.compare.PlaneReport(M * K, flipped, bad)
    print(f"{matrix}: {flipped} allowed flips in {M * K} entries")
    assert total.ok, total
