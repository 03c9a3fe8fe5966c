"""rb_gemv / rb_gemv_grouped on the GPU against the fp64 oracle.

Kernel parity: the oracle packs the weight, and the GPU and the oracle both
evaluate those planes and stored scales on the same x, so no oracle input
comes from the GPU. Outputs must be within 1e-3 * sum_k sum_j |alpha_k x_j|.
"""
import numpy as np
import pytest
import torch

import oracle
import residual_binary_weight_b200 as rb
import synth
from gpu_util import check_gemv_on_oracle_planes, planes_np, to_dev_planes

pytestmark = pytest.mark.gpu


def _ok(res, what):
    nbad, worst = res
    assert nbad == 0, (what, worst)
    assert worst < 1e-3


def test_layer256_full():
    wl = synth.WORKLOADS["layer256"]
    W = synth.host_weight(wl, 0, "w")
    x = synth.host_activations(wl, 0, "w", 1)
    _ok(check_gemv_on_oracle_planes(W, x, 2, 0, alpha_f16=False), "layer256")


ORDERS = ["rows", "sliced"]


@pytest.mark.parametrize("order", ORDERS)
@pytest.mark.parametrize("matrix,rows,T", [("q", 1000, 1), ("gate", 700, 2), ("down", 300, 3)])
def test_llama2_shapes(matrix, rows, T, order):
    wl = synth.WORKLOADS["llama2_7b_decode"]
    W = synth.host_rows(wl, 1, matrix, range(rows))
    x = synth.host_activations(wl, 1, matrix, T)
    _ok(check_gemv_on_oracle_planes(W, x, 2, 0, alpha_f16=False, order=order), matrix)


@pytest.mark.parametrize("order", ORDERS)
@pytest.mark.parametrize("T", [1, 4, 16])
@pytest.mark.parametrize("matrix,rows", [("up", 200), ("down", 150)])
def test_qbb_g128(matrix, rows, T, order):
    wl = synth.WORKLOADS["qbb_g128"]
    W = synth.host_rows(wl, 0, matrix, range(rows))
    x = synth.host_activations(wl, 0, matrix, T)
    _ok(check_gemv_on_oracle_planes(W, x, 4, 128, alpha_f16=True, order=order), (matrix, T))


@pytest.mark.parametrize("order", ORDERS)
@pytest.mark.parametrize("n_paths", [1, 3, 5, 6, 8])
@pytest.mark.parametrize("group", [0, 128])
def test_path_counts(n_paths, group, order):
    rng = np.random.default_rng(7 * n_paths + group)
    W = (rng.standard_normal((333, 1152)) * 0.02).astype(np.float16)
    x = rng.standard_normal((2, 1152)).astype(np.float16)
    _ok(check_gemv_on_oracle_planes(W, x, n_paths, group, alpha_f16=(group == 128), order=order),
        (n_paths, group))


@pytest.mark.parametrize("alpha_f16,y_dtype", [(True, torch.float32), (False, torch.float32), (True, torch.float16)])
def test_dtypes_and_pitches(alpha_f16, y_dtype):
    rng = np.random.default_rng(3)
    W = (rng.standard_normal((96, 640)) * 0.02).astype(np.float16)
    x = rng.standard_normal((3, 640)).astype(np.float16)
    _ok(check_gemv_on_oracle_planes(W, x, 2, 0, alpha_f16, y_dtype, ldx_pad=8, ldy_pad=5), "pitch")
    _ok(check_gemv_on_oracle_planes(W, x, 2, 128, alpha_f16, y_dtype, ldx_pad=8, ldy_pad=3), "pitch g128")


@pytest.mark.parametrize("order", ORDERS)
@pytest.mark.parametrize("K", [128, 384, 640])
def test_small_and_ragged(K, order):
    rng = np.random.default_rng(K)
    for M in (1, 33, 514):
        W = (rng.standard_normal((M, K)) * 0.02).astype(np.float32)
        x = rng.standard_normal((1, K)).astype(np.float16)
        _ok(check_gemv_on_oracle_planes(W, x, 2, 0, False, order=order), (M, K))
        _ok(check_gemv_on_oracle_planes(W, x, 2, 128, False, order=order), (M, K, 128))


@pytest.mark.parametrize("order", ORDERS)
def test_split_k_single_matrix(order):
    """Few rows and long rows: the single-matrix plan splits K into chunks and
    the last CTA of a row block adds the partial sums."""
    rng = np.random.default_rng(11)
    W = (rng.standard_normal((64, 28672)) * 0.02).astype(np.float16)
    x = rng.standard_normal((1, 28672)).astype(np.float16)
    _ok(check_gemv_on_oracle_planes(W, x, 2, 0, False, order=order), "split")
    _ok(check_gemv_on_oracle_planes(W, x, 4, 128, True, order=order), "split g128")


def test_x_equal_one_and_unit_vectors():
    """Closed forms through the GPU path: x = 1 gives alpha-weighted popcounts,
    x = e_j extracts column j of the reconstructed weight."""
    rng = np.random.default_rng(17)
    M, K = 40, 512
    W = (rng.standard_normal((M, K)) * 0.02).astype(np.float32)
    ref_p, ref_a, _ = oracle.pack(W, 2, 0)
    a32 = ref_a.astype(np.float32)
    ones = np.ones((1, K), dtype=np.float16)
    y = rb.gemv(to_dev_planes(ref_p), torch.from_numpy(a32).cuda(), torch.from_numpy(ones).cuda(),
                y_dtype=torch.float32).cpu().numpy()[0]
    pc = np.array([[sum(int(w).bit_count() for w in ref_p[k, i]) for i in range(M)] for k in range(2)])
    exp = (a32.astype(np.float64)[:, :, 0] * (2 * pc - K)).sum(0)
    assert np.allclose(y, exp, rtol=0, atol=1e-5 * np.abs(a32).sum(0).max() * K)
    for j in (0, 37, 511):
        e = np.zeros((1, K), dtype=np.float16)
        e[0, j] = 1.0
        y = rb.gemv(to_dev_planes(ref_p), torch.from_numpy(a32).cuda(), torch.from_numpy(e).cuda(),
                    y_dtype=torch.float32).cpu().numpy()[0]
        col = sum(a32[k, :, 0].astype(np.float64) * np.where((ref_p[k, :, j // 32] >> (j % 32)) & 1, 1.0, -1.0)
                  for k in range(2))
        assert np.allclose(y, col, rtol=1e-6, atol=1e-9)


def _grouped_case(wl_name, layer, scale_rows, T, n_paths, group, alpha_f16, order="rows"):
    wl = synth.WORKLOADS[wl_name]
    items, refs = [], []
    for spec in wl.matrices:
        M = max(1, spec.M // scale_rows)
        W = synth.host_rows(wl, layer, spec.name, range(M))
        x = synth.host_activations(wl, layer, spec.name, T)
        ref_p, ref_a, _ = oracle.pack(W, n_paths, group)
        stored = oracle.alpha_to_f16(ref_a) if alpha_f16 else ref_a.astype(np.float32)
        y_ref, den = oracle.matvec(ref_p, stored.astype(np.float64), x.astype(np.float64))
        y = torch.full((T, M), float("nan"), dtype=torch.float16, device="cuda")
        items.append((to_dev_planes(ref_p, order=order), torch.from_numpy(stored).cuda(),
                      torch.from_numpy(x).cuda(), y))
        refs.append((y_ref, den))
    return items, refs


@pytest.mark.parametrize("order", ORDERS)
@pytest.mark.parametrize("T", [1, 2])
def test_grouped_llama2_layer(T, order):
    items, refs = _grouped_case("llama2_7b_decode", 2, 8, T, 2, 0, False, order)
    g = rb.GroupedGemv(items, n_paths=2, group=0, T=T)
    for _ in range(2):              # the arrival counters are cleared on every call
        for it in items:
            it[3].fill_(float("nan"))
        g.run()
        torch.cuda.synchronize()
        g.check_device_flag()
        for (_, _, _, y), (y_ref, den) in zip(items, refs):
            nbad, worst = oracle.compare_outputs(y.float().cpu().numpy(), y_ref, den)
            assert nbad == 0, worst


@pytest.mark.parametrize("order", ORDERS)
def test_grouped_qbb_g128(order):
    items, refs = _grouped_case("qbb_g128", 0, 16, 1, 4, 128, True, order)
    g = rb.GroupedGemv(items, n_paths=4, group=128, T=1)
    g.run()
    torch.cuda.synchronize()
    g.check_device_flag()
    for (_, _, _, y), (y_ref, den) in zip(items, refs):
        nbad, worst = oracle.compare_outputs(y.float().cpu().numpy(), y_ref, den)
        assert nbad == 0, worst


def test_grouped_output_in_pinned_host_memory():
    """y given as pinned host tensors: the launch writes the rows over the bus
    and they equal the oracle's (and the device-y run's)."""
    items, refs = _grouped_case("llama2_7b_decode", 1, 16, 1, 2, 0, False, "sliced")
    host_items = [(p, a, x, torch.empty(y.shape, dtype=y.dtype, pin_memory=True).fill_(float("nan")))
                  for p, a, x, y in items]
    g = rb.GroupedGemv(host_items, n_paths=2, group=0, T=1)
    g.run()
    torch.cuda.synchronize()
    g.check_device_flag()
    gd = rb.GroupedGemv(items, n_paths=2, group=0, T=1)
    gd.run()
    torch.cuda.synchronize()
    for (_, _, _, yh), (_, _, _, yd), (y_ref, den) in zip(host_items, items, refs):
        assert torch.equal(yh, yd.cpu())
        nbad, worst = oracle.compare_outputs(yh.float().numpy(), y_ref, den)
        assert nbad == 0, worst


@pytest.mark.parametrize("T", [1, 2])
def test_grouped_input_and_output_in_pinned_host_memory(T):
    """x and y given as pinned host tensors (zero-copy): the launch reads x and
    writes y over the bus, and y equals the device run's and the oracle's."""
    items, refs = _grouped_case("llama2_7b_decode", 1, 16, T, 2, 0, False, "sliced")
    host_items = [(p, a, x.cpu().pin_memory(), torch.empty(y.shape, dtype=y.dtype, pin_memory=True).fill_(float("nan")))
                  for p, a, x, y in items]
    g = rb.GroupedGemv(host_items, n_paths=2, group=0, T=T)
    g.run()
    torch.cuda.synchronize()
    g.check_device_flag()
    gd = rb.GroupedGemv(items, n_paths=2, group=0, T=T)
    gd.run()
    torch.cuda.synchronize()
    for (_, _, _, yh), (_, _, _, yd), (y_ref, den) in zip(host_items, items, refs):
        assert torch.equal(yh, yd.cpu())
        nbad, worst = oracle.compare_outputs(yh.float().numpy().reshape(y_ref.shape), y_ref, den)
        assert nbad == 0, worst


@pytest.mark.parametrize("order", ORDERS)
def test_grouped_many_units_per_cta(order):
    """The largest grouped launch (2047 descriptors) of small matrices at
    T = 16: ~220 units per CTA, more than the 128 unit records a CTA holds at
    once, so the records are refilled while the CTA runs (and some units are
    K-split)."""
    rng = np.random.default_rng(23)
    items, refs = [], []
    T = 16
    for i in range(2047):
        M = int(rng.integers(1, 70))
        K = int(rng.choice([128, 256, 640, 6656]) if i % 50 == 0 else rng.choice([128, 256, 640]))
        W = (rng.standard_normal((M, K)) * 0.02).astype(np.float16)
        x = rng.standard_normal((T, K)).astype(np.float16)
        ref_p, ref_a, _ = oracle.pack(W, 2, 0)
        a32 = ref_a.astype(np.float32)
        y_ref, den = oracle.matvec(ref_p, a32.astype(np.float64), x.astype(np.float64))
        y = torch.full((T, M), float("nan"), dtype=torch.float16, device="cuda")
        items.append((to_dev_planes(ref_p, order=order), torch.from_numpy(a32).cuda(),
                      torch.from_numpy(x).cuda(), y))
        refs.append((y_ref, den))
    g = rb.GroupedGemv(items, n_paths=2, group=0, T=T)
    g.run()
    torch.cuda.synchronize()
    g.check_device_flag()
    for (_, _, _, y), (y_ref, den) in zip(items, refs):
        nbad, worst = oracle.compare_outputs(y.float().cpu().numpy(), y_ref, den)
        assert nbad == 0, worst


def test_full_size_layer_sampled_rows():
    """One full Llama-2-7B-shaped layer (7 matrices) drawn on the device,
    packed in the sliced order and evaluated by one grouped launch (the
    bench's configuration). For 48 sampled rows per
    matrix the oracle packs the host copy of the weight row; the GPU planes of
    those rows must match, and after the rows are replaced by the oracle's
    planes and scales, the GPU outputs must match the oracle's."""
    wl = synth.WORKLOADS["llama2_7b_decode"]
    rng = np.random.default_rng(2)
    items, checks = [], []
    for spec in wl.matrices:
        W = synth.device_weight(wl, 0, spec.name, "cuda")
        x = synth.device_activations(wl, 0, spec.name, 1, "cuda")
        planes, alpha, _ = rb.pack(W, 2, 0, order="sliced")       # [N, S, M, 16]
        rows = np.sort(rng.choice(spec.M, 48, replace=False))
        idx = torch.from_numpy(rows).cuda()
        Wr = W.index_select(0, idx).cpu().numpy()
        ref_p, ref_a, rabs = oracle.pack(Wr, 2, 0, want_rabs=True)
        rep = oracle.compare_planes(planes_np(planes[:, :, idx], spec.K), ref_p, rabs, ref_a)
        print(f"{spec.name}: {rep.flipped} allowed flips in {rep.entries} sampled entries")
        assert rep.ok, (spec.name, rep)
        assert oracle.compare_scales(alpha[:, idx].cpu().numpy(), ref_a)[0] == 0
        planes[:, :, idx] = to_dev_planes(ref_p, order="sliced")
        a32 = ref_a.astype(np.float32)
        alpha[:, idx] = torch.from_numpy(a32).cuda()
        del W
        y = torch.empty((1, spec.M), dtype=torch.float16, device="cuda")
        items.append((planes, alpha, x, y))
        y_ref, den = oracle.matvec(ref_p, a32.astype(np.float64), x.cpu().numpy().astype(np.float64))
        checks.append((idx, y_ref, den))
    g = rb.GroupedGemv(items, n_paths=2, group=0, T=1)
    g.run()
    torch.cuda.synchronize()
    g.check_device_flag()
    for (_, _, _, y), (idx, y_ref, den) in zip(items, checks):
        got = y[:, idx].float().cpu().numpy()
        nbad, worst = oracle.compare_outputs(got, y_ref, den)
        assert nbad == 0, worst


@pytest.mark.parametrize("T", [1, 4, 16, 64])
@pytest.mark.parametrize("matrix", ["attn", "up", "down"])
def test_llama3_full_size_sampled(matrix, T):
    """A full Llama-3-70B-shaped projection at batch T through the single-matrix
    launch (K split into chunks, partial sums reduced by the last CTA). The
    weight is drawn and packed on the device; 32 sampled rows get the oracle's
    planes and scales, and their outputs for every token (at most 16 sampled
    tokens) are checked against the oracle."""
    wl = synth.WORKLOADS["llama3_70b_decode"]
    spec = {m.name: m for m in wl.matrices}[matrix]
    W = synth.device_weight(wl, 0, matrix, "cuda")
    planes, alpha, _ = rb.pack(W, 2, 0, order="sliced")
    rng = np.random.default_rng(T + spec.M)
    rows = np.sort(rng.choice(spec.M, 32, replace=False))
    idx = torch.from_numpy(rows).cuda()
    Wr = W.index_select(0, idx).cpu().numpy()
    del W
    ref_p, ref_a, _ = oracle.pack(Wr, 2, 0)
    planes[:, :, idx] = to_dev_planes(ref_p, order="sliced")
    a32 = ref_a.astype(np.float32)
    alpha[:, idx] = torch.from_numpy(a32).cuda()
    x = synth.device_activations(wl, 0, matrix, T, "cuda")
    y = rb.gemv(planes, alpha, x)
    torch.cuda.synchronize()
    toks = np.sort(rng.choice(T, min(T, 16), replace=False))
    xs = x[torch.from_numpy(toks).cuda()].cpu().numpy().astype(np.float64)
    y_ref, den = oracle.matvec(ref_p, a32.astype(np.float64), xs)
    got = y[torch.from_numpy(toks).cuda()][:, idx].float().cpu().numpy()
    _ok(oracle.compare_outputs(got, y_ref, den), (matrix, T))


def _qbb_full(matrix):
    """The full QBB matrix drawn on the host, packed by the oracle; planes
    (sliced order) and fp16 scales uploaded."""
    wl = synth.WORKLOADS["qbb_g128"]
    W = synth.host_weight(wl, 0, matrix)
    ref_p, ref_a, _ = oracle.pack(W, 4, 128)
    a16 = oracle.alpha_to_f16(ref_a)
    return wl, ref_p, a16


@pytest.mark.parametrize("T", [1, 16])
def test_qbb_full_size_single_and_grouped(T):
    """Both QBB matrices (11008 x 4096, 4096 x 11008; 4 paths, fp16 scales per
    128 columns) at full size, every row, at batch 1 and 16: through the
    single-matrix launch and through one grouped launch of both."""
    items, refs = [], []
    for matrix in ("up", "down"):
        wl, ref_p, a16 = _qbb_full(matrix)
        x = synth.host_activations(wl, 0, matrix, T)
        toks = np.arange(T) if T <= 4 else np.array([0, 5, 10, 15])
        y_ref, den = oracle.matvec(ref_p, a16.astype(np.float64), x[toks].astype(np.float64))
        planes = to_dev_planes(ref_p, order="sliced")
        alpha = torch.from_numpy(a16).cuda()
        xd = torch.from_numpy(x).cuda()
        y = rb.gemv(planes, alpha, xd, group=128, check_device=True)
        nbad, worst = oracle.compare_outputs(y[torch.from_numpy(toks).cuda()].float().cpu().numpy(), y_ref, den)
        assert nbad == 0, (matrix, T, worst)
        yg = torch.full((T, ref_p.shape[1]), float("nan"), dtype=torch.float16, device="cuda")
        items.append((planes, alpha, xd, yg))
        refs.append((toks, y_ref, den))
    g = rb.GroupedGemv(items, n_paths=4, group=128, T=T)
    g.run()
    g.check_device_flag()
    for (_, _, _, yg), (toks, y_ref, den) in zip(items, refs):
        nbad, worst = oracle.compare_outputs(yg[torch.from_numpy(toks).cuda()].float().cpu().numpy(), y_ref, den)
        assert nbad == 0, (T, worst)


def test_workspace_reused_across_shapes_without_clearing():
    """A workspace zeroed once serves later calls of other shapes: every call
    that splits K leaves its arrival counters at zero again."""
    rng = np.random.default_rng(41)
    ws = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    R = 512   # rows per CTA for two paths
    for M, K, T in [(700, 8192, 3), (300, 6656, 1), (1100, 8192, 2), (700, 8192, 3)]:
        assert rb.gemv_workspace_bytes(M, K, 2, 0, T) > 256, "the case must split K"
        W = (rng.standard_normal((M, K)) * 0.02).astype(np.float16)
        x = rng.standard_normal((T, K)).astype(np.float16)
        ref_p, ref_a, _ = oracle.pack(W, 2, 0)
        y = rb.gemv(to_dev_planes(ref_p), torch.from_numpy(ref_a.astype(np.float32)).cuda(),
                    torch.from_numpy(x).cuda(), workspace=ws, check_device=True)
        y_ref, den = oracle.matvec(ref_p, ref_a.astype(np.float32).astype(np.float64), x.astype(np.float64))
        nbad, worst = oracle.compare_outputs(y.float().cpu().numpy(), y_ref, den)
        assert nbad == 0, (M, K, T, worst)
        n_ctr = -(-M // R) * T
        assert int(ws[256:256 + 4 * n_ctr].view(torch.int32).abs().sum()) == 0, "counters left non-zero"


def test_a_counter_left_non_zero_is_reported():
    """A workspace that was not zeroed (here: one counter set on the host)
    is reported by rb_gemv_check instead of passing silently."""
    rng = np.random.default_rng(42)
    M, K, T = 700, 8192, 1
    W = (rng.standard_normal((M, K)) * 0.02).astype(np.float16)
    ref_p, ref_a, _ = oracle.pack(W, 2, 0)
    planes, alpha = to_dev_planes(ref_p), torch.from_numpy(ref_a.astype(np.float32)).cuda()
    x = torch.from_numpy(rng.standard_normal((T, K)).astype(np.float16)).cuda()
    ws = torch.zeros(rb.gemv_workspace_bytes(M, K, 2, 0, T), dtype=torch.uint8, device="cuda")
    ws[256:260].view(torch.int32)[0] = 1000
    rb.gemv(planes, alpha, x, workspace=ws)
    with pytest.raises(rb.RbError, match="not zero"):
        rb.gemv(planes, alpha, x, workspace=ws, check_device=True)
    ws.zero_()
    rb.gemv(planes, alpha, x, workspace=ws, check_device=True)


@pytest.mark.parametrize("M,K,group", [(8192, 4096, 0), (700, 8192, 0), (1000, 4096, 128)])
def test_planes_rewritten_by_pack_right_before_the_matvec(M, K, group):
    """A single-matrix matvec is a dependent launch that starts while the
    previous kernel of its stream runs, and brings its first planes into L2
    before it waits for that kernel. An rb_pack that rewrites those very
    planes just before it, with no synchronisation in between, must still be
    seen: with two weights packed in turn into the same buffers, every
    result equals the same call made after a device synchronise (the kernel
    is deterministic, so bit for bit)."""
    g = torch.Generator(device="cuda").manual_seed(M + K + group)
    a16 = group == 128
    Ws = [(torch.randn(M, K, device="cuda", generator=g) * 0.02).half() for _ in range(2)]
    x = torch.randn(1, K, device="cuda", generator=g).half()
    planes, alpha, al16 = rb.pack(Ws[0], 2, group, alpha_f16=a16, order="sliced")
    sc = al16 if a16 else alpha
    ws = torch.zeros(max(16, rb.gemv_workspace_bytes(M, K, 2, group, 1)), dtype=torch.uint8, device="cuda")
    n = 6
    ys = [torch.empty(1, M, dtype=torch.float16, device="cuda") for _ in range(n)]
    torch.cuda.synchronize()
    for i in range(n):   # pack, then matvec at once: adjacent kernels of one stream
        rb.pack(Ws[i % 2], 2, group, alpha_f16=a16, order="sliced", planes=planes, alpha=alpha, alpha16=al16)
        rb.gemv(planes, sc, x, group=group, y=ys[i], workspace=ws)
    torch.cuda.synchronize()
    ref = []
    for w in range(2):
        rb.pack(Ws[w], 2, group, alpha_f16=a16, order="sliced", planes=planes, alpha=alpha, alpha16=al16)
        torch.cuda.synchronize()
        ref.append(rb.gemv(planes, sc, x, group=group, workspace=ws, check_device=True))
        torch.cuda.synchronize()
    assert not torch.equal(ref[0], ref[1])
    for i in range(n):
        assert torch.equal(ys[i], ref[i % 2]), i
