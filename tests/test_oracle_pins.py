"""Pins of the fp64 oracle to facts that do not come from the oracle itself.

* brute force over every sign pattern and a scale search on short rows
  (the scale and sign choice are the least-squares optimum for one path,
  and every later path is the optimum for the residual the earlier ones left);
* hand-worked derivations and packed-word fixtures under tests/golden/;
* invariants the derivation implies (energy identity, orthogonality of the
  residual to the last sign plane, non-increasing residual norm);
* the N = 1 special case (plain sign binarisation with a mean-|w| scale);
* the matvec against a dense BLAS product, closed forms for x = 1 and x = e_j;
* population values for Gaussian and Student-t rows (quadrature, not sampling);
* the paper's storage ratios (RaBiT section 4.1 and 5, appendix D).
"""
import itertools
import math
import os

import numpy as np
import pytest

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _signs(planes):
    b = np.ascontiguousarray(planes, dtype="<u4").view(np.uint8)
    bits = np.unpackbits(b, axis=-1, bitorder="little").reshape(planes.shape[0], planes.shape[1], -1)
    return np.where(bits == 1, 1.0, -1.0)


def _residuals(W, planes, alpha, G):
    """R_k for k = 0..N rebuilt from the oracle's outputs (numpy, not the oracle)."""
    S = _signs(planes)
    N = S.shape[0]
    A = np.repeat(alpha, G, axis=2)
    R = [W.astype(np.float64)]
    for k in range(N):
        R.append(R[-1] - A[k] * S[k])
    return R


def _best_scale_objective(r, s):
    """min over a >= 0 of ||r - a s||^2 by a grid plus golden-section search."""
    hi = float(np.max(np.abs(r))) * 1.5 + 1e-12
    f = lambda a: float(np.sum((r - a * s) ** 2))
    grid = np.linspace(0.0, hi, 401)
    vals = np.array([f(a) for a in grid])
    m = int(np.argmin(vals))
    lo_, hi_ = grid[max(m - 1, 0)], grid[min(m + 1, len(grid) - 1)]
    g = (math.sqrt(5) - 1) / 2
    c, d = hi_ - g * (hi_ - lo_), lo_ + g * (hi_ - lo_)
    for _ in range(200):
        if f(c) < f(d):
            hi_ = d
        else:
            lo_ = c
        c, d = hi_ - g * (hi_ - lo_), lo_ + g * (hi_ - lo_)
    a = (lo_ + hi_) / 2
    return f(a), a


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_brute_force_one_path_is_optimal(seed):
    """(sign(r), mean|r|) attains the global least-squares optimum over all
    2^n sign patterns and every scale a >= 0 (n = 10 free columns; the other
    22 columns of the 32-column group are zero and cost a^2 each whatever
    their sign)."""
    rng = np.random.default_rng(seed)
    n = 10
    r = rng.standard_normal(n)
    r[3] = 0.0
    W = np.zeros((1, 32))
    W[0, :n] = r
    planes, alpha, _ = oracle.pack(W, 1, 32)
    s_or, a_or = _signs(planes)[0, 0], alpha[0, 0, 0]
    best, best_s = math.inf, None
    for bits in itertools.product((1.0, -1.0), repeat=n):
        s = np.concatenate([np.array(bits), np.ones(32 - n)])
        v, _ = _best_scale_objective(W[0], s)
        if v < best:
            best, best_s = v, s
    v_or = float(np.sum((W[0] - a_or * s_or) ** 2))
    assert v_or <= best * (1 + 1e-10) + 1e-14
    nz = r != 0
    assert np.all(best_s[:n][nz] == s_or[:n][nz])
    # on a dense 32-column row, no single sign flip (with its own best scale) does better
    base = np.tile(r, 4)[:32]
    planes, alpha, _ = oracle.pack(base[None, :], 1, 32)
    s0, a0 = _signs(planes)[0, 0], alpha[0, 0, 0]
    v0 = float(np.sum((base - a0 * s0) ** 2))
    for j in range(32):
        s2 = s0.copy()
        s2[j] = -s2[j]
        v2, _ = _best_scale_objective(base, s2)
        assert v0 <= v2 * (1 + 1e-12) + 1e-15


@pytest.mark.parametrize("seed", [4, 5])
def test_brute_force_each_path_fits_previous_residual(seed):
    """Path k+1 is the single-path optimum for R_k (sequential derivation)."""
    rng = np.random.default_rng(seed)
    n = 9
    W = np.zeros((1, 32))
    W[0, :n] = rng.standard_normal(n) * 0.02
    N = 3
    planes, alpha, _ = oracle.pack(W, N, 32)
    R = _residuals(W, planes, alpha, 32)
    S = _signs(planes)
    for k in range(N):
        r = R[k][0]
        best = math.inf
        for bits in itertools.product((1.0, -1.0), repeat=n):
            s = np.concatenate([np.array(bits), np.ones(32 - n)])
            v, _ = _best_scale_objective(r, s)
            best = min(best, v)
        v_or = float(np.sum((r - alpha[k, 0, 0] * S[k, 0]) ** 2))
        assert v_or <= best * (1 + 1e-9) + 1e-18, (k, v_or, best)


def _golden_lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield [p.strip() for p in line.split("|")]


def test_bit_layout_fixtures():
    rows = list(_golden_lines("bit_layout.txt"))
    assert len(rows) >= 8
    for name, vals, word in rows:
        w = np.array([float(v) for v in vals.split(",")])
        assert w.size == 32
        planes, alpha, _ = oracle.pack(w[None, :], 1, 0)
        assert int(planes[0, 0, 0]) == int(word, 16), name


def test_worked_examples():
    for name, vals, n, alphas, words in _golden_lines("worked_examples.txt"):
        w = np.array([float(v) for v in vals.split(",")])
        N = int(n)
        planes, alpha, _ = oracle.pack(w[None, :], N, 0)
        exp_a = [float(a) for a in alphas.split(",")]
        exp_w = [int(x, 16) for x in words.split(",")]
        assert np.allclose(alpha[:, 0, 0], exp_a, rtol=0, atol=1e-15), name
        assert [int(planes[k, 0, 0]) for k in range(N)] == exp_w, name


@pytest.mark.parametrize("group", [0, 128])
def test_energy_identity_and_orthogonality(group):
    wl = synth.WORKLOADS["llama2_7b_decode"]
    W = synth.host_weight(wl, 0, "q", M=16, K=512).astype(np.float64)
    N = 4
    planes, alpha, _ = oracle.pack(W, N, group)
    G = 512 if group == 0 else group
    R = _residuals(W, planes, alpha, G)
    S = _signs(planes)
    ng = 512 // G
    for k in range(N):
        e0 = (R[k].reshape(16, ng, G) ** 2).sum(-1)
        e1 = (R[k + 1].reshape(16, ng, G) ** 2).sum(-1)
        # ||R_k||^2 = ||R_{k-1}||^2 - G alpha_k^2 in every row / group
        assert np.allclose(e1, e0 - G * alpha[k] ** 2, rtol=1e-10, atol=1e-18)
        assert np.all(e1 <= e0 * (1 + 1e-12))
        # the residual is orthogonal to the sign plane it was reduced by
        dot = (R[k + 1] * S[k]).reshape(16, ng, G).sum(-1)
        assert np.all(np.abs(dot) <= 1e-10 * np.sqrt(e0 * G) + 1e-18)


def test_single_path_is_sign_binarisation():
    rng = np.random.default_rng(7)
    W = rng.standard_normal((8, 256)).astype(np.float32)
    W[0, :5] = 0.0
    W[1, :3] = -0.0
    planes, alpha, _ = oracle.pack(W, 1, 0)
    S = _signs(planes)[0]
    assert np.array_equal(S, np.where(W >= 0, 1.0, -1.0))
    assert np.allclose(alpha[0, :, 0], np.abs(W.astype(np.float64)).mean(1), rtol=1e-15)


def test_zero_rows_and_groups():
    W = np.zeros((3, 256))
    W[1, 128:] = np.linspace(-1, 1, 128)
    planes, alpha, _ = oracle.pack(W, 3, 128)
    assert np.all(planes[:, 0] == 0xFFFFFFFF)
    assert np.all(alpha[:, 0] == 0.0)
    assert np.all(alpha[:, 1, 0] == 0.0) and np.all(planes[:, 1, :4] == 0xFFFFFFFF)
    assert alpha[0, 1, 1] > 0


def test_groups_are_independent():
    rng = np.random.default_rng(9)
    W = rng.standard_normal((4, 512))
    p1, a1, _ = oracle.pack(W, 3, 128)
    W2 = W.copy()
    W2[:, 128:256] *= 7.0
    p2, a2, _ = oracle.pack(W2, 3, 128)
    keep = np.r_[0:4, 8:16]
    assert np.array_equal(p1[:, :, keep], p2[:, :, keep])
    assert np.array_equal(a1[:, :, [0, 2, 3]], a2[:, :, [0, 2, 3]])
    assert np.allclose(a2[:, :, 1], 7.0 * a1[:, :, 1], rtol=1e-14)


@pytest.mark.parametrize("group", [0, 128])
def test_matvec_against_dense_blas(group):
    rng = np.random.default_rng(11)
    M, K, N, T = 24, 384, 3, 5
    W = rng.standard_normal((M, K))
    planes, alpha, _ = oracle.pack(W, N, group)
    G = K if group == 0 else group
    x = rng.standard_normal((T, K))
    y, den = oracle.matvec(planes, alpha, x)
    What = (np.repeat(alpha, G, axis=2) * _signs(planes)).sum(0)      # [M, K]
    ref = x @ What.T
    assert np.allclose(y, ref, rtol=0, atol=1e-12 * np.abs(den).max())
    assert np.allclose(den, np.abs(x) @ np.repeat(alpha, G, axis=2).sum(0).T, rtol=1e-12)


def test_matvec_closed_forms():
    rng = np.random.default_rng(12)
    M, K, N = 10, 256, 2
    W = rng.standard_normal((M, K))
    planes, alpha, _ = oracle.pack(W, N, 128)
    # x = 1: y_i = sum_k sum_g alpha_k[i,g] (2 popcount(group bits) - 128)
    y, _ = oracle.matvec(planes, alpha, np.ones((1, K)))
    for i in range(M):
        acc = 0.0
        for k in range(N):
            for g in range(2):
                pc = sum(int(w).bit_count() for w in planes[k, i, 4 * g:4 * g + 4])
                acc += alpha[k, i, g] * (2 * pc - 128)
        assert abs(y[0, i] - acc) <= 1e-12 * abs(alpha[:, i]).sum() * K
    # x = e_j: the column j of W^
    for j in (0, 31, 32, 200, 255):
        e = np.zeros((1, K))
        e[0, j] = 1.0
        y, _ = oracle.matvec(planes, alpha, e)
        col = sum(alpha[k, :, j // 128] * np.where((planes[k, :, j // 32] >> (j % 32)) & 1, 1.0, -1.0)
                  for k in range(N))
        assert np.allclose(y[0], col, rtol=0, atol=1e-15)


def _gauss_pop_constants():
    from scipy import integrate
    a1 = math.sqrt(2 / math.pi)
    phi = lambda z: math.exp(-z * z / 2) / math.sqrt(2 * math.pi)
    # E| |Z| - a1 | for a standard normal Z
    a2 = integrate.quad(lambda z: abs(z - a1) * 2 * phi(z), 0, a1)[0] + \
        integrate.quad(lambda z: abs(z - a1) * 2 * phi(z), a1, np.inf)[0]
    return a1, a2


def test_gaussian_population_scales():
    a1, a2 = _gauss_pop_constants()
    assert abs(a1 - 0.797885) < 1e-6 and abs(a2 - 0.482624) < 1e-6
    wl = synth.WORKLOADS["llama3_70b_decode"]
    W = synth.host_weight(wl, 0, "attn", M=256, K=4096).astype(np.float64)
    planes, alpha, _ = oracle.pack(W, 2, 0)
    sigma = synth.configs.W_STD
    m1 = alpha[0].mean() / sigma
    m2 = alpha[1].mean() / sigma
    assert abs(m1 / a1 - 1) < 5e-3, m1
    assert abs(m2 / a2 - 1) < 5e-3, m2
    R = _residuals(W, planes, alpha, 4096)
    e0 = (W ** 2).sum()
    mse1 = (R[1] ** 2).sum() / e0
    mse2 = (R[2] ** 2).sum() / e0
    assert abs(mse1 - (1 - 2 / math.pi)) < 5e-3
    assert abs(mse2 - (1 - 2 / math.pi - a2 * a2)) < 5e-3


def test_student_t_population_scale():
    from scipy import stats
    e_abs = stats.t(4).expect(abs)
    assert abs(e_abs - 1.0) < 1e-9        # E|T_4| = 1
    wl = synth.WORKLOADS["qbb_g128"]
    W = synth.host_weight(wl, 0, "up", M=256, K=4096).astype(np.float64)
    planes, alpha, _ = oracle.pack(W, 4, 128)
    target = synth.configs.W_STD / math.sqrt(2.0) * e_abs
    assert abs(alpha[0].mean() / target - 1) < 1e-2
    assert np.all(np.diff(alpha.mean(axis=(1, 2))) < 0)


def test_storage_ratios_from_the_paper():
    """RaBiT: 8x smaller than FP16 at two paths (section 5), 32x per plane vs
    fp32 (appendix D), about 2.02 effective bits with per-channel vectors
    (section 4.1)."""
    M = K = 4096
    planes, alpha, _ = oracle.pack(np.ones((2, K)), 2, 0)
    words_per_row = planes.shape[2]
    plane_bytes = 2 * M * words_per_row * 4
    assert (M * K * 2) / plane_bytes == 8.0
    assert (M * K * 4) / (M * words_per_row * 4) == 32.0
    # two paths, an fp16 output-channel and input-channel vector per path
    bits = (plane_bytes * 8 + 2 * 16 * (M + K)) / (M * K)
    assert round(bits, 2) == 2.02


def test_compare_helpers_catch_plausible_mistakes():
    rng = np.random.default_rng(21)
    W = rng.standard_normal((8, 256))
    planes, alpha, rabs = oracle.pack(W, 2, 0, want_rabs=True)
    assert oracle.compare_planes(planes, planes, rabs, alpha).ok
    bad = planes.copy()
    bad[1, 3, 2] ^= 1 << 5
    assert not oracle.compare_planes(bad, planes, rabs, alpha).ok
    assert oracle.compare_scales(alpha * (1 + 2e-6), alpha)[0] > 0
    assert oracle.compare_scales(alpha * (1 + 5e-7), alpha)[0] == 0
    x = rng.standard_normal((2, 256))
    y, den = oracle.matvec(planes, alpha, x)
    # a transposed operand or a dropped path is far outside the tolerance
    y_drop, _ = oracle.matvec(planes[:1], alpha[:1], x)
    assert oracle.compare_outputs(y_drop, y, den)[0] > 0
    y_flip, _ = oracle.matvec(planes[::-1].copy(), alpha, x)
    assert oracle.compare_outputs(y_flip, y, den)[0] > 0
    assert oracle.compare_scales_f16(oracle.alpha_to_f16(alpha), alpha) == 0


def _runs_row(vals):
    """A 32-column row of four runs of 8 equal values."""
    return np.repeat(np.array(vals, dtype=np.float64), 8)


def test_rabs_is_the_magnitude_each_sign_was_taken_on():
    """rabs[k] = |R_{k-1}|, against hand values for rows C and D
    (tests/golden/residual_magnitudes.txt): recording it after the update
    (|R_k|) or only for the first path fails here."""
    rows = {name: vals for name, vals, *_ in _golden_lines("worked_examples.txt")}
    expected = {}
    for name, k, runs in _golden_lines("residual_magnitudes.txt"):
        expected.setdefault(name, {})[int(k)] = _runs_row([float(v) for v in runs.split(",")])
    assert set(expected) == {"C", "D"}
    for name, per_path in expected.items():
        w = np.array([float(v) for v in rows[name].split(",")])
        planes, alpha, rabs = oracle.pack(w[None, :], 3, 0, want_rabs=True)
        for k, want in per_path.items():
            assert np.array_equal(rabs[k - 1, 0], want), (name, k, rabs[k - 1, 0])


def _allowance_case():
    """1024 x 1024 weights (1,048,576 entries, so the count bound admits one
    flipped entry and not two), 3 paths, scale groups of 32 columns. Row 0
    group 0 is worked example D (exact ties at path 2), row 1 group 0 is
    example C (exact ties at path 3), row 2 group 0 holds 31 ones and one
    entry of 5e-7 (below 1e-6 * alpha1 = 9.7e-7), row 3 group 0 the same
    with 2e-6 (above it)."""
    rng = np.random.default_rng(31)
    W = rng.standard_normal((1024, 1024))
    rows = {name: vals for name, vals, *_ in _golden_lines("worked_examples.txt")}
    W[0, :32] = [float(v) for v in rows["D"].split(",")]
    W[1, :32] = [float(v) for v in rows["C"].split(",")]
    W[2, :32] = 1.0
    W[2, 5] = 5e-7
    W[3, :32] = 1.0
    W[3, 5] = 2e-6
    planes, alpha, rabs = oracle.pack(W, 3, 32, want_rabs=True)
    return planes, alpha, rabs


def _flip(p, k, i, j):
    p[k, i, j // 32] ^= np.uint32(1 << (j % 32))


def test_compare_planes_allowance_cascade_and_count_bound():
    """The lenient branches of the plane comparison, each with a case a
    plausible mistake would get wrong: an allowed flip is counted once even
    when later planes of the entry follow it (taking the last differing path
    instead of the first rejects it); a later-plane difference with no allowed
    flip before it fails; the threshold |R| <= 1e-6 * alpha is applied in the
    right direction; two flipped entries exceed the count bound."""
    ref, alpha, rabs = _allowance_case()
    assert alpha[1, 0, 0] == 0.5 and rabs[1, 0, 0] == 0.0 and rabs[2, 0, 0] == 0.5
    rep = oracle.compare_planes(ref.copy(), ref, rabs, alpha)
    assert (rep.flipped, rep.bad, rep.ok) == (0, 0, True)

    # D: the tie at path 2 flips, and path 3 follows it (the cascade)
    c = ref.copy()
    _flip(c, 1, 0, 3)
    _flip(c, 2, 0, 3)
    rep = oracle.compare_planes(c, ref, rabs, alpha)
    assert (rep.flipped, rep.bad, rep.ok) == (1, 0, True), rep

    # path 3 alone differs where |R_2| = 0.5: no earlier allowed flip, so it fails
    c = ref.copy()
    _flip(c, 2, 0, 3)
    rep = oracle.compare_planes(c, ref, rabs, alpha)
    assert (rep.flipped, rep.bad, rep.ok) == (0, 1, False), rep

    # the threshold: 5e-7 <= 1e-6 * alpha1 is allowed, 2e-6 is not
    a1 = alpha[0, 2, 0]
    assert 5e-7 <= 1e-6 * a1 < 2e-6
    c = ref.copy()
    _flip(c, 0, 2, 5)
    rep = oracle.compare_planes(c, ref, rabs, alpha)
    assert (rep.flipped, rep.bad, rep.ok) == (1, 0, True), rep
    c = ref.copy()
    _flip(c, 0, 3, 5)
    rep = oracle.compare_planes(c, ref, rabs, alpha)
    assert (rep.flipped, rep.bad, rep.ok) == (0, 1, False), rep

    # two allowed entries (D at path 2, C's exact tie at path 3 col 10):
    # 2 >= 1e-6 * 1,048,576, so the count bound fails
    c = ref.copy()
    _flip(c, 1, 0, 3)
    _flip(c, 2, 1, 10)
    rep = oracle.compare_planes(c, ref, rabs, alpha)
    assert (rep.flipped, rep.bad, rep.ok) == (2, 0, False), rep

    # a flip at an entry far from zero (D col 8 at path 1: |R_0| = 1)
    c = ref.copy()
    _flip(c, 0, 0, 8)
    rep = oracle.compare_planes(c, ref, rabs, alpha)
    assert rep.bad == 1 and not rep.ok


def test_compare_scales_f16_midpoint_branch():
    """Near an fp16 rounding midpoint either neighbour is accepted, elsewhere
    only the round-to-nearest-even value: 1 + 2^-11 lies half way between
    0x3C00 and 0x3C01."""
    def f16(bits):
        return np.array([bits], dtype=np.uint16).view(np.float16)

    mid = np.array([1.0 + 2.0 ** -11])
    assert oracle.compare_scales_f16(f16(0x3C00), mid) == 0
    assert oracle.compare_scales_f16(f16(0x3C01), mid) == 0
    for bad in (0x3C02, 0x3BFF, 0x0000):
        assert oracle.compare_scales_f16(f16(bad), mid) == 1, hex(bad)
    # within 1e-6 relative of the midpoint: still either neighbour
    near = mid * (1 + 5e-7)
    assert oracle.compare_scales_f16(f16(0x3C00), near) == 0
    assert oracle.compare_scales_f16(f16(0x3C01), near) == 0
    # 3e-6 above it: only the nearest value, 0x3C01
    above = mid * (1 + 3e-6)
    assert oracle.compare_scales_f16(f16(0x3C01), above) == 0
    assert oracle.compare_scales_f16(f16(0x3C00), above) == 1
    below = mid * (1 - 3e-6)
    assert oracle.compare_scales_f16(f16(0x3C00), below) == 0
    assert oracle.compare_scales_f16(f16(0x3C01), below) == 1


def test_alpha_to_f16_bit_patterns():
    """The stored fp16 scale copy, against hand-written IEEE half patterns:
    1/3 -> 0x3555, 0.1 -> 0x2E66, the largest finite half 0x7BFF, the
    smallest subnormal 0x0001, ties to even at 1 + 2^-11 (-> 0x3C00) and
    1 + 3 * 2^-11 (-> 0x3C02), and 1 + 2^-11 + 2^-40, just above the
    midpoint (-> 0x3C01; rounding through fp32 first would give 0x3C00)."""
    vals = np.array([1 / 3, 0.1, 65504.0, 2.0 ** -24, 1 + 2.0 ** -11, 1 + 3 * 2.0 ** -11,
                     1 + 2.0 ** -11 + 2.0 ** -40])
    want = [0x3555, 0x2E66, 0x7BFF, 0x0001, 0x3C00, 0x3C02, 0x3C01]
    got = oracle.alpha_to_f16(vals).view(np.uint16).tolist()
    assert got == want, [hex(g) for g in got]


# ---------------------------------------------------------------- dual-scale block
def test_pack_fixed_hand_worked_row():
    """tests/golden/fixed_scales.txt: words and |R_{k-1}| of a 4-path row with
    given output scales h and input scales g."""
    rows = list(_golden_lines("fixed_scales.txt"))
    assert len(rows) == 4
    W = np.repeat([3.0, -1.0], 16)[None, :]
    h = np.array([[float(r[1])] for r in rows])
    g = np.array([np.repeat([float(v) for v in r[2].split(",")], 16) for r in rows])
    planes, rabs = oracle.pack_fixed(W, h, g, want_rabs=True)
    for k, (_, _, _, word, ra) in enumerate(rows):
        assert int(planes[k, 0, 0]) == int(word, 16), k
        assert np.array_equal(rabs[k, 0], np.repeat([float(v) for v in ra.split(",")], 16)), k


@pytest.mark.parametrize("group", [0, 128])
def test_pack_fixed_with_mean_abs_scales_is_pack(group):
    """Given the scales the analytical derivation computes (mean |R|, g = 1),
    the fixed-scale derivation takes the same signs (pinned pack above)."""
    rng = np.random.default_rng(41)
    W = rng.standard_normal((12, 256)) * 0.02
    planes, alpha, _ = oracle.pack(W, 3, 0)
    pf, _ = oracle.pack_fixed(W, alpha[:, :, 0])
    assert np.array_equal(pf, planes)
    pf1, _ = oracle.pack_fixed(W, alpha[:, :, 0], np.ones((3, 256)))
    assert np.array_equal(pf1, planes)


def test_pack_fixed_energy_identity():
    """R_k = R_{k-1} - h g B with B = sign(R_{k-1}) gives, per row,
    sum R_k^2 = sum R_{k-1}^2 - 2 h sum g |R_{k-1}| + h^2 sum g^2 (R B = |R|):
    a dropped term, a wrong sign or a transposed g fails it."""
    rng = np.random.default_rng(42)
    M, K, N = 10, 192, 3
    W = rng.standard_normal((M, K))
    h = rng.uniform(0.1, 1.0, (N, M))
    g = rng.uniform(0.2, 2.0, (N, K))
    planes, rabs = oracle.pack_fixed(W, h, g, want_rabs=True)
    S = _signs(planes)
    R = W.copy()
    for k in range(N):
        assert np.allclose(np.abs(R), rabs[k], rtol=0, atol=1e-12)
        assert np.array_equal(S[k], np.where(R >= 0, 1.0, -1.0))
        Rn = R - h[k][:, None] * g[k][None, :] * S[k]
        lhs = (Rn ** 2).sum(1)
        rhs = (R ** 2).sum(1) - 2 * h[k] * (g[k][None, :] * np.abs(R)).sum(1) + h[k] ** 2 * (g[k] ** 2).sum()
        assert np.allclose(lhs, rhs, rtol=1e-12)
        R = Rn


def test_dual_inputs_round_to_fp16():
    """x_k = RN_fp16(g_k x): 1/3 * 1 -> 0x3555, 0.1 * 1 -> 0x2E66, 3 * (1/3 in fp64) -> 1.0."""
    g = np.array([[1 / 3, 0.1, 3.0]])
    x = np.array([[1.0, 1.0, 1 / 3]])
    xk = oracle.dual_inputs(g, x, 1)
    assert xk.astype(np.float16).view(np.uint16).tolist() == [[[0x3555, 0x2E66, 0x3C00]]]


def test_dual_matvec_against_blas_and_single_scale_matvec():
    rng = np.random.default_rng(43)
    M, K, N, T = 20, 256, 2, 3
    W = rng.standard_normal((M, K))
    h = rng.uniform(0.1, 1.0, (N, M))
    g = rng.uniform(0.2, 2.0, (N, K))
    planes, _ = oracle.pack_fixed(W, h, g)
    x = rng.standard_normal((T, K)).astype(np.float16).astype(np.float64)
    xk = oracle.dual_inputs(g, x, N)
    y, den = oracle.dual_matvec(planes, h, xk)
    S = _signs(planes)
    ref = sum(xk[k] @ (h[k][:, None] * S[k]).T for k in range(N))
    assert np.allclose(y, ref, rtol=0, atol=1e-12 * den.max())
    assert np.allclose(den, sum(np.abs(xk[k]) @ np.repeat(h[k][:, None], K, 1).T for k in range(N)), rtol=1e-12)
    # g = 1: the dual block is the single-scale layer with alpha_k = h_k (pinned matvec)
    y1, den1 = oracle.dual_matvec(planes, h, oracle.dual_inputs(None, x, N))
    y2, den2 = oracle.matvec(planes, h[:, :, None], x)
    assert np.allclose(y1, y2, rtol=0, atol=1e-12 * den2.max()) and np.allclose(den1, den2, rtol=1e-13)
    # x = e_j reads column j of sum_k h_k B_k g_k (with g_k[j] rounded as an fp16 activation)
    for j in (0, 100, 255):
        e = np.zeros((1, K))
        e[0, j] = 1.0
        ye, _ = oracle.dual_matvec(planes, h, oracle.dual_inputs(g, e, N))
        col = sum(h[k] * S[k][:, j] * float(np.float16(g[k, j])) for k in range(N))
        assert np.allclose(ye[0], col, rtol=0, atol=1e-14)


# ------------------------------------------------------------ reconstruct-once
def test_reconstruct_hand_values_and_single_rounding():
    """Two paths, scales (0.75, 0.25): the four weight values are +-1.0 and
    +-0.5 by sign pattern. And the sum is rounded once from its exact value:
    1 + 2^-11 + 2^-30 rounds up to 1 + 2^-10 (0x3C01); rounding through fp32
    first would land on the tie 1 + 2^-11 and give 0x3C00."""
    w = np.array([[1.0, 1.0, -1.0, -1.0] * 8])
    w2 = np.array([[1.0, -1.0, 1.0, -1.0] * 8])
    p1, _, _ = oracle.pack(w, 1, 0)
    p2, _, _ = oracle.pack(w2, 1, 0)
    planes = np.concatenate([p1, p2])
    alpha = np.array([[[0.75]], [[0.25]]])
    Wr = oracle.reconstruct_f16(planes, alpha)
    assert Wr.dtype == np.float16
    assert Wr[0, :4].tolist() == [1.0, 0.5, -0.5, -1.0]
    alpha = np.array([[[1 + 2.0 ** -11]], [[2.0 ** -30]]])
    ones = np.full((1, 1, 1), 0xFFFFFFFF, dtype=np.uint32)
    Wr = oracle.reconstruct_f16(np.concatenate([ones, ones]), alpha)
    assert Wr.view(np.uint16)[0, 0] == 0x3C01


def test_reconstruct_matches_the_paths_and_dense_matvec_is_blas():
    """Before rounding, W^ x equals sum_k alpha_k (B_k x) (the pinned matvec);
    after rounding each weight moves by at most half an fp16 ulp."""
    rng = np.random.default_rng(51)
    W = rng.standard_normal((16, 384)) * 0.02
    for group in (0, 128):
        planes, alpha, _ = oracle.pack(W, 2, group)
        Wr = oracle.reconstruct_f16(planes, alpha).astype(np.float64)
        exact = (np.repeat(alpha, 384 // alpha.shape[2], axis=2) * _signs(planes)).sum(0)
        assert np.all(np.abs(Wr - exact) <= np.abs(exact) * 2.0 ** -11 + 2.0 ** -25)
        x = rng.standard_normal((3, 384))
        y, den = oracle.dense_matvec(exact, x)
        y2, den2 = oracle.matvec(planes, alpha, x)
        assert np.allclose(y, y2, rtol=0, atol=1e-12 * den2.max())
        assert np.all(den <= den2 * (1 + 1e-12))


# ---------------------------------------------------------- SiLU-gated pair
def test_silu_gate_closed_forms():
    """silu(0) = 0; silu(ln 3) = (3/4) ln 3 (e^-ln3 = 1/3); the odd part
    silu(g) - silu(-g) = g; silu(g) -> g as g -> +inf and -> 0 as g -> -inf."""
    assert oracle.silu_gate(0.0, 5.0) == 0.0
    assert abs(oracle.silu_gate(np.log(3.0), 1.0) - 0.75 * np.log(3.0)) < 1e-15
    rng = np.random.default_rng(3)
    g = rng.standard_normal(1000) * 4
    u = rng.standard_normal(1000)
    assert np.allclose(oracle.silu_gate(g, u) - oracle.silu_gate(-g, u), g * u, rtol=0, atol=1e-12)
    assert abs(oracle.silu_gate(60.0, 2.0) - 120.0) < 1e-20 * 120 + 1e-13
    assert 0.0 > oracle.silu_gate(-60.0, 1.0) > -60.0 * np.exp(-59.0)
    assert oracle.silu_gate(-1000.0, 1.0) == 0.0   # e^1000 overflows; the quotient is -0


def test_swiglu_matvec_takes_the_gate_from_the_first_half():
    """Gate planes all +1 (alpha 1), up planes all -1 (alpha 2), x = 1 over
    K = 64: g = 64, u = -128, h = silu(64) * -128 (the halves swapped would
    give silu(-128) * 64, about 0)."""
    K = 64
    planes = np.zeros((2, 1, K // 32), dtype=np.uint32)
    planes[0] = 0xFFFFFFFF
    alpha = np.array([[[1.0]], [[2.0]]])
    h, g, u, dg, du = oracle.swiglu_matvec(planes, alpha, np.ones((1, K)))
    assert g[0, 0] == 64.0 and u[0, 0] == -128.0
    assert abs(h[0, 0] - (-128.0 * 64.0 / (1.0 + np.exp(-64.0)))) < 1e-9
    assert dg[0, 0] == 64.0 and du[0, 0] == 128.0
