"""rb_gemm_from_weight (the training forward: planes and scales derived
from W in the same call, then contracted) on the GPU.

* It equals rb_pack followed by rb_gemm bit for bit (both pinned to the
  oracle by their own tests).
* Against the oracle directly: oracle pack + oracle matvec of the same W and
  X. Entries whose residual is within the near-zero allowance (|R_{k-1}| <=
  1e-6 alpha_k, known from the oracle's own residual magnitudes) may take
  either sign on the GPU, and so may the later paths of such an entry; each
  widens the bound of its row by 2 sum_{k' >= k} alpha_k' |x_j|. Otherwise
  the bar is the matvec's 1e-3 * sum_k sum_j |alpha_k x_j|.
"""
import numpy as np
import pytest
import torch

import oracle
import residual_binary_weight_b200 as rb
import synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("order", ["rows", "sliced"])
@pytest.mark.parametrize("n,group", [(1, 0), (2, 0), (4, 0), (2, 128), (4, 128)])
@pytest.mark.parametrize("T", [5, 16, 300])
def test_equals_pack_then_gemm(n, group, order, T):
    rng = np.random.default_rng(n + group + T)
    W = torch.from_numpy((rng.standard_normal((333, 1024)) * 0.02).astype(np.float16)).cuda()
    X = torch.from_numpy(rng.standard_normal((T, 1024)).astype(np.float16)).cuda()
    Y = rb.gemm_from_weight(W, X, n_paths=n, group=group, order=order, check_device=True)
    planes, alpha, a16 = rb.pack(W, n, group, alpha_f16=group == 128, order=order)
    Y2 = rb.gemm(planes, a16 if group == 128 else alpha, X, group=group, check_device=True)
    assert torch.equal(Y, Y2)


def _bound(W, X, n, group):
    """Oracle output and the per-element bound (allowance-aware)."""
    p, a, rabs = oracle.pack(W, n, group, want_rabs=True)
    stored = (oracle.alpha_to_f16(a) if group else a.astype(np.float32)).astype(np.float64)
    x = X.astype(np.float64)
    y, den = oracle.matvec(p, stored, x)
    M, K = W.shape
    G = K if group == 0 else group
    al = np.repeat(np.asarray(a, dtype=np.float64), G, axis=2)            # [n, M, K]
    amb = rabs <= 1e-6 * al                                               # [n, M, K]
    tail = np.cumsum(al[::-1], axis=0)[::-1]                              # sum_{k' >= k} alpha_k'
    first = np.zeros((M, K))
    seen = np.zeros((M, K), dtype=bool)
    for k in range(n):
        new = amb[k] & ~seen
        first[new] = 2.0 * tail[k][new]
        seen |= amb[k]
    extra = np.abs(x) @ first.T                                           # [T, M]
    return y, 1e-3 * den + extra, int(seen.sum())


@pytest.mark.parametrize("n,group", [(2, 0), (4, 128)])
@pytest.mark.parametrize("T", [5, 130])
def test_matches_oracle(n, group, T):
    rng = np.random.default_rng(100 + n + T)
    W = (rng.standard_normal((300, 2048)) * 0.02).astype(np.float16)
    X = rng.standard_normal((T, 2048)).astype(np.float16)
    Y = rb.gemm_from_weight(torch.from_numpy(W).cuda(), torch.from_numpy(X).cuda(), n_paths=n, group=group,
                            check_device=True)
    y, bound, n_amb = _bound(W, X, n, group)
    assert n_amb <= 20   # the widened rows stay few: the bound is not vacuous
    err = np.abs(Y.float().cpu().numpy().astype(np.float64) - y)
    assert (err <= bound).all(), float((err / bound).max())


def test_prefill_full_size_equals_pack_then_gemm():
    """The 2048-token prefill block through the 14336 x 4096 projection."""
    wl = synth.WORKLOADS["prefill"]
    W = synth.device_weight(wl, 0, "up", "cuda")
    X = synth.device_activations(wl, 0, "up", 2048, "cuda")
    Y = rb.gemm_from_weight(W, X, check_device=True)
    planes, alpha, _ = rb.pack(W, 2, 0, order="sliced")
    assert torch.equal(Y, rb.gemm(planes, alpha, X, check_device=True))
