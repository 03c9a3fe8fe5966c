"""Helpers shared by the GPU parity tests (imported only by tests)."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import residual_binary_weight_b200 as rb


def rows_to_sliced(p: np.ndarray) -> np.ndarray:
    """[N, M, K/32] words -> [N, S, M, 16] (512-column slices, zero padding)."""
    N, M, W32 = p.shape
    S = (W32 + 15) // 16
    out = np.zeros((N, S, M, 16), dtype=np.uint32)
    for s in range(S):
        w = p[:, :, 16 * s:16 * s + 16]
        out[:, s, :, :w.shape[2]] = w
    return out


def sliced_to_rows(q: np.ndarray, K: int) -> np.ndarray:
    N, S, M, _ = q.shape
    return np.concatenate([q[:, s] for s in range(S)], axis=2)[:, :, :K // 32].copy()


def planes_np(t: torch.Tensor, K: int | None = None) -> np.ndarray:
    """GPU planes as row-major uint32 words (sliced planes are converted)."""
    a = t.cpu().numpy().view(np.uint32)
    if a.ndim == 4:
        a = sliced_to_rows(a, K)
    return a


def to_dev_planes(p: np.ndarray, device="cuda", order: str = "rows") -> torch.Tensor:
    if order == "sliced":
        p = rows_to_sliced(p)
    return torch.from_numpy(np.ascontiguousarray(p).view(np.int32)).to(device)


def check_pack(W: np.ndarray, n_paths: int, group: int, ldw_pad: int = 0, alpha_f16: bool = True,
               order: str = "rows"):
    """GPU pack of W against the oracle: planes (near-zero allowance), fp32 and fp16 scales."""
    M, K = W.shape
    Wt = torch.from_numpy(np.ascontiguousarray(W))
    if ldw_pad:
        big = torch.zeros((M, K + ldw_pad), dtype=Wt.dtype)
        big[:, :K] = Wt
        Wd = big.cuda()[:, :K]
    else:
        Wd = Wt.cuda()
    planes, alpha, a16 = rb.pack(Wd, n_paths, group, alpha_f16=alpha_f16, order=order)
    torch.cuda.synchronize()
    ref_p, ref_a, rabs = oracle.pack(W, n_paths, group, want_rabs=True)
    if order == "sliced":
        # the padding words of the last slice are zero
        q = planes.cpu().numpy().view(np.uint32)
        assert np.all(q[:, -1, :, (K // 32) % 16 or 16:] == 0)
    rep = oracle.compare_planes(planes_np(planes, K), ref_p, rabs, ref_a)
    nbad_a, worst_a = oracle.compare_scales(alpha.cpu().numpy(), ref_a)
    nbad16 = oracle.compare_scales_f16(a16.cpu().numpy(), ref_a) if alpha_f16 else 0
    return rep, nbad_a, worst_a, nbad16


def check_gemv_on_oracle_planes(W: np.ndarray, x: np.ndarray, n_paths: int, group: int,
                                alpha_f16: bool, y_dtype=torch.float16, ldx_pad: int = 0, ldy_pad: int = 0,
                                order: str = "rows"):
    """Kernel parity: the oracle packs W; the GPU and the oracle evaluate the
    same planes and stored scales on the same x."""
    ref_p, ref_a, _ = oracle.pack(W, n_paths, group)
    stored = oracle.alpha_to_f16(ref_a) if alpha_f16 else ref_a.astype(np.float32)
    y_ref, den = oracle.matvec(ref_p, stored.astype(np.float64), x.astype(np.float64))
    T, K = x.shape
    M = W.shape[0]
    xt = torch.zeros((T, K + ldx_pad), dtype=torch.float16)
    xt[:, :K] = torch.from_numpy(x)
    xd = xt.cuda()[:, :K]
    yd = torch.full((T, M + ldy_pad), float("nan"), dtype=y_dtype, device="cuda")
    y = rb.gemv(to_dev_planes(ref_p, order=order), torch.from_numpy(stored).cuda(), xd, group=group, y=yd[:, :M])
    torch.cuda.synchronize()
    yh = yd.float().cpu().numpy()
    if ldy_pad:
        assert np.all(np.isnan(yh[:, M:])), "wrote past the row"
    nbad, worst = oracle.compare_outputs(yh[:, :M], y_ref, den)
    return nbad, worst
