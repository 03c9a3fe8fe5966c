"""Workload shapes, value distributions and seeded draws (no method arithmetic).

The five workloads follow the synthetic stand-ins for the settings the RaBiT
paper (arXiv 2602.05367, sections 4.1 and 5, appendix D) and the QBB summary
("W(4x1)A16g128", key results) describe: a small square layer, Llama-2-7B and
Llama-3-70B shaped decode linears, a QBB-style four-path grouped layer, and a
prefill block. No public dataset or checkpoint is used; weights and activations
are drawn from the distributions below.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Dict, List, Sequence, Tuple

import numpy as np

ROOT_SEED = 20260205


@dataclass(frozen=True)
class MatrixSpec:
    name: str
    M: int  # output rows
    K: int  # input columns


@dataclass(frozen=True)
class Workload:
    wid: int
    name: str
    matrices: Tuple[MatrixSpec, ...]
    layers: int
    n_paths: int
    group: int  # 0: one scale per row; 128: one scale per 128 columns
    w_dist: str  # "normal", "row_lognormal_outliers" or "student_t4"
    w_dtype: str  # "f32" or "f16"
    x_dist: str  # "normal" or "outlier_channels"
    batches: Tuple[int, ...]
    scale_dtype: str = "f32"  # dtype the matvec/matmul reads the scales in
    notes: str = ""


WORKLOADS: Dict[str, Workload] = {}


def _add(w: Workload) -> None:
    WORKLOADS[w.name] = w


# Small square layer: fp32 weights, two paths, per-row scales, one token.
_add(Workload(0, "layer256", (MatrixSpec("w", 256, 256),), 1, 2, 0, "normal",
              "f32", "normal", (1,)))

# Llama-2-7B shaped decode linears (q, k, v, o, gate, up, down) over 32 layers.
_add(Workload(1, "llama2_7b_decode",
              (MatrixSpec("q", 4096, 4096), MatrixSpec("k", 4096, 4096),
               MatrixSpec("v", 4096, 4096), MatrixSpec("o", 4096, 4096),
               MatrixSpec("gate", 11008, 4096), MatrixSpec("up", 11008, 4096),
               MatrixSpec("down", 4096, 11008)),
              32, 2, 0, "row_lognormal_outliers", "f16", "outlier_channels", (1,)))

# Llama-3-70B shaped decode linears, batches 1..64.
_add(Workload(2, "llama3_70b_decode",
              (MatrixSpec("attn", 8192, 8192), MatrixSpec("up", 28672, 8192),
               MatrixSpec("down", 8192, 28672)),
              1, 2, 0, "normal", "f16", "normal", (1, 4, 16, 64)))

# QBB-style four binary bases with fp16 scales per 128 input columns.
_add(Workload(3, "qbb_g128",
              (MatrixSpec("up", 11008, 4096), MatrixSpec("down", 4096, 11008)),
              1, 4, 128, "student_t4", "f16", "normal", (1, 16), scale_dtype="f16"))

# Prefill block: 2048 tokens through two 14336-wide projections.
_add(Workload(4, "prefill",
              (MatrixSpec("up", 14336, 4096), MatrixSpec("down", 4096, 14336)),
              1, 2, 0, "normal", "f16", "normal", (2048,)))

W_STD = 0.02           # std of the "normal" and "student_t4" weights
SIGMA_LO, SIGMA_HI = 0.005, 0.05   # per-row std range (log-uniform)
W_OUTLIER_P, W_OUTLIER_X = 1e-3, 10.0
X_OUTLIER_FRAC, X_OUTLIER_X = 0.005, 20.0


def _matrix_index(wl: Workload, name: str) -> int:
    for i, m in enumerate(wl.matrices):
        if m.name == name:
            return i
    raise KeyError(f"{wl.name} has no matrix {name!r}")


def child_seed(wl: Workload, layer: int, matrix: str, tensor: int,
               row: int | None = None) -> np.random.SeedSequence:
    key = [ROOT_SEED, wl.wid, layer, _matrix_index(wl, matrix), tensor]
    if row is not None:
        key.append(row)
    return np.random.SeedSequence(key)


def _np_dtype(s: str):
    return {"f32": np.float32, "f16": np.float16}[s]


# ---------------------------------------------------------------- host draws
def _host_row(wl: Workload, layer: int, matrix: str, i: int, K: int) -> np.ndarray:
    rng = np.random.Generator(np.random.PCG64(child_seed(wl, layer, matrix, 0, i)))
    if wl.w_dist == "normal":
        r = rng.standard_normal(K) * W_STD
    elif wl.w_dist == "row_lognormal_outliers":
        sigma = math.exp(rng.uniform(math.log(SIGMA_LO), math.log(SIGMA_HI)))
        r = rng.standard_normal(K) * sigma
        r = np.where(rng.random(K) < W_OUTLIER_P, r * W_OUTLIER_X, r)
    elif wl.w_dist == "student_t4":
        r = rng.standard_t(4, K) * (W_STD / math.sqrt(2.0))
    else:
        raise ValueError(wl.w_dist)
    return r.astype(_np_dtype(wl.w_dtype))


def host_rows(wl: Workload, layer: int, matrix: str, rows: Sequence[int]) -> np.ndarray:
    """Selected rows of one weight matrix (each row has its own stream)."""
    spec = wl.matrices[_matrix_index(wl, matrix)]
    out = np.empty((len(rows), spec.K), dtype=_np_dtype(wl.w_dtype))
    for n, i in enumerate(rows):
        out[n] = _host_row(wl, layer, matrix, int(i), spec.K)
    return out


def host_weight(wl: Workload, layer: int, matrix: str, M: int | None = None,
                K: int | None = None) -> np.ndarray:
    """A full weight matrix; M and K may shrink the shape for small cases."""
    spec = wl.matrices[_matrix_index(wl, matrix)]
    M = spec.M if M is None else M
    K = spec.K if K is None else K
    out = np.empty((M, K), dtype=_np_dtype(wl.w_dtype))
    for i in range(M):
        out[i] = _host_row(wl, layer, matrix, i, K)
    return out


def host_activations(wl: Workload, layer: int, matrix: str, T: int,
                     K: int | None = None) -> np.ndarray:
    """fp16 activations [T, K]; outlier channels are shared by the T tokens."""
    spec = wl.matrices[_matrix_index(wl, matrix)]
    K = spec.K if K is None else K
    rng = np.random.Generator(np.random.PCG64(child_seed(wl, layer, matrix, 1)))
    x = rng.standard_normal((T, K))
    if wl.x_dist == "outlier_channels":
        n = int(round(X_OUTLIER_FRAC * K))
        ch = rng.choice(K, size=n, replace=False)
        x[:, ch] *= X_OUTLIER_X
    elif wl.x_dist != "normal":
        raise ValueError(wl.x_dist)
    return x.astype(np.float16)


# -------------------------------------------------------------- device draws
def _torch_gen(device, ss: np.random.SeedSequence):
    import torch
    s = ss.generate_state(2, dtype=np.uint32)
    g = torch.Generator(device=device)
    g.manual_seed(int((int(s[0]) << 31) ^ int(s[1])) & ((1 << 63) - 1))
    return g


def device_weight(wl: Workload, layer: int, matrix: str, device,
                  M: int | None = None, K: int | None = None):
    """A weight matrix drawn on a CUDA device (torch Philox stream)."""
    import torch
    spec = wl.matrices[_matrix_index(wl, matrix)]
    M = spec.M if M is None else M
    K = spec.K if K is None else K
    g = _torch_gen(device, child_seed(wl, layer, matrix, 0))
    if wl.w_dist == "normal":
        w = torch.randn((M, K), generator=g, device=device) * W_STD
    elif wl.w_dist == "row_lognormal_outliers":
        lo, hi = math.log(SIGMA_LO), math.log(SIGMA_HI)
        sigma = torch.exp(torch.rand((M, 1), generator=g, device=device) * (hi - lo) + lo)
        w = torch.randn((M, K), generator=g, device=device) * sigma
        mask = torch.rand((M, K), generator=g, device=device) < W_OUTLIER_P
        w = torch.where(mask, w * W_OUTLIER_X, w)
        del mask
    elif wl.w_dist == "student_t4":
        # t with 4 degrees of freedom: Z / sqrt(V / 4), V ~ chi-square(4) = -2 ln(U1 U2)
        z = torch.randn((M, K), generator=g, device=device)
        u1 = torch.rand((M, K), generator=g, device=device).clamp_min_(1e-30)
        u2 = torch.rand((M, K), generator=g, device=device).clamp_min_(1e-30)
        v = -2.0 * torch.log(u1 * u2)
        del u1, u2
        w = z / torch.sqrt(v / 4.0) * (W_STD / math.sqrt(2.0))
        del z, v
    else:
        raise ValueError(wl.w_dist)
    dt = {"f32": torch.float32, "f16": torch.float16}[wl.w_dtype]
    return w.to(dt)


def device_activations(wl: Workload, layer: int, matrix: str, T: int, device,
                       K: int | None = None):
    import torch
    spec = wl.matrices[_matrix_index(wl, matrix)]
    K = spec.K if K is None else K
    g = _torch_gen(device, child_seed(wl, layer, matrix, 1))
    x = torch.randn((T, K), generator=g, device=device)
    if wl.x_dist == "outlier_channels":
        n = int(round(X_OUTLIER_FRAC * K))
        ch = torch.randperm(K, generator=g, device=device)[:n]
        x[:, ch] *= X_OUTLIER_X
    return x.to(torch.float16)
