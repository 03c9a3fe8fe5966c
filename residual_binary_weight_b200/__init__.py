"""Residual-binary-weight linear layers on B200 (sm_100a).

A weight W (M x K) is stored as N bit-packed sign planes and scales,
W ~= sum_k alpha_k (.) B_k (RaBiT, arXiv 2602.05367, sections 4.1-4.2; QBB
grouped variant). This package is a thin binding over the C ABI of
``librb.so`` (include/rb_api.h): tensors are torch CUDA tensors, the stream is
torch's current stream, and every step of the computation runs in the
library's CUDA kernels.

    planes, alpha, alpha16 = pack(W, n_paths=2, group=0)
    y = gemv(planes, alpha, x, group=0)               # decode, T <= 64 tokens
    Y = gemm(planes, alpha, X, group=0)               # any batch, tcgen05 tensor cores
"""
from ._lib import RbError, load  # noqa: F401
from .api import (  # noqa: F401
    GroupedGemv,
    dual_gemv,
    gemm,
    gemm_from_weight,
    gemm_from_weight_workspace_bytes,
    gemm_workspace_bytes,
    gemv,
    gemv_swiglu,
    gemv_swiglu_workspace_bytes,
    gemv_workspace_bytes,
    layout,
    mlp_gemv,
    pack,
    pack_fixed,
    planes_words,
    scales_count,
)

__all__ = ["pack", "pack_fixed", "gemv", "gemv_swiglu", "mlp_gemv", "dual_gemv", "gemm", "gemm_from_weight",
           "GroupedGemv", "layout", "planes_words", "scales_count", "gemv_workspace_bytes",
           "gemv_swiglu_workspace_bytes", "gemm_workspace_bytes", "gemm_from_weight_workspace_bytes", "RbError",
           "load"]
