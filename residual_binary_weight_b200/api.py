"""Python entry points: marshal torch tensors into the C ABI of librb.so."""
from __future__ import annotations

import ctypes
from typing import Optional, Sequence

import torch

from . import _lib
from ._lib import GemvDesc, Layout, check

_DT = {torch.float32: _lib.RB_F32, torch.float16: _lib.RB_F16}


def _stream(device: torch.device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _p(t: Optional[torch.Tensor]):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


_ORDERS = {"rows": _lib.RB_ROWS, "sliced": _lib.RB_SLICED}


def layout(M: int, K: int, n_paths: int, group: int = 0, order: str = "rows") -> Layout:
    return Layout(M, K, n_paths, group, _ORDERS[order], 0)


def planes_words(M: int, K: int, n_paths: int, group: int = 0, order: str = "rows") -> int:
    return _lib.load().rb_planes_words(layout(M, K, n_paths, group, order))


def scales_count(M: int, K: int, n_paths: int, group: int = 0) -> int:
    return _lib.load().rb_scales_count(layout(M, K, n_paths, group))


def _planes_geometry(planes: torch.Tensor, K: int):
    """(N, M, order) of a planes tensor: [N, M, K/32] rows or [N, S, M, 16] sliced."""
    if planes.dim() == 3:
        N, M, W32 = planes.shape
        if W32 * 32 != K:
            raise ValueError("planes and x disagree on K")
        return N, M, "rows"
    if planes.dim() == 4:
        N, S, M, sixteen = planes.shape
        if sixteen != 16 or S != (K + 511) // 512:
            raise ValueError("sliced planes and x disagree on K")
        return N, M, "sliced"
    raise ValueError("planes must be [N, M, K/32] (rows) or [N, S, M, 16] (sliced)")


def _require_cuda(*ts: torch.Tensor) -> torch.device:
    dev = None
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("tensors must live on a CUDA device")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError("tensors are on different devices")
    return dev


def _mapped_host_ptr(t: torch.Tensor) -> int:
    """Device address of a pinned host tensor (the kernel writes it over the
    bus). Page-locked host memory is mapped into the device address space
    under unified addressing; the runtime is asked for the address rather
    than assuming it."""
    if t.is_cuda or not t.is_pinned():
        raise ValueError("expected a pinned host tensor")
    try:
        from cuda.bindings import runtime as rt
    except ImportError as e:   # pragma: no cover - cuda-python is part of the image
        raise ValueError("a pinned host output needs cuda-python (cuda.bindings)") from e
    base = t.untyped_storage().data_ptr()          # the allocation the runtime knows
    err, dptr = rt.cudaHostGetDevicePointer(base, 0)
    if int(err) != 0 or not dptr:
        raise ValueError(f"pinned host tensor is not mapped for the device (cudaHostGetDevicePointer: {err})")
    return int(dptr) + (t.data_ptr() - base)


def pack(W: torch.Tensor, n_paths: int = 2, group: int = 0, alpha_f16: bool = False, order: str = "rows",
         planes: Optional[torch.Tensor] = None, alpha: Optional[torch.Tensor] = None,
         alpha16: Optional[torch.Tensor] = None):
    """Derive N residual sign planes and scales from the shared weight W (M x K).

    Returns (planes, alpha fp32 [N, M, K/G], alpha16 fp16 [N, M, K/G] or None).
    planes holds uint32 words in an int32 tensor: [N, M, K/32] for
    order="rows", [N, ceil(K/512), M, 16] for order="sliced" (the order the
    matvec kernel streams fastest). Output tensors of those shapes may be
    passed in to be filled instead of allocated.
    """
    lib = _lib.load()
    dev = _require_cuda(W, planes, alpha, alpha16)
    if W.dim() != 2 or W.stride(1) != 1 or W.dtype not in _DT:
        raise ValueError("W must be a 2-D fp16/fp32 tensor with unit column stride")
    M, K = W.shape
    G = K if group == 0 else group
    shape = (n_paths, M, K // 32) if order == "rows" else (n_paths, (K + 511) // 512, M, 16)

    def out(t, shp, dt):
        if t is None:
            return torch.empty(shp, dtype=dt, device=dev)
        if tuple(t.shape) != tuple(shp) or t.dtype != dt or not t.is_contiguous():
            raise ValueError(f"output tensor must be contiguous {dt} of shape {shp}")
        return t
    planes = out(planes, shape, torch.int32)
    alpha = out(alpha, (n_paths, M, K // G), torch.float32)
    a16 = out(alpha16, (n_paths, M, K // G), torch.float16) if alpha_f16 else None
    with torch.cuda.device(dev):
        check(lib.rb_pack(_p(W), _DT[W.dtype], W.stride(0), layout(M, K, n_paths, group, order),
                          _p(planes), _p(alpha), _p(a16), _stream(dev)))
    return planes, alpha, a16


def gemv_workspace_bytes(M: int, K: int, n_paths: int, group: int, T: int) -> int:
    return _lib.load().rb_gemv_workspace_bytes(layout(M, K, n_paths, group), T)


def _x2d(x: torch.Tensor) -> torch.Tensor:
    if x.dim() == 1:
        x = x.unsqueeze(0)
    if x.dtype != torch.float16 or x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be fp16 [T, K] with unit column stride")
    return x


def gemv(planes: torch.Tensor, alpha: torch.Tensor, x: torch.Tensor, group: int = 0,
         y: Optional[torch.Tensor] = None, y_dtype: torch.dtype = torch.float16,
         workspace: Optional[torch.Tensor] = None, check_device: bool = False) -> torch.Tensor:
    """y[t] = sum_k alpha_k (.) (B_k x[t]) for T <= 64 tokens (CUDA-core table kernel).

    A caller-given workspace must have been zeroed once before its first use
    (torch.zeros); each call leaves it ready for the next. Without one, a
    zeroed workspace is allocated for the call. With check_device=True the
    call waits for the stream and raises if the kernel recorded a failure in
    its workspace (rb_gemv_check).
    """
    lib = _lib.load()
    x = _x2d(x)
    dev = _require_cuda(planes, alpha, x, y, workspace)
    K = x.shape[1]
    N, M, order = _planes_geometry(planes, K)
    T = x.shape[0]
    if y is None:
        y = torch.empty((T, M), dtype=y_dtype, device=dev)
    L = layout(M, K, N, group, order)
    need = lib.rb_gemv_workspace_bytes(L, T)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.zeros(max(need, 16), dtype=torch.uint8, device=dev)
    with torch.cuda.device(dev):
        check(lib.rb_gemv(_p(planes), _p(alpha), _DT[alpha.dtype], L, _p(x), x.stride(0), T,
                          _p(y), _DT[y.dtype], y.stride(0), _p(workspace),
                          workspace.numel() * workspace.element_size(), _stream(dev)))
        if check_device:
            check(lib.rb_gemv_check(_p(workspace), _stream(dev)))
    return y


def gemv_swiglu_workspace_bytes(M: int, K: int, n_paths: int, group: int, T: int) -> int:
    return _lib.load().rb_gemv_swiglu_workspace_bytes(layout(M, K, n_paths, group), T)


def gemv_swiglu(planes: torch.Tensor, alpha: torch.Tensor, x: torch.Tensor, group: int = 0,
                h: Optional[torch.Tensor] = None, h_dtype: torch.dtype = torch.float16,
                workspace: Optional[torch.Tensor] = None, check_device: bool = False) -> torch.Tensor:
    """h[t] = silu(G x[t]) * (U x[t]) in one launch (rb_gemv_swiglu).

    planes / alpha hold the gate's N paths followed by the up projection's N
    paths (e.g. torch.cat of two pack() outputs along dim 0). The workspace
    contract is gemv()'s (zeroed once before its first use).
    """
    lib = _lib.load()
    x = _x2d(x)
    dev = _require_cuda(planes, alpha, x, h, workspace)
    K = x.shape[1]
    N2, M, order = _planes_geometry(planes, K)
    if N2 % 2:
        raise ValueError("planes must hold the gate's and the up projection's paths (an even count)")
    T = x.shape[0]
    if h is None:
        h = torch.empty((T, M), dtype=h_dtype, device=dev)
    L = layout(M, K, N2 // 2, group, order)
    need = lib.rb_gemv_swiglu_workspace_bytes(L, T)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.zeros(max(need, 16), dtype=torch.uint8, device=dev)
    with torch.cuda.device(dev):
        check(lib.rb_gemv_swiglu(_p(planes), _p(alpha), _DT[alpha.dtype], L, _p(x), x.stride(0), T,
                                 _p(h), _DT[h.dtype], h.stride(0), _p(workspace),
                                 workspace.numel() * workspace.element_size(), _stream(dev)))
        if check_device:
            check(lib.rb_gemv_check(_p(workspace), _stream(dev)))
    return h


def mlp_gemv(gu_planes: torch.Tensor, gu_alpha: torch.Tensor, d_planes: torch.Tensor, d_alpha: torch.Tensor,
             x: torch.Tensor, group: int = 0, y: Optional[torch.Tensor] = None,
             workspace: Optional[torch.Tensor] = None, check_device: bool = False):
    """The gated MLP block for decode tokens: y = D (silu(G x) * (U x)).

    Two launches on the current stream: rb_gemv_swiglu (gate and up, gated
    in the epilogue, h in fp16) and rb_gemv for the down projection D.
    Returns (y, h). One workspace (zeroed once) serves both launches.
    """
    x = _x2d(x)
    K = x.shape[1]
    _, M, order = _planes_geometry(gu_planes, K)
    Nd, Md, _ = _planes_geometry(d_planes, M)
    T = x.shape[0]
    need = max(gemv_swiglu_workspace_bytes(M, K, gu_planes.shape[0] // 2, group, T),
               gemv_workspace_bytes(Md, M, Nd, group, T), 16)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.zeros(need, dtype=torch.uint8, device=x.device)
    h = gemv_swiglu(gu_planes, gu_alpha, x, group=group, workspace=workspace, check_device=check_device)
    y = gemv(d_planes, d_alpha, h, group=group, y=y, workspace=workspace, check_device=check_device)
    return y, h


class GroupedGemv:
    """One persistent launch over many (planes, alpha, x, y) matrices.

    The descriptor table is uploaded once at construction; call ``run()`` for
    every step (the x tensors are read and the y tensors written in place).
    An x or y tensor may also be a pinned host tensor: the kernel then reads
    x from, or writes y to, host memory over the bus (zero-copy), so a step
    needs no separate host-to-device or device-to-host copy.
    """

    def __init__(self, items: Sequence[tuple], n_paths: int, group: int = 0, T: int = 1):
        lib = _lib.load()
        self.n_paths, self.group, self.T = n_paths, group, T
        self.items = list(items)   # keep tensors alive
        n = len(self.items)
        self.host = (GemvDesc * n)()
        adt = ydt = order = None
        dev = None
        for i, (planes, alpha, x, y) in enumerate(self.items):
            host_x = not x.is_cuda and x.is_pinned()
            host_y = not y.is_cuda and y.is_pinned()
            dev = _require_cuda(planes, alpha, None if host_x else x, None if host_y else y)
            K = x.shape[-1]
            N, M, o = _planes_geometry(planes, K)
            order = o if order is None else order
            if N != n_paths or y.shape[-1] != M or o != order:
                raise ValueError(f"item {i}: inconsistent shapes or plane orders")
            if not (x.is_contiguous() and y.is_contiguous()):
                raise ValueError(f"item {i}: x and y must be contiguous [T, K] / [T, M]")
            # the descriptors are dense [T][K] / [T][M]: exactly T rows each
            if x.numel() != T * K or y.numel() != T * M:
                raise ValueError(f"item {i}: x must hold {T} x {K} and y {T} x {M} values")
            adt = alpha.dtype if adt is None else adt
            ydt = y.dtype if ydt is None else ydt
            if alpha.dtype != adt or y.dtype != ydt:
                raise ValueError("all items must share the scale and output dtypes")
            x_ptr = x.data_ptr() if x.is_cuda else _mapped_host_ptr(x)
            y_ptr = y.data_ptr() if y.is_cuda else _mapped_host_ptr(y)
            self.host[i] = GemvDesc(planes.data_ptr(), alpha.data_ptr(), x_ptr, y_ptr, M, K)
        self.device = dev
        raw = bytes(self.host)
        self.dev_descs = torch.frombuffer(bytearray(raw), dtype=torch.uint8).to(dev)
        self.alpha_dtype, self.y_dtype = _DT[adt], _DT[ydt]
        self.order = _ORDERS[order]
        need = lib.rb_gemv_grouped_workspace_bytes(self.host, n, n_paths, T)
        self.workspace = torch.zeros(max(need, 16), dtype=torch.uint8, device=dev)
        self.n = n

    def run(self) -> None:
        lib = _lib.load()
        with torch.cuda.device(self.device):
            check(lib.rb_gemv_grouped(ctypes.cast(self.host, ctypes.c_void_p), _p(self.dev_descs), self.n,
                                      self.n_paths, self.group, self.order, self.alpha_dtype, self.y_dtype, self.T,
                                      _p(self.workspace), self.workspace.numel(), _stream(self.device)))

    def check_device_flag(self) -> None:
        check(_lib.load().rb_gemv_check(_p(self.workspace), _stream(self.device)))


def gemm_workspace_bytes(M: int, K: int, n_paths: int, group: int, T: int) -> int:
    return _lib.load().rb_gemm_workspace_bytes(layout(M, K, n_paths, group), T)


def gemm(planes: torch.Tensor, alpha: torch.Tensor, X: torch.Tensor, group: int = 0,
         Y: Optional[torch.Tensor] = None, y_dtype: torch.dtype = torch.float16,
         workspace: Optional[torch.Tensor] = None, check_device: bool = False,
         reconstruct: bool = False) -> torch.Tensor:
    """Y[t] = sum_k alpha_k (.) (B_k X[t]) on the tcgen05 tensor cores (any T).

    reconstruct=True (two paths, per-row scales): one fp16 operand
    RN(alpha_0 B_0 + alpha_1 B_1) per weight and one MMA chain
    (rb_gemm_reconstruct). With check_device=True the call waits for the
    stream and raises if a kernel recorded a failure in its workspace
    (rb_gemm_check).
    """
    lib = _lib.load()
    X = _x2d(X)
    dev = _require_cuda(planes, alpha, X, Y, workspace)
    K = X.shape[1]
    N, M, order = _planes_geometry(planes, K)
    T = X.shape[0]
    if Y is None:
        Y = torch.empty((T, M), dtype=y_dtype, device=dev)
    L = layout(M, K, N, group, order)
    need = 256 if reconstruct else lib.rb_gemm_workspace_bytes(L, T)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    fn = lib.rb_gemm_reconstruct if reconstruct else lib.rb_gemm
    with torch.cuda.device(dev):
        check(fn(_p(planes), _p(alpha), _DT[alpha.dtype], L, _p(X), X.stride(0), T,
                 _p(Y), _DT[Y.dtype], Y.stride(0), _p(workspace),
                 workspace.numel() * workspace.element_size(), _stream(dev)))
        if check_device:
            check(lib.rb_gemm_check(_p(workspace), _stream(dev)))
    return Y


def gemm_from_weight_workspace_bytes(M: int, K: int, n_paths: int, group: int, T: int, order: str = "sliced") -> int:
    return _lib.load().rb_gemm_from_weight_workspace_bytes(layout(M, K, n_paths, group, order), T)


def gemm_from_weight(W: torch.Tensor, X: torch.Tensor, n_paths: int = 2, group: int = 0, order: str = "sliced",
                     Y: Optional[torch.Tensor] = None, y_dtype: torch.dtype = torch.float16,
                     workspace: Optional[torch.Tensor] = None, check_device: bool = False) -> torch.Tensor:
    """Training forward: Y[t] = sum_k alpha_k (.) (B_k X[t]) with the planes
    and scales derived afresh from the full-precision weight W (M x K) in the
    same call (rb_gemm_from_weight: pack into the workspace, then rb_gemm)."""
    lib = _lib.load()
    X = _x2d(X)
    dev = _require_cuda(W, X, Y, workspace)
    if W.dim() != 2 or W.stride(1) != 1 or W.dtype not in _DT:
        raise ValueError("W must be a 2-D fp16/fp32 tensor with unit column stride")
    M, K = W.shape
    if X.shape[1] != K:
        raise ValueError("X must have K columns")
    T = X.shape[0]
    if Y is None:
        Y = torch.empty((T, M), dtype=y_dtype, device=dev)
    L = layout(M, K, n_paths, group, order)
    need = lib.rb_gemm_from_weight_workspace_bytes(L, T)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    with torch.cuda.device(dev):
        check(lib.rb_gemm_from_weight(_p(W), _DT[W.dtype], W.stride(0), L, _p(X), X.stride(0), T, _p(Y),
                                      _DT[Y.dtype], Y.stride(0), _p(workspace),
                                      workspace.numel() * workspace.element_size(), _stream(dev)))
        if check_device:
            check(lib.rb_gemm_check(_p(workspace), _stream(dev)))
    return Y


def pack_fixed(W: torch.Tensor, h: torch.Tensor, g: Optional[torch.Tensor] = None, order: str = "rows",
               planes: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Sign planes of the dual-scale block for given scales: h fp32 [N, M]
    (output channels), g fp32 [N, K] (input channels) or None.
    B_k = sign(R_{k-1}), R_k = R_{k-1} - h_k[i] g_k[j] B_k."""
    lib = _lib.load()
    dev = _require_cuda(W, h, g, planes)
    if W.dim() != 2 or W.stride(1) != 1 or W.dtype not in _DT:
        raise ValueError("W must be a 2-D fp16/fp32 tensor with unit column stride")
    M, K = W.shape
    N = h.shape[0]
    if h.shape != (N, M) or h.dtype != torch.float32 or not h.is_contiguous():
        raise ValueError("h must be contiguous fp32 [N, M]")
    if g is not None and (g.shape != (N, K) or g.dtype != torch.float32 or not g.is_contiguous()):
        raise ValueError("g must be contiguous fp32 [N, K]")
    shape = (N, M, K // 32) if order == "rows" else (N, (K + 511) // 512, M, 16)
    if planes is None:
        planes = torch.empty(shape, dtype=torch.int32, device=dev)
    elif tuple(planes.shape) != shape or planes.dtype != torch.int32 or not planes.is_contiguous():
        raise ValueError(f"planes must be contiguous int32 of shape {shape}")
    with torch.cuda.device(dev):
        check(lib.rb_pack_fixed(_p(W), _DT[W.dtype], W.stride(0), layout(M, K, N, 0, order), _p(h), _p(g),
                                _p(planes), _stream(dev)))
    return planes


def dual_gemv(planes: torch.Tensor, h: torch.Tensor, g: Optional[torch.Tensor], x: torch.Tensor,
              y: Optional[torch.Tensor] = None, y_dtype: torch.dtype = torch.float16,
              workspace: Optional[torch.Tensor] = None, check_device: bool = False) -> torch.Tensor:
    """y[t] = sum_k h_k (.) (B_k RN_fp16(g_k (.) x[t])) for T <= 64 tokens."""
    lib = _lib.load()
    x = _x2d(x)
    dev = _require_cuda(planes, h, g, x, y, workspace)
    K = x.shape[1]
    N, M, order = _planes_geometry(planes, K)
    T = x.shape[0]
    if h.shape != (N, M) or h.dtype != torch.float32 or not h.is_contiguous():
        raise ValueError("h must be contiguous fp32 [N, M]")
    if g is not None and (g.shape != (N, K) or g.dtype != torch.float32 or not g.is_contiguous()):
        raise ValueError("g must be contiguous fp32 [N, K]")
    if y is None:
        y = torch.empty((T, M), dtype=y_dtype, device=dev)
    L = layout(M, K, N, 0, order)
    need = lib.rb_dual_gemv_workspace_bytes(L, T)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    with torch.cuda.device(dev):
        check(lib.rb_dual_gemv(_p(planes), L, _p(h), _p(g), _p(x), x.stride(0), T, _p(y), _DT[y.dtype], y.stride(0),
                               _p(workspace), workspace.numel() * workspace.element_size(), _stream(dev)))
        if check_device:
            check(lib.rb_gemv_check(_p(workspace), _stream(dev)))
    return y
