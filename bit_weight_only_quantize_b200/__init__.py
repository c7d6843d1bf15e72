"""B200 (sm_100a) Q4 weight-only quantisation: quantise, decode GEMV, prefill GEMM.

Thin torch-facing wrappers over the C ABI in ``include/q4.h``.  torch supplies
device memory and the current stream; every step of the computation runs in the
library's CUDA kernels.  The weight format is 4-bit symmetric with one binary16
scale per group of 32 weights along K (QORA-4B thread, section "量化与内存管理";
QORA-LLM-0.8B model card, section "Weight Format").
"""
from __future__ import annotations

import contextlib
import ctypes

import torch

from . import _lib
from ._lib import Q4Error, FLAG_NONFINITE, FLAG_SCALE_OVERFLOW, GEMV_MAX_M  # noqa: F401

__all__ = [
    "quantize", "gemv", "gemv_host", "gemv_multi", "gemv_mixed", "gemv_mixed_workspace_size", "GemvMulti", "gemv_gate_up", "gemv_argmax", "gemv_topk",
    "gemv_topk_workspace_size", "topk_merge", "f16_gemv", "int8_quantize", "int8_gemv", "gemm", "gemv_workspace_size", "gemv_multi_workspace_size",
    "Q4Error", "FLAG_NONFINITE", "FLAG_SCALE_OVERFLOW", "GEMV_MAX_M",
]


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _on(device: torch.device):
    """Make ``device`` current for the call (a no-op context when it already is)."""
    if device.index is None or device.index == torch.cuda.current_device():
        return contextlib.nullcontext()
    return torch.cuda.device(device)


def _need(t: torch.Tensor, name: str, dtype: torch.dtype, ndim: int, device: torch.device | None = None) -> None:
    """Type, dtype, device, rank and contiguity of one argument (``device``: the device
    every tensor of the call must share; None: any CUDA device)."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype is not dtype:
        raise TypeError(f"{name} must have dtype {dtype}, got {t.dtype}")
    if device is None:
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
    elif t.device != device:
        raise ValueError(f"{name} must be on {device}, got {t.device}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def quantize(W: torch.Tensor, flags: torch.Tensor | None = None):
    """f32 W[N,K] -> (packed uint8 [N,K/2], scales binary16 as int16 bits [N,K/32]).

    ``flags`` (optional int32 tensor of one element) receives the OR of the
    Q4 flag bits; it is not cleared first.
    """
    _need(W, "W", torch.float32, 2)
    N, K = W.shape
    packed = torch.empty((N, K // 2), dtype=torch.uint8, device=W.device)
    scales = torch.empty((N, max(K // 32, 0)), dtype=torch.int16, device=W.device)
    fptr = None
    if flags is not None:
        _need(flags, "flags", torch.int32, 1, W.device)
        fptr = flags.data_ptr()
    with _on(W.device):
        st = _lib.load().q4_quantize(W.data_ptr(), N, K, packed.data_ptr(), scales.data_ptr(), fptr, _stream())
    _lib.check(st, "q4_quantize")
    return packed, scales


def int8_quantize(W: torch.Tensor, flags: torch.Tensor | None = None):
    """f32 W[N,K] -> (codes int8 [N,K], scales binary16 as int16 bits [N,K/32]) in the
    library's INT8 format (the INT8 layers of a mixed INT8/INT4 model); ``flags`` as for
    ``quantize``."""
    _need(W, "W", torch.float32, 2)
    N, K = W.shape
    codes = torch.empty((N, K), dtype=torch.int8, device=W.device)
    scales = torch.empty((N, max(K // 32, 0)), dtype=torch.int16, device=W.device)
    fptr = None
    if flags is not None:
        _need(flags, "flags", torch.int32, 1, W.device)
        fptr = flags.data_ptr()
    with _on(W.device):
        st = _lib.load().q4_int8_quantize(W.data_ptr(), N, K, codes.data_ptr(), scales.data_ptr(), fptr, _stream())
    _lib.check(st, "q4_int8_quantize")
    return codes, scales


def int8_gemv(x: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor, out: torch.Tensor | None = None):
    """y[M,N] (f32) = x[M,K] . dequant8(W)^T for M <= 16; x is float32 or bfloat16."""
    if x.dtype is torch.float32:
        xt = _lib.Q4_F32
    elif x.dtype is torch.bfloat16:
        xt = _lib.Q4_BF16
    else:
        raise TypeError("x must be float32 or bfloat16")
    _need(x, "x", x.dtype, 2)
    _need(codes, "codes", torch.int8, 2, x.device)
    _need(scales, "scales", torch.int16, 2, x.device)
    M, K = x.shape
    N = codes.shape[0]
    if codes.shape[1] != K or tuple(scales.shape) != (N, K // 32):
        raise ValueError("shape mismatch between x, codes and scales")
    if out is None:
        out = torch.empty((M, N), dtype=torch.float32, device=x.device)
    else:
        _need(out, "out", torch.float32, 2, x.device)
        if tuple(out.shape) != (M, N):
            raise ValueError("out must be [M, N]")
    with _on(x.device):
        st = _lib.load().q4_int8_gemv(x.data_ptr(), xt, M, K, codes.data_ptr(), scales.data_ptr(), N, out.data_ptr(),
                                      _stream())
    _lib.check(st, "q4_int8_gemv")
    return out


def gemv_workspace_size(M: int, N: int, K: int) -> int:
    return int(_lib.load().q4_gemv_workspace_size(M, N, K))


def gemv(x: torch.Tensor, packed: torch.Tensor, scales: torch.Tensor, out: torch.Tensor | None = None,
         workspace: torch.Tensor | None = None) -> torch.Tensor:
    """y[M,N] (f32) = x[M,K] . dequant(W)^T for M <= 16; x is float32 or bfloat16.

    ``workspace`` (uint8, zero-filled before first use) is allocated here when
    the shape needs one and none is given.
    """
    if x.dtype == torch.float32:
        xt = _lib.Q4_F32
    elif x.dtype == torch.bfloat16:
        xt = _lib.Q4_BF16
    else:
        raise TypeError("x must be float32 or bfloat16")
    _need(x, "x", x.dtype, 2)
    _need(packed, "packed", torch.uint8, 2, x.device)
    _need(scales, "scales", torch.int16, 2, x.device)
    M, K = x.shape
    N = packed.shape[0]
    if packed.shape[1] * 2 != K or tuple(scales.shape) != (N, K // 32):
        raise ValueError("shape mismatch between x, packed and scales")
    if out is None:
        out = torch.empty((M, N), dtype=torch.float32, device=x.device)
    else:
        _need(out, "out", torch.float32, 2, x.device)
        if tuple(out.shape) != (M, N):
            raise ValueError("out has the wrong shape")
    if workspace is not None:
        _need(workspace, "workspace", torch.uint8, 1, x.device)
    lib = _lib.load()
    with _on(x.device):
        if workspace is None:
            need = int(lib.q4_gemv_workspace_size(M, N, K))
            if need:
                workspace = torch.zeros(need, dtype=torch.uint8, device=x.device)
        ws_ptr = workspace.data_ptr() if workspace is not None else None
        ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
        st = lib.q4_gemv(x.data_ptr(), xt, M, K, packed.data_ptr(), scales.data_ptr(), N,
                         out.data_ptr(), ws_ptr, ws_bytes, _stream())
    _lib.check(st, "q4_gemv")
    return out


def gemv_host(x_host: torch.Tensor, packed: torch.Tensor, scales: torch.Tensor, y_host: torch.Tensor | None = None,
              x_dev: torch.Tensor | None = None, y_dev: torch.Tensor | None = None,
              workspace: torch.Tensor | None = None, weights_static: bool = False) -> torch.Tensor:
    """q4_gemv_host: x from host memory, y back to host memory, in one blocking call.

    ``x_host`` (CPU, float32 or bfloat16, [M,K]; pin it for an asynchronous copy) is copied
    to ``x_dev``, the product runs into ``y_dev`` and is copied to ``y_host`` (CPU f32 [M,N])
    before the call returns.  Staging buffers and the workspace are allocated here when not
    given (give them to keep allocation out of a loop)."""
    if x_host.dtype == torch.float32:
        xt = _lib.Q4_F32
    elif x_host.dtype == torch.bfloat16:
        xt = _lib.Q4_BF16
    else:
        raise TypeError("x_host must be float32 or bfloat16")
    if x_host.is_cuda or x_host.dim() != 2 or not x_host.is_contiguous():
        raise ValueError("x_host must be a contiguous 2-D CPU tensor")
    _need(packed, "packed", torch.uint8, 2)
    dev = packed.device
    _need(scales, "scales", torch.int16, 2, dev)
    M, K = x_host.shape
    N = packed.shape[0]
    if packed.shape[1] * 2 != K or tuple(scales.shape) != (N, K // 32):
        raise ValueError("shape mismatch between x_host, packed and scales")
    if y_host is None:
        y_host = torch.empty((M, N), dtype=torch.float32, pin_memory=True)
    elif y_host.is_cuda or y_host.dtype is not torch.float32 or tuple(y_host.shape) != (M, N) \
            or not y_host.is_contiguous():
        raise ValueError("y_host must be a contiguous float32 CPU tensor of shape (M, N)")
    if x_dev is None:
        x_dev = torch.empty((M, K), dtype=x_host.dtype, device=dev)
    _need(x_dev, "x_dev", x_host.dtype, 2, dev)
    if y_dev is None:
        y_dev = torch.empty((M, N), dtype=torch.float32, device=dev)
    _need(y_dev, "y_dev", torch.float32, 2, dev)
    lib = _lib.load()
    with _on(dev):
        if workspace is None:
            need = int(lib.q4_gemv_workspace_size(M, N, K))
            if need:
                workspace = torch.zeros(need, dtype=torch.uint8, device=dev)
        ws_ptr = workspace.data_ptr() if workspace is not None else None
        ws_bytes = workspace.numel() if workspace is not None else 0
        st = lib.q4_gemv_host(x_host.data_ptr(), xt, M, K, packed.data_ptr(), scales.data_ptr(), N,
                              y_host.data_ptr(), x_dev.data_ptr(), y_dev.data_ptr(),
                              _lib.WEIGHTS_STATIC if weights_static else 0, ws_ptr, ws_bytes, _stream())
    _lib.check(st, "q4_gemv_host")
    return y_host


def _mixed_array(weights, outs):
    arr = (_lib.MixedWeight * len(weights))()
    for i, ((codes, scales, bits), y) in enumerate(zip(weights, outs)):
        arr[i] = _lib.MixedWeight(codes.data_ptr(), scales.data_ptr(), codes.shape[0], y.data_ptr(), bits, 0)
    return arr


def gemv_mixed_workspace_size(M: int, K: int, Ns_bits) -> int:
    """Workspace bytes of gemv_mixed for matrices [(N, bits), ...]."""
    arr = (_lib.MixedWeight * len(Ns_bits))()
    for i, (n, bits) in enumerate(Ns_bits):
        arr[i] = _lib.MixedWeight(None, None, n, None, bits, 0)
    return int(_lib.load().q4_gemv_mixed_workspace_size(M, K, ctypes.cast(arr, ctypes.c_void_p), len(Ns_bits)))


def gemv_mixed(x: torch.Tensor, weights, outs=None, workspace: torch.Tensor | None = None,
               weights_static: bool = False):
    """y_i[M,N_i] (f32) = x . dequant(W_i)^T for matrices of mixed precision sharing x:
    ``weights`` is a list of (codes, scales, bits) with bits 4 (Q4: codes uint8 [N, K/2]) or
    8 (INT8: codes int8 [N, K]), scales binary16 bits as int16 [N, K/32]."""
    if x.dtype == torch.float32:
        xt = _lib.Q4_F32
    elif x.dtype == torch.bfloat16:
        xt = _lib.Q4_BF16
    else:
        raise TypeError("x must be float32 or bfloat16")
    _need(x, "x", x.dtype, 2)
    M, K = x.shape
    if not 1 <= len(weights) <= _lib.MULTI_MAX:
        raise ValueError(f"between 1 and {_lib.MULTI_MAX} weight matrices")
    for codes, scales, bits in weights:
        if bits == 4:
            _need(codes, "codes", torch.uint8, 2, x.device)
            if codes.shape[1] * 2 != K:
                raise ValueError("Q4 codes must be [N, K/2]")
        elif bits == 8:
            _need(codes, "codes", torch.int8, 2, x.device)
            if codes.shape[1] != K:
                raise ValueError("INT8 codes must be [N, K]")
        else:
            raise ValueError("bits must be 4 or 8")
        _need(scales, "scales", torch.int16, 2, x.device)
        if tuple(scales.shape) != (codes.shape[0], K // 32):
            raise ValueError("scales must be [N, K/32]")
    if outs is None:
        outs = [torch.empty((M, c.shape[0]), dtype=torch.float32, device=x.device) for c, _, _ in weights]
    for y, (c, _, _) in zip(outs, weights):
        _need(y, "out", torch.float32, 2, x.device)
        if tuple(y.shape) != (M, c.shape[0]):
            raise ValueError("out has the wrong shape")
    arr = _mixed_array(weights, outs)
    lib = _lib.load()
    with _on(x.device):
        if workspace is None:
            need = gemv_mixed_workspace_size(M, K, [(c.shape[0], b) for c, _, b in weights])
            if need:
                workspace = torch.zeros(need, dtype=torch.uint8, device=x.device)
        ws_ptr = workspace.data_ptr() if workspace is not None else None
        ws_bytes = workspace.numel() if workspace is not None else 0
        st = lib.q4_gemv_mixed(x.data_ptr(), xt, M, K, ctypes.cast(arr, ctypes.c_void_p), len(weights),
                               _lib.WEIGHTS_STATIC if weights_static else 0, ws_ptr, ws_bytes, _stream())
    _lib.check(st, "q4_gemv_mixed")
    return outs


def gemv_multi_workspace_size(M: int, K: int, Ns) -> int:
    arr = (ctypes.c_int64 * len(Ns))(*Ns)
    return int(_lib.load().q4_gemv_multi_workspace_size(M, K, ctypes.cast(arr, ctypes.c_void_p), len(Ns)))


def gemv_multi(x: torch.Tensor, weights, outs=None, workspace: torch.Tensor | None = None,
               weights_static: bool = False):
    """[y_i = x . dequant(W_i)^T for (packed_i, scales_i) in weights] in one launch.

    ``weights_static=True`` declares that no kernel still running on the stream writes
    these weights, so they may be streamed before the preceding kernel finishes.
    """
    if x.dtype == torch.float32:
        xt = _lib.Q4_F32
    elif x.dtype == torch.bfloat16:
        xt = _lib.Q4_BF16
    else:
        raise TypeError("x must be float32 or bfloat16")
    _need(x, "x", x.dtype, 2)
    M, K = x.shape
    if not 1 <= len(weights) <= _lib.MULTI_MAX:
        raise ValueError(f"between 1 and {_lib.MULTI_MAX} weight matrices")
    if outs is None:
        outs = [torch.empty((M, p.shape[0]), dtype=torch.float32, device=x.device) for p, _ in weights]
    arr = (_lib.Weight * len(weights))()
    for i, ((packed, scales), y) in enumerate(zip(weights, outs)):
        _need(packed, "packed", torch.uint8, 2, x.device)
        _need(scales, "scales", torch.int16, 2, x.device)
        _need(y, "out", torch.float32, 2, x.device)
        N = packed.shape[0]
        if packed.shape[1] * 2 != K or tuple(scales.shape) != (N, K // 32) or tuple(y.shape) != (M, N):
            raise ValueError("shape mismatch between x, packed, scales and out")
        arr[i] = _lib.Weight(packed.data_ptr(), scales.data_ptr(), N, y.data_ptr())
    if workspace is not None:
        _need(workspace, "workspace", torch.uint8, 1, x.device)
    lib = _lib.load()
    with _on(x.device):
        if workspace is None:
            need = gemv_multi_workspace_size(M, K, [p.shape[0] for p, _ in weights])
            if need:
                workspace = torch.zeros(need, dtype=torch.uint8, device=x.device)
        ws_ptr = workspace.data_ptr() if workspace is not None else None
        ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
        st = lib.q4_gemv_multi(x.data_ptr(), xt, M, K, ctypes.cast(arr, ctypes.c_void_p), len(weights),
                               _lib.WEIGHTS_STATIC if weights_static else 0, ws_ptr, ws_bytes, _stream())
    _lib.check(st, "q4_gemv_multi")
    return outs


def gemv_gate_up(x: torch.Tensor, gate, up, out: torch.Tensor | None = None, weights_static: bool = False):
    """y[M,N] (f32) = silu(x . dequant(Wg)^T) * (x . dequant(Wu)^T) in one launch.

    gate, up: (packed, scales) of equal shapes.  K must be a multiple of 256; x is f32
    (M == 1) or bf16 (M <= 16).  SiLU(g) = g / (1 + exp(-g)).
    """
    if x.dtype is torch.float32:
        xt = _lib.Q4_F32
    elif x.dtype is torch.bfloat16:
        xt = _lib.Q4_BF16
    else:
        raise TypeError("x must be float32 or bfloat16")
    _need(x, "x", x.dtype, 2)
    (gp, gs), (upk, us) = gate, up
    for t, name, dt in ((gp, "gate packed", torch.uint8), (gs, "gate scales", torch.int16),
                        (upk, "up packed", torch.uint8), (us, "up scales", torch.int16)):
        _need(t, name, dt, 2, x.device)
    M, K = x.shape
    N = gp.shape[0]
    if gp.shape[1] * 2 != K or tuple(gs.shape) != (N, K // 32) or gp.shape != upk.shape or gs.shape != us.shape:
        raise ValueError("shape mismatch between x, gate and up")
    if out is None:
        out = torch.empty((M, N), dtype=torch.float32, device=x.device)
    else:
        _need(out, "out", torch.float32, 2, x.device)
        if tuple(out.shape) != (M, N):
            raise ValueError("out has the wrong shape")
    with _on(x.device):
        st = _lib.load().q4_gemv_gate_up(x.data_ptr(), xt, M, K, gp.data_ptr(), gs.data_ptr(), upk.data_ptr(),
                                         us.data_ptr(), N, out.data_ptr(),
                                         _lib.WEIGHTS_STATIC if weights_static else 0, _stream())
    _lib.check(st, "q4_gemv_gate_up")
    return out


def gemv_argmax(x: torch.Tensor, packed: torch.Tensor, scales: torch.Tensor, logits: bool = False,
                workspace: torch.Tensor | None = None, weights_static: bool = False):
    """Greedy LM-head step in one launch: (index int64 [M], value f32 [M], y or None) with
    index[m] the row of the largest logit of x[m] . dequant(W)^T (lowest row on ties).

    ``logits=True`` also returns the f32 logits [M,N].  ``workspace`` (uint8, zero before
    its first use, left zero by every call) is allocated here when not given; calls in
    flight at the same time on different streams need their own.
    """
    if x.dtype is torch.float32:
        xt = _lib.Q4_F32
    elif x.dtype is torch.bfloat16:
        xt = _lib.Q4_BF16
    else:
        raise TypeError("x must be float32 or bfloat16")
    _need(x, "x", x.dtype, 2)
    _need(packed, "packed", torch.uint8, 2, x.device)
    _need(scales, "scales", torch.int16, 2, x.device)
    M, K = x.shape
    N = packed.shape[0]
    if packed.shape[1] * 2 != K or tuple(scales.shape) != (N, K // 32):
        raise ValueError("shape mismatch between x, packed and scales")
    lib = _lib.load()
    index = torch.empty((M,), dtype=torch.int64, device=x.device)
    value = torch.empty((M,), dtype=torch.float32, device=x.device)
    y = torch.empty((M, N), dtype=torch.float32, device=x.device) if logits else None
    if workspace is None:
        workspace = torch.zeros(int(lib.q4_gemv_argmax_workspace_size()), dtype=torch.uint8, device=x.device)
    else:
        _need(workspace, "workspace", torch.uint8, 1, x.device)
    with _on(x.device):
        st = lib.q4_gemv_argmax(x.data_ptr(), xt, M, K, packed.data_ptr(), scales.data_ptr(), N,
                                y.data_ptr() if y is not None else None, index.data_ptr(), value.data_ptr(),
                                _lib.WEIGHTS_STATIC if weights_static else 0, workspace.data_ptr(),
                                workspace.numel(), _stream())
    _lib.check(st, "q4_gemv_argmax")
    return index, value, y


def gemv_topk(x: torch.Tensor, packed: torch.Tensor, scales: torch.Tensor, k: int, row_base: int = 0,
              logits: bool = False, workspace: torch.Tensor | None = None, weights_static: bool = False):
    """The k largest logits of an LM head per x row in one launch: (index int64 [M,k],
    value f32 [M,k], y or None), larger first, the lower row on ties, rows reported as
    ``row_base`` + row; past N rows the lists hold -1 / NaN.

    ``logits=True`` also returns the f32 logits [M,N].  ``workspace`` (uint8, its first
    16 bytes zero before its first use and left zero by every call, at least
    ``gemv_topk_workspace_size`` bytes) is allocated here when not given.
    """
    if x.dtype is torch.float32:
        xt = _lib.Q4_F32
    elif x.dtype is torch.bfloat16:
        xt = _lib.Q4_BF16
    else:
        raise TypeError("x must be float32 or bfloat16")
    _need(x, "x", x.dtype, 2)
    _need(packed, "packed", torch.uint8, 2, x.device)
    _need(scales, "scales", torch.int16, 2, x.device)
    M, K = x.shape
    N = packed.shape[0]
    if packed.shape[1] * 2 != K or tuple(scales.shape) != (N, K // 32):
        raise ValueError("shape mismatch between x, packed and scales")
    lib = _lib.load()
    index = torch.empty((M, k), dtype=torch.int64, device=x.device)
    value = torch.empty((M, k), dtype=torch.float32, device=x.device)
    y = torch.empty((M, N), dtype=torch.float32, device=x.device) if logits else None
    with _on(x.device):
        if workspace is None:
            size = int(lib.q4_gemv_topk_workspace_size(M, N, K, k, xt)) if M and N else 16
            workspace = torch.zeros(max(size, 16), dtype=torch.uint8, device=x.device)
        else:
            _need(workspace, "workspace", torch.uint8, 1, x.device)
        st = lib.q4_gemv_topk(x.data_ptr(), xt, M, K, packed.data_ptr(), scales.data_ptr(), N, k, row_base,
                              y.data_ptr() if y is not None else None, index.data_ptr(), value.data_ptr(),
                              _lib.WEIGHTS_STATIC if weights_static else 0, workspace.data_ptr(),
                              workspace.numel(), _stream())
    _lib.check(st, "q4_gemv_topk")
    if N == 0:                         # no rows: the lists are all padding
        index.fill_(-1)
        value.fill_(float("nan"))
    return index, value, y


def topk_merge(values: torch.Tensor, indices: torch.Tensor, k: int):
    """The k best entries per x row over S top-k lists (values f32 [S,M,k], indices int64
    [S,M,k], as gathered from the shards of an LM head), ordered as ``gemv_topk`` orders
    them: (index int64 [M,k], value f32 [M,k])."""
    _need(values, "values", torch.float32, 3)
    _need(indices, "indices", torch.int64, 3, values.device)
    if tuple(values.shape) != tuple(indices.shape):
        raise ValueError("values and indices must have the same shape")
    S, M, kin = values.shape
    if kin != k:
        raise ValueError("the lists must hold k entries each")
    index = torch.empty((M, k), dtype=torch.int64, device=values.device)
    value = torch.empty((M, k), dtype=torch.float32, device=values.device)
    with _on(values.device):
        st = _lib.load().q4_topk_merge(values.data_ptr(), indices.data_ptr(), S, M, k, index.data_ptr(),
                                       value.data_ptr(), _stream())
    _lib.check(st, "q4_topk_merge")
    return index, value


def gemv_topk_workspace_size(M: int, N: int, K: int, k: int, x_dtype: torch.dtype = torch.bfloat16) -> int:
    """Bytes of workspace ``gemv_topk`` needs on the current device (0: shape not served)."""
    xt = _lib.Q4_F32 if x_dtype is torch.float32 else _lib.Q4_BF16
    return int(_lib.load().q4_gemv_topk_workspace_size(M, N, K, k, xt))


def f16_gemv(x: torch.Tensor, w: torch.Tensor, out: torch.Tensor | None = None, weights_static: bool = False):
    """y[M,N] (f32) = x[M,K] . W^T for binary16 weights W [N,K] (torch.float16), on the
    tensor cores; x is f32 (M == 1) or bf16 (M <= 16), K a multiple of 8."""
    if x.dtype is torch.float32:
        xt = _lib.Q4_F32
    elif x.dtype is torch.bfloat16:
        xt = _lib.Q4_BF16
    else:
        raise TypeError("x must be float32 or bfloat16")
    _need(x, "x", x.dtype, 2)
    _need(w, "w", torch.float16, 2, x.device)
    M, K = x.shape
    N = w.shape[0]
    if w.shape[1] != K:
        raise ValueError("shape mismatch between x and w")
    if out is None:
        out = torch.empty((M, N), dtype=torch.float32, device=x.device)
    else:
        _need(out, "out", torch.float32, 2, x.device)
        if tuple(out.shape) != (M, N):
            raise ValueError("out has the wrong shape")
    with _on(x.device):
        st = _lib.load().q4_f16_gemv(x.data_ptr(), xt, M, K, w.data_ptr(), N, out.data_ptr(),
                                     _lib.WEIGHTS_STATIC if weights_static else 0, _stream())
    _lib.check(st, "q4_f16_gemv")
    return out


class GemvMulti:
    """A prepared ``gemv_multi`` for a decode loop: the weights, outputs and workspace are
    checked once, and each call checks only x before the launch.

    The tensors are held by reference; their storage must not be replaced (``set_``,
    ``resize_``) while the object is in use.
    """

    def __init__(self, weights, M: int, K: int, x_dtype: torch.dtype, outs=None,
                 workspace: torch.Tensor | None = None, weights_static: bool = False):
        if x_dtype is torch.float32:
            self._xt = _lib.Q4_F32
        elif x_dtype is torch.bfloat16:
            self._xt = _lib.Q4_BF16
        else:
            raise TypeError("x must be float32 or bfloat16")
        if not 1 <= len(weights) <= _lib.MULTI_MAX:
            raise ValueError(f"between 1 and {_lib.MULTI_MAX} weight matrices")
        dev = weights[0][0].device
        if outs is None:
            outs = [torch.empty((M, p.shape[0]), dtype=torch.float32, device=dev) for p, _ in weights]
        self._arr = (_lib.Weight * len(weights))()
        for i, ((packed, scales), y) in enumerate(zip(weights, outs)):
            _need(packed, "packed", torch.uint8, 2, dev)
            _need(scales, "scales", torch.int16, 2, dev)
            _need(y, "out", torch.float32, 2, dev)
            N = packed.shape[0]
            if packed.shape[1] * 2 != K or tuple(scales.shape) != (N, K // 32) or tuple(y.shape) != (M, N):
                raise ValueError("shape mismatch between x, packed, scales and out")
            self._arr[i] = _lib.Weight(packed.data_ptr(), scales.data_ptr(), N, y.data_ptr())
        with _on(dev):
            if workspace is None:
                need = gemv_multi_workspace_size(M, K, [p.shape[0] for p, _ in weights])
                if need:
                    workspace = torch.zeros(need, dtype=torch.uint8, device=dev)
        if workspace is not None:
            _need(workspace, "workspace", torch.uint8, 1, dev)
        self._keep = (weights, workspace)
        self._vp = ctypes.cast(self._arr, ctypes.c_void_p)
        self._ws = workspace.data_ptr() if workspace is not None else None
        self._wsb = workspace.numel() if workspace is not None else 0
        self._count = len(weights)
        self._flags = _lib.WEIGHTS_STATIC if weights_static else 0
        self._shape = (M, K)
        self._dtype = x_dtype
        self.device = dev
        self.outs = outs
        self._lib = _lib.load()

    def __call__(self, x: torch.Tensor):
        """Launch on the current stream; returns the output list given at construction."""
        if not isinstance(x, torch.Tensor) or x.dtype is not self._dtype:
            raise TypeError(f"x must be a {self._dtype} tensor")
        if x.device != self.device or x.shape != self._shape or not x.is_contiguous():
            raise ValueError(f"x must be a contiguous {self._shape} tensor on {self.device}")
        with _on(self.device):
            st = self._lib.q4_gemv_multi(x.data_ptr(), self._xt, self._shape[0], self._shape[1], self._vp,
                                         self._count, self._flags, self._ws, self._wsb, _stream())
        _lib.check(st, "q4_gemv_multi")
        return self.outs

    def host_step(self, x_host: torch.Tensor, y_host, y_dev: torch.Tensor | None = None):
        """One decode step fed from pinned host memory, captured as a CUDA graph: x_host ->
        device, the GEMVs, the outputs -> pinned host memory.  ``y_host`` is a list of
        pinned tensors, one per output, or, with ``y_dev`` (a device tensor whose storage
        holds every output), one pinned tensor of y_dev's shape that receives it in one
        copy.  Returns a callable that replays the step on the current stream; the caller
        synchronizes before reading y_host.  The host tensors are held by reference."""
        if not (x_host.is_pinned() and x_host.dtype is self._dtype and tuple(x_host.shape) == self._shape):
            raise ValueError(f"x_host must be a pinned {self._dtype} tensor of shape {self._shape}")
        if y_dev is not None:
            if not (isinstance(y_host, torch.Tensor) and y_host.is_pinned() and y_host.shape == y_dev.shape
                    and y_host.dtype is y_dev.dtype and y_dev.device == self.device):
                raise ValueError("y_host must be a pinned tensor shaped like y_dev")
            base, end = y_dev.data_ptr(), y_dev.data_ptr() + y_dev.numel() * y_dev.element_size()
            if any(not base <= o.data_ptr() < end for o in self.outs):
                raise ValueError("every output must lie in y_dev")
            pairs = [(y_host, y_dev)]
        else:
            if len(y_host) != len(self.outs) or any(not (h.is_pinned() and h.shape == o.shape and h.dtype is o.dtype)
                                                    for h, o in zip(y_host, self.outs)):
                raise ValueError("y_host must hold one pinned tensor per output, shaped like it")
            pairs = list(zip(y_host, self.outs))
        x_dev = torch.empty(self._shape, dtype=self._dtype, device=self.device)
        graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(device=self.device)
        with _on(self.device), torch.cuda.stream(side):
            self(x_dev)                                   # the launch works before it is captured
            side.synchronize()
            with torch.cuda.graph(graph, stream=side):
                x_dev.copy_(x_host, non_blocking=True)
                self(x_dev)
                for h, d in pairs:
                    h.copy_(d, non_blocking=True)
        keep = (x_host, y_host, x_dev, graph)

        def replay():
            keep[3].replay()
        return replay


def gemm(x: torch.Tensor, packed: torch.Tensor, scales: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
    """y[M,N] (bf16) = x[M,K] (bf16) . dequant(W)^T on the tensor cores (prefill)."""
    _need(x, "x", torch.bfloat16, 2)
    _need(packed, "packed", torch.uint8, 2, x.device)
    _need(scales, "scales", torch.int16, 2, x.device)
    M, K = x.shape
    N = packed.shape[0]
    if packed.shape[1] * 2 != K or tuple(scales.shape) != (N, K // 32):
        raise ValueError("shape mismatch between x, packed and scales")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    else:
        _need(out, "out", torch.bfloat16, 2, x.device)
        if tuple(out.shape) != (M, N):
            raise ValueError("out has the wrong shape")
    with _on(x.device):
        st = _lib.load().q4_gemm(x.data_ptr(), M, K, packed.data_ptr(), scales.data_ptr(), N, out.data_ptr(),
                                 _stream())
    _lib.check(st, "q4_gemm")
    return out
