"""Python binding of libcq, the B200 CubicQuant weight-only GEMM library.

This module only marshals arguments: every step of the computation runs in
the CUDA kernels of ``libcq.so`` (built in-tree by ``build.py``).  There is
no CPU fallback; if the library is missing or a call fails, an exception is
raised.  PyTorch is used for device memory and streams.

The calls mirror ``include/cq.h``:

* ``cq_pack(codes, B)``                         -> packed [N][K*B/8] uint8
* ``cq_decode(packed, scales, ab, K, B, G)``    -> W [N][K] (float32 / bfloat16)
* ``cq_gemm(x, packed, scales, ab, N, K, B, G)`` -> y [M][N] (or [M][N/2])
* ``cq_moe_grouped_gemm(tokens, topk_ids, ...)`` -> per-route / combined outputs
"""
from __future__ import annotations

import contextlib
import ctypes
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libcq.so")

MIDRISE, MIDTREAD = 0, 1
F32, BF16 = 0, 1
EPI_NONE, EPI_SWIGLU = 0, 1

_STATUS = {
    0: "ok", 1: "invalid argument", 2: "unsupported", 3: "CUDA runtime error",
    4: "a bounded device wait ran out", 5: "workspace missing or too small",
}


class CQError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: libcq status {status} ({_STATUS.get(status, '?')})")
        self.status = status


_lib = None


class MatrixDesc(ctypes.Structure):
    _fields_ = [("packed", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("ab", ctypes.c_void_p), ("B", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class ExpertDesc(ctypes.Structure):
    _fields_ = [("gate_up", MatrixDesc), ("down", MatrixDesc)]


def lib():
    """Load libcq.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"libcq.so not found at {LIB_PATH}; build it with "
            "`python -m bit_non_uniform_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, i64, i32, sz, u64 = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t,
                            ctypes.c_uint64)
    sigs = {
        "cq_version": (i32, []),
        "cq_status_string": (ctypes.c_char_p, [i32]),
        "cq_pack": (i32, [P, i64, i64, i32, P, P]),
        "cq_decode": (i32, [P, P, P, i64, i64, i32, i32, i32, i32, P, P]),
        "cq_gemm_workspace_size": (sz, [i64, i64, i64, i32, i32, i32]),
        "cq_gemm": (i32, [P, i64, P, P, P, i64, i64, i32, i32, i32, i32, i32, P, P, sz, P]),
        "cq_moe_layer_bytes": (sz, [i32]),
        "cq_moe_prepare_layer": (i32, [P, i32, i64, i64, i32, P]),
        "cq_moe_workspace_size": (sz, [i64, i32, i32, i64, i64, i32]),
        "cq_moe_grouped_gemm": (i32, [P, i64, P, P, i32, i32, P, i64, i64, i32, i32, i32,
                                      P, P, P, sz, P]),
        "cq_gemm_noalloc": (i32, [P, i64, P, P, P, i64, i64, i32, i32, i32, i32, i32, P, P]),
        "cq_gemm_host": (i32, [P, i64, P, P, P, i64, i64, i32, i32, i32, i32, i32, P, P, P, P,
                               sz, P]),
        "cq_get_device_error": (i32, [P, ctypes.POINTER(ctypes.c_int)]),
        "cq_test_gemm_bounded": (i32, [P, i64, P, P, P, i64, i64, i32, i32, P, P, sz, u64,
                                       i32, P]),
        "cq_test_gemm_path_workspace_size": (sz, [i64, i64, i64, i32, i32, i32, i32]),
        "cq_quant_rows": (i32, [P, i64, i64, P, P, P]),
        "cq_gemm_a8_workspace_size": (sz, [i64, i64, i64, i32, i32, i32]),
        "cq_gemm_a8": (i32, [P, i64, P, P, P, i64, i64, i32, i32, i32, i32, i32, P, P, sz, P]),
        "cq_test_gemm_path": (i32, [P, i64, P, P, P, i64, i64, i32, i32, i32, i32, i32, P, P,
                                    sz, i32, P]),
    }
    for name, (res, args) in sigs.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    _lib = L
    return L


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _on_stream(stream=None):
    """Allocations and fills of a binding call go on the call's stream, so
    that the buffers it creates are ready (and are recycled) in that
    stream's order."""
    return torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext()


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(st: int, where: str):
    if st != 0:
        raise CQError(st, where)


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("libcq works on CUDA tensors only")


def version() -> int:
    return int(lib().cq_version())


def cq_pack(codes: torch.Tensor, B: int, out: torch.Tensor | None = None, stream=None):
    """codes uint8 [N][K] (CUDA) -> packed uint8 [N][K*B/8]."""
    with _on_stream(stream):
        _need_cuda(codes)
        codes = codes.contiguous()
        N, K = codes.shape
        if out is None:
            out = torch.empty((N, K * B // 8), dtype=torch.uint8, device=codes.device)
        _check(lib().cq_pack(_ptr(codes), N, K, B, _ptr(out), _stream(stream)), "cq_pack")
        return out


def cq_decode(packed, scales, ab, K: int, B: int, G: int, mode: int = MIDRISE,
              out_dtype: int = F32, stream=None):
    """Decode packed codes + (s, a, b) into W [N][K] (float32 or bfloat16)."""
    with _on_stream(stream):
        _need_cuda(packed, scales, ab)
        N = packed.shape[0]
        dt = torch.float32 if out_dtype == F32 else torch.bfloat16
        W = torch.empty((N, K), dtype=dt, device=packed.device)
        _check(lib().cq_decode(_ptr(packed), _ptr(scales), _ptr(ab), N, K, B, G, mode, out_dtype,
                               _ptr(W), _stream(stream)), "cq_decode")
        return W


def gemm_workspace_size(M, N, K, B, G, epilogue=EPI_NONE) -> int:
    return int(lib().cq_gemm_workspace_size(M, N, K, B, G, epilogue))


def gemm_workspace(M, N, K, B, G, epilogue=EPI_NONE, device="cuda"):
    """A zero-initialised workspace buffer for cq_gemm."""
    n = gemm_workspace_size(M, N, K, B, G, epilogue)
    return torch.zeros(max(n, 16), dtype=torch.uint8, device=device)


def cq_gemm(x, packed, scales, ab, N: int, K: int, B: int, G: int, mode: int = MIDRISE,
            epilogue: int = EPI_NONE, out_dtype: int = F32, workspace=None, out=None,
            stream=None):
    """y = x W^T with W given packed; x bfloat16 [M][K]."""
    with _on_stream(stream):
        _need_cuda(x, packed, scales, ab)
        assert x.dtype == torch.bfloat16 and x.is_contiguous()
        M = x.shape[0]
        ncol = N // 2 if epilogue == EPI_SWIGLU else N
        if out is None:
            dt = torch.float32 if out_dtype == F32 else torch.bfloat16
            out = torch.empty((M, ncol), dtype=dt, device=x.device)
        if workspace is None:
            workspace = gemm_workspace(M, N, K, B, G, epilogue, x.device)
        _check(lib().cq_gemm(_ptr(x), M, _ptr(packed), _ptr(scales), _ptr(ab), N, K, B, G, mode,
                             epilogue, out_dtype, _ptr(out), _ptr(workspace),
                             workspace.numel() * workspace.element_size(), _stream(stream)),
               "cq_gemm")
        return out


# kernels of cq_gemm (test hook cq_test_gemm_path)
PATH_AUTO, PATH_NARROW, PATH_GEMV, PATH_ENGINE = 0, 1, 2, 3


def gemm_on_path(path: int, x, packed, scales, ab, N: int, K: int, B: int, G: int,
                 mode: int = MIDRISE, epilogue: int = EPI_NONE, out_dtype: int = F32,
                 stream=None):
    """cq_gemm on a chosen kernel (a test hook); raises CQError with status 2
    when that kernel does not take the problem."""
    with _on_stream(stream):
        _need_cuda(x, packed, scales, ab)
        M = x.shape[0]
        ncol = N // 2 if epilogue == EPI_SWIGLU else N
        dt = torch.float32 if out_dtype == F32 else torch.bfloat16
        out = torch.empty((M, ncol), dtype=dt, device=x.device)
        n = int(lib().cq_test_gemm_path_workspace_size(M, N, K, B, G, epilogue, path))
        ws = torch.zeros(max(n, 16), dtype=torch.uint8, device=x.device)
        _check(lib().cq_test_gemm_path(_ptr(x), M, _ptr(packed), _ptr(scales), _ptr(ab), N, K, B, G,
                                       mode, epilogue, out_dtype, _ptr(out), _ptr(ws), ws.numel(),
                                       path, _stream(stream)), "cq_test_gemm_path")
        return out


def cq_gemm_host(x_host, packed, scales, ab, N: int, K: int, B: int, G: int,
                 mode: int = MIDRISE, epilogue: int = EPI_NONE, out_dtype: int = F32,
                 y_host=None, x_dev=None, y_dev=None, workspace=None, stream=None):
    """cq_gemm with x and y in host memory (pinned CPU tensors keep the
    copies asynchronous): the copies and the GEMM are queued on `stream`;
    synchronize it before reading y_host."""
    with _on_stream(stream):
        _need_cuda(packed, scales, ab)
        assert x_host.device.type == "cpu" and x_host.dtype == torch.bfloat16
        assert x_host.is_contiguous()
        M = x_host.shape[0]
        dev = packed.device
        ncol = N // 2 if epilogue == EPI_SWIGLU else N
        dt = torch.float32 if out_dtype == F32 else torch.bfloat16
        if y_host is None:
            y_host = torch.empty((M, ncol), dtype=dt).pin_memory()
        if x_dev is None:
            x_dev = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
        if y_dev is None:
            y_dev = torch.empty((M, ncol), dtype=dt, device=dev)
        if workspace is None:
            workspace = gemm_workspace(M, N, K, B, G, epilogue, dev)
        _check(lib().cq_gemm_host(x_host.data_ptr(), M, _ptr(packed), _ptr(scales), _ptr(ab), N, K,
                                  B, G, mode, epilogue, out_dtype, y_host.data_ptr(), _ptr(x_dev),
                                  _ptr(y_dev), _ptr(workspace), workspace.numel(), _stream(stream)),
               "cq_gemm_host")
        return y_host


def cq_gemm_noalloc(x, packed, scales, ab, N: int, K: int, B: int, G: int,
                    mode: int = MIDRISE, epilogue: int = EPI_NONE, out_dtype: int = F32,
                    out=None, stream=None):
    """cq_gemm without a workspace (scratch in libcq's fixed array; M <= 16)."""
    with _on_stream(stream):
        _need_cuda(x, packed, scales, ab)
        M = x.shape[0]
        ncol = N // 2 if epilogue == EPI_SWIGLU else N
        if out is None:
            dt = torch.float32 if out_dtype == F32 else torch.bfloat16
            out = torch.empty((M, ncol), dtype=dt, device=x.device)
        _check(lib().cq_gemm_noalloc(_ptr(x), M, _ptr(packed), _ptr(scales), _ptr(ab), N, K, B, G,
                                     mode, epilogue, out_dtype, _ptr(out), _stream(stream)),
               "cq_gemm_noalloc")
        return out


def gemm_a8_workspace_size(M, N, K, B, G, epilogue=EPI_NONE) -> int:
    return int(lib().cq_gemm_a8_workspace_size(M, N, K, B, G, epilogue))


def cq_quant_rows(x, stream=None):
    """Per-row dynamic INT8 quantization: (xq int8 [M][K], absmax f32 [M])."""
    with _on_stream(stream):
        _need_cuda(x)
        assert x.dtype == torch.bfloat16 and x.is_contiguous()
        M, K = x.shape
        xq = torch.empty((M, K), dtype=torch.int8, device=x.device)
        absmax = torch.empty(M, dtype=torch.float32, device=x.device)
        _check(lib().cq_quant_rows(_ptr(x), M, K, _ptr(xq), _ptr(absmax), _stream(stream)),
               "cq_quant_rows")
        return xq, absmax


def cq_gemm_a8(x, packed, scales, ab, N: int, K: int, B: int, G: int, mode: int = MIDRISE,
               epilogue: int = EPI_NONE, out_dtype: int = F32, out=None, workspace=None,
               stream=None):
    """Dynamic-A8 y = x W^T: x quantized per row to INT8 inside the call."""
    with _on_stream(stream):
        _need_cuda(x, packed, scales, ab)
        assert x.dtype == torch.bfloat16 and x.is_contiguous()
        M = x.shape[0]
        ncol = N // 2 if epilogue == EPI_SWIGLU else N
        if out is None:
            dt = torch.float32 if out_dtype == F32 else torch.bfloat16
            out = torch.empty((M, ncol), dtype=dt, device=x.device)
        if workspace is None:
            n = gemm_a8_workspace_size(M, N, K, B, G, epilogue)
            workspace = torch.empty(max(n, 256), dtype=torch.uint8, device=x.device)
        _check(lib().cq_gemm_a8(_ptr(x), M, _ptr(packed), _ptr(scales), _ptr(ab), N, K, B, G, mode,
                                epilogue, out_dtype, _ptr(out), _ptr(workspace),
                                workspace.numel(), _stream(stream)), "cq_gemm_a8")
        return out


def moe_workspace_size(T, k, E, H, I, G) -> int:
    return int(lib().cq_moe_workspace_size(T, k, E, H, I, G))


def moe_prepare_layer(experts, H: int, I: int, G: int, device="cuda"):
    """Build the device-side layer table (TMA descriptors + operand
    descriptions) for a list of per-expert dicts with keys packed_gu,
    scales_gu, ab_gu, B_gu, packed_dn, scales_dn, ab_dn, B_dn (CUDA tensors).
    Returns the table (a uint8 CUDA tensor the caller keeps alive)."""
    E = len(experts)
    arr = (ExpertDesc * E)()
    for e, ex in enumerate(experts):
        for fld, key in (("gate_up", "gu"), ("down", "dn")):
            d = getattr(arr[e], fld)
            d.packed = ex[f"packed_{key}"].data_ptr()
            d.scales = ex[f"scales_{key}"].data_ptr()
            d.ab = ex[f"ab_{key}"].data_ptr()
            d.B = int(ex[f"B_{key}"])
            d.reserved = 0
    nbytes = int(lib().cq_moe_layer_bytes(E))
    table = torch.empty(nbytes + 64, dtype=torch.uint8, device=device)
    off = (-table.data_ptr()) % 64
    table = table[off:off + nbytes]
    _check(lib().cq_moe_prepare_layer(ctypes.cast(arr, ctypes.c_void_p), E, H, I, G,
                                      _ptr(table)), "cq_moe_prepare_layer")
    return table


def moe_workspace(T, k, E, H, I, G, device="cuda"):
    n = moe_workspace_size(T, k, E, H, I, G)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device)


def cq_moe_grouped_gemm(tokens, topk_ids, topk_w, layer, E: int, H: int, I: int, G: int,
                        mode: int = MIDRISE, out_dtype: int = F32, route_out=True,
                        combine=True, workspace=None, stream=None):
    """Routed-expert FFN of one MoE layer.  Returns (route_out, out)."""
    with _on_stream(stream):
        _need_cuda(tokens, topk_ids, layer)
        T, k = topk_ids.shape
        ro = None
        if route_out is True:
            ro = torch.empty((T * k, H), dtype=torch.float32, device=tokens.device)
        elif route_out is not None and route_out is not False:
            ro = route_out
        out = None
        if combine:
            dt = torch.float32 if out_dtype == F32 else torch.bfloat16
            out = torch.empty((T, H), dtype=dt, device=tokens.device)
        if workspace is None:
            workspace = moe_workspace(T, k, E, H, I, G, tokens.device)
        _check(lib().cq_moe_grouped_gemm(
            _ptr(tokens), T, _ptr(topk_ids), _ptr(topk_w) if topk_w is not None else None, k, E,
            _ptr(layer), H, I, G, mode, out_dtype, _ptr(ro), _ptr(out), _ptr(workspace),
            workspace.numel(), _stream(stream)), "cq_moe_grouped_gemm")
        return ro, out


def device_error(stream=None) -> tuple[int, int]:
    """(status, site) of the device error word; clears it."""
    site = ctypes.c_int(0)
    st = lib().cq_get_device_error(_stream(stream), ctypes.byref(site))
    return int(st), int(site.value)
